// Prefill-chunk GEMM with Q4_0 weights on the 5th-generation tensor cores (tcgen05):
//   Y[t, n] = sum_k X[t, k] * W[n, k],   X fp16 [tokens x k] (tokens <= 128), W Q4_0 [n x k],
//   fp32 accumulation in tensor memory, Y fp16 (round to nearest even).
//
// Source: TurboFieldfare wiki, "메모리·전문가 스트리밍" (prefill in chunks of at most 128 tokens,
// so that each weight read is reused by every prompt row of the chunk); Camelid README,
// "Engine status" (GPU-resident single-shot prefill).
//
// One CTA computes a 128 (tokens, padded) x 128 (output features) tile over a range of k.
//   warp 0     TMA: X tiles (128 rows x 64 k, fp16, 128-byte swizzle; 5-deep ring) and raw Q4_0
//              row chunks (128 rows x 144 bytes = 256 k; 3-deep ring) into shared memory.
//   warp 1     allocates the 128-column fp32 accumulator in tensor memory and issues the
//              tcgen05.mma instructions (M=128, N=128, K=16 each, both operands K-major in
//              shared memory); tcgen05.commit frees each stage when its MMAs have read it.
//   warps 2-5  dequantize: each thread owns one weight row, turns 64 Q4_0 weights into fp16
//              (q - 8) * d (exact nibble, one rounding of the product) and writes them into the
//              B stage in the swizzled K-major layout the MMA reads; after the last stage they
//              read the accumulator rows (one warp per 32 tensor-memory lanes), round to fp16
//              and store Y.
// With several k-splits per tile (small n), the CTAs of one tile form a thread-block cluster
// and the partial tiles are summed through distributed shared memory in a fixed order.
// BQG_PF_ISSUERS (1, 2, 4: MMA-issuing warps, each with its own partial accumulator over a
// share of the k steps) and BQG_PF_DQ_WARPS (4, 8: a thread per row, or per row and block) are
// build-time choices; 1 and 4 measured best (2/4 issuers and 8 dequant warps: 32.6-35.2 us
// against 32.9 us at n = 14336).  Launched as a dependent launch: the next kernel's prologue
// overlaps this one's tail.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "host_common.h"
#include "tcgen05.cuh"

namespace bqg {

#ifndef BQG_PF_ISSUERS
#define BQG_PF_ISSUERS 1
#endif
#ifndef BQG_PF_DQ_WARPS
#define BQG_PF_DQ_WARPS 4
#endif
constexpr int kPfIssuers = BQG_PF_ISSUERS;   // MMA-issuing warps = partial accumulators (k steps split)
constexpr int kPfDqWarps = BQG_PF_DQ_WARPS;  // 4: a thread per weight row; 8: a thread per row and block
static_assert(kPfIssuers == 1 || kPfIssuers == 2 || kPfIssuers == 4, "1, 2 or 4 issuers");
static_assert(kPfDqWarps == 4 || kPfDqWarps == 8, "4 or 8 dequant warps");
constexpr int kPfDqThreads = 32 * kPfDqWarps;
constexpr int kPfWarpIss2 = 2 + kPfDqWarps;  // first extra issuer warp
constexpr int kPfThreads = 32 * (2 + kPfDqWarps + kPfIssuers - 1);
constexpr int kPfTileN = 128;             // output features per CTA
constexpr int kPfTileM = 128;             // tokens per CTA (MMA M)
constexpr int kPfStageK = 64;             // k per stage (one 128-byte swizzle row of fp16)
constexpr int kPfStages = 5;              // A/B stage ring depth
constexpr int kPfRawK = 256;              // k per raw Q4_0 chunk (8 blocks = 144 bytes per row)
constexpr int kPfRawBytesRow = kPfRawK / 32 * 18;  // 144
constexpr int kPfRawStages = 3;
constexpr int kPfABytes = kPfTileM * kPfStageK * 2;  // 16 KB
constexpr int kPfBBytes = kPfTileN * kPfStageK * 2;  // 16 KB
constexpr int kPfRawBytes = kPfTileN * kPfRawBytesRow;  // 18 KB
constexpr int kPfMaxSplit = 8;            // k-splits per tile (cluster size)
// smem: [A ring | B ring] (1024-aligned), raw ring, barriers, tmem address; + 1 KB alignment slack
constexpr size_t kPfSmemBytes = 1024 + size_t(kPfStages) * (kPfABytes + kPfBBytes) +
                                size_t(kPfRawStages) * kPfRawBytes + 256;
static_assert(kPfSmemBytes <= 227 * 1024, "prefill shared memory");
static_assert(size_t(kPfStages) * kPfABytes >= size_t(kPfTileN + 4) * kPfTileM * 4, "split-k partial tile parks in the A ring");
static_assert((2 * kPfStages + 2 * kPfRawStages + 1) * 8 + 8 <= 256, "barrier area");

struct PfParams {
  void* Y;           // fp16 [tokens x n]
  int tokens, n, k;
  int ksplit;        // CTAs (cluster size) sharing one output tile
  int kchunks;       // k / kPfRawK; split s owns chunks [s*kchunks/ksplit, (s+1)*kchunks/ksplit)
};

// 16 accumulator columns of this warp's lanes, the kPfIssuers partials (kPfTileN columns apart)
// added in a fixed order.
__device__ __forceinline__ void pf_acc16(uint32_t taddr, float (&o)[16]) {
  uint32_t v[16];
  tmem_ld16(taddr, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = __uint_as_float(v[i]);
#pragma unroll
  for (int p = 1; p < kPfIssuers; ++p) {
    tmem_ld16(taddr + uint32_t(p * kPfTileN), v);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] += __uint_as_float(v[i]);
  }
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kPfThreads, 1)
    k_prefill_q4(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                 const __grid_constant__ PfParams prm) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled operand tiles
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_s & 1023)) & 1023);
  uint8_t* a_ring = smem;                                        // kPfStages x 16 KB
  uint8_t* b_ring = a_ring + size_t(kPfStages) * kPfABytes;     // kPfStages x 16 KB
  uint8_t* w_ring = b_ring + size_t(kPfStages) * kPfBBytes;     // kPfRawStages x 18 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(w_ring + size_t(kPfRawStages) * kPfRawBytes);
  uint64_t* a_full = bars;                        // [kPfStages] TMA bytes of X
  uint64_t* b_full = a_full + kPfStages;          // [kPfStages] 128 dequant threads
  uint64_t* st_empty = b_full + kPfStages;        // [kPfStages] MMA commit
  uint64_t* w_full = st_empty + kPfStages;        // [kPfRawStages] TMA bytes of raw W
  uint64_t* w_empty = w_full + kPfRawStages;      // [kPfRawStages] 128 dequant threads
  uint64_t* done = w_empty + kPfRawStages;        // final MMA commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / prm.ksplit;
  const int split = blockIdx.x - tile * prm.ksplit;
  const int n0 = tile * kPfTileN;
  const int c0 = split * prm.kchunks / prm.ksplit;
  const int nraw = (split + 1) * prm.kchunks / prm.ksplit - c0;  // >= 1 (kchunks >= ksplit)
  const int k_begin = c0 * kPfRawK;
  const int nst = nraw * (kPfRawK / kPfStageK);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&b_full[i], kPfDqThreads);
      mbar_init(&st_empty[i], kPfIssuers);
    }
    for (int i = 0; i < kPfRawStages; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], kPfDqThreads);
    }
    mbar_init(done, kPfIssuers);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    // 128 fp32 columns of tensor memory for the 128 x 128 accumulator
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kPfIssuers * kPfTileN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Dependent launch: the next kernel on the stream may start its prologue now; every global
  // read and write of this one waits for the previous kernel (X may be its output, Y its input).
  griddep_launch_dependents();
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0, r = 0;
      for (; r < nraw && !*abort_flag; ++r) {
        const int rs = r % kPfRawStages;
        if (r >= kPfRawStages && !mbar_wait(&w_empty[rs], uint32_t(r / kPfRawStages - 1) & 1u)) {
          *abort_flag = 1;
          break;
        }
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&w_full[rs], uint32_t(kPfRawBytes));
        tma_load_2d(w_ring + size_t(rs) * kPfRawBytes, &tmap_w, (k_begin / kPfRawK + r) * kPfRawBytesRow, n0,
                    &w_full[rs]);
        for (int q = 0; q < kPfRawK / kPfStageK; ++q, ++s) {
          const int st = s % kPfStages;
          if (s >= kPfStages && !mbar_wait(&st_empty[st], uint32_t(s / kPfStages - 1) & 1u)) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&a_full[st], uint32_t(kPfABytes));
          tma_load_2d(a_ring + size_t(st) * kPfABytes, &tmap_x, k_begin + s * kPfStageK, 0, &a_full[st]);
        }
      }
      if (*abort_flag) {
        // bounded wait for the copies already issued, so none lands after the CTA exits
        for (int q = (s > kPfStages ? s - kPfStages : 0); q < s; ++q)
          mbar_wait(&a_full[q % kPfStages], uint32_t(q / kPfStages) & 1u);
        for (int q = (r > kPfRawStages ? r - kPfRawStages : 0); q < r; ++q)
          mbar_wait(&w_full[q % kPfRawStages], uint32_t(q / kPfRawStages) & 1u);
      }
    }
  } else if (warp == 1 || warp >= kPfWarpIss2) {
    // ------------------------------------------------ MMA issuers: issuer p takes k steps p, p + I, ...
    if (lane == 0) {
      const int p = warp == 1 ? 0 : warp - kPfWarpIss2 + 1;
      const uint32_t idesc = umma_idesc_f16(kPfTileM, kPfTileN);
      const uint32_t acc = tmem + uint32_t(p * kPfTileN);
      for (int s = 0; s < nst; ++s) {
        const int st = s % kPfStages;
        const uint32_t par = uint32_t(s / kPfStages) & 1u;
        if (!mbar_wait(&a_full[st], par) || !mbar_wait(&b_full[st], par)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_s = smem_u32(a_ring + size_t(st) * kPfABytes);
        const uint32_t b_s = smem_u32(b_ring + size_t(st) * kPfBBytes);
#pragma unroll
        for (int kk = p; kk < kPfStageK / 16; kk += kPfIssuers)  // 16 fp16 = 32 bytes per MMA along k
          umma_f16(acc, umma_desc_sw128(a_s + 32 * kk), umma_desc_sw128(b_s + 32 * kk), idesc,
                   (s > 0 || kk != p) ? 1u : 0u);
        umma_commit(&st_empty[st]);  // frees the stage once these MMAs have read it
      }
      umma_commit(done);  // all MMAs issued by this thread have completed
    }
  } else {
    // ------------------------------------------------ dequantize W into the B stages
    const int tt = threadIdx.x - 64;     // 0 .. kPfDqThreads - 1
    const int t = tt & 127;              // weight row n0 + t of the tile
    const int half = kPfDqWarps == 8 ? (tt >> 7) : -1;  // 8 warps: block A (0) or B (1) of the stage
    const uint32_t b_row_base = uint32_t(t >> 3) * 1024 + uint32_t(t & 7) * 128;
    const int sw = t & 7;            // swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
    int s = 0;
    bool ok = true;
    for (int r = 0; r < nraw && ok; ++r) {
      const int rs = r % kPfRawStages;
      if (!mbar_wait(&w_full[rs], uint32_t(r / kPfRawStages) & 1u)) {
        ok = false;
        break;
      }
      const uint32_t raw_row = smem_u32(w_ring + size_t(rs) * kPfRawBytes) + uint32_t(t) * kPfRawBytesRow;
      for (int q = 0; q < kPfRawK / kPfStageK; ++q, ++s) {
        const int st = s % kPfStages;
        if (s >= kPfStages && !mbar_wait(&st_empty[st], uint32_t(s / kPfStages - 1) & 1u)) {
          ok = false;
          break;
        }
        // two Q4_0 blocks (36 bytes) of this row: block A at bytes 0..17, block B at 18..35
        const uint32_t b_s = smem_u32(b_ring + size_t(st) * kPfBBytes) + b_row_base;
        if (half <= 0) {
          uint32_t v[5];
#pragma unroll
          for (int i = 0; i < 5; ++i) v[i] = lds32(raw_row + 36 * q + 4 * i);
          const __half2 dA = __half2half2(__ushort_as_half(static_cast<unsigned short>(v[0] & 0xFFFFu)));
#pragma unroll
          for (int m = 0; m < 4; ++m) {  // block A: k = 8m .. 8m+7
            uint32_t o[4];
            q4_word_to_f16(__funnelshift_r(v[m], v[m + 1], 16), dA, o);
            sts128(b_s + uint32_t((m ^ sw) * 16), o[0], o[1], o[2], o[3]);
          }
        }
        if (half != 0) {
          uint32_t v[5];
#pragma unroll
          for (int i = 0; i < 5; ++i) v[i] = lds32(raw_row + 36 * q + 16 + 4 * i);
          const __half2 dB = __half2half2(__ushort_as_half(static_cast<unsigned short>(v[0] >> 16)));
#pragma unroll
          for (int m = 0; m < 4; ++m) {  // block B: k = 32 + 8m .. 32 + 8m + 7
            uint32_t o[4];
            q4_word_to_f16(v[1 + m], dB, o);
            sts128(b_s + uint32_t(((4 + m) ^ sw) * 16), o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();  // make the fp16 tile visible to the tensor core
        mbar_arrive(&b_full[st]);
      }
      mbar_arrive(&w_empty[rs]);
    }
    if (!ok) *abort_flag = 1;
  }

  // ------------------------------------------------ epilogue: accumulator -> fp16 Y
  // Warps 2-5 own the accumulator rows (tensor-memory lanes 32*(warp%4) .. +31 = tokens).  With a
  // k-split cluster every CTA parks its partial tile in its (now idle) A ring; rank r then sums
  // its slice of the columns over all ranks, in rank order, through distributed shared memory.
  // Every thread of every CTA takes part in the two cluster barriers.
  const bool epi_warp = warp >= 2 && warp < 6;  // the first four dequant warps: one per lane quarter
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;  // token
  bool have = false;
  if (epi_warp) {
    have = !*abort_flag && mbar_wait(done, 0);
    tc_fence_after();
  }
  // partial tile, row-major with a 4-float pad per row (conflict-free 16-byte accesses)
  constexpr int kPitch = kPfTileN + 4;
  float* park = reinterpret_cast<float*>(a_ring);  // [kPfTileM][kPitch] fp32 = 66 KB
  const uint32_t tm_row = tmem + (uint32_t(quarter * 32) << 16);
  if (prm.ksplit > 1) {
    if (epi_warp) {
#pragma unroll 1
      for (int c = 0; c < kPfTileN; c += 16) {
        float r16[16];
        if (have) pf_acc16(tm_row + uint32_t(c), r16);
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(&park[row * kPitch + c + i]) =
              have ? make_float4(r16[i], r16[i + 1], r16[i + 2], r16[i + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    __syncwarp();
    cluster_sync();
    // rank r sums columns [r * cw, (r + 1) * cw) of every rank's tile, in rank order
    const int cw = kPfTileN / prm.ksplit;  // 16, 32 or 64
    const int rank = int(cluster_ctarank());
    const int c0 = rank * cw;
    const int ncols = min(cw, prm.n - n0 - c0);
    if (epi_warp && row < prm.tokens && ncols > 0) {
      __half* y = static_cast<__half*>(prm.Y) + size_t(row) * prm.n + n0 + c0;
#pragma unroll 1
      for (int c = 0; c < ncols; c += 8) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
        for (int rk = 0; rk < prm.ksplit; ++rk) {
          const uint32_t a = smem_u32(&park[row * kPitch + c0 + c]);
          const float4 lo = ld_dsmem_f32x4(a, uint32_t(rk));
          const float4 hi = ld_dsmem_f32x4(a + 16, uint32_t(rk));
          v[0] += lo.x; v[1] += lo.y; v[2] += lo.z; v[3] += lo.w;
          v[4] += hi.x; v[5] += hi.y; v[6] += hi.z; v[7] += hi.w;
        }
        uint4 pk;
        pk.x = h2_bits(__floats2half2_rn(v[0], v[1]));
        pk.y = h2_bits(__floats2half2_rn(v[2], v[3]));
        pk.z = h2_bits(__floats2half2_rn(v[4], v[5]));
        pk.w = h2_bits(__floats2half2_rn(v[6], v[7]));
        *reinterpret_cast<uint4*>(y + c) = pk;
      }
    }
    __syncwarp();
    cluster_sync();  // every rank keeps its shared memory until all ranks have read it
  } else if (epi_warp && have) {
    // tcgen05.ld is warp-collective: every lane loads, only rows < tokens store
    __half* y = static_cast<__half*>(prm.Y) + size_t(row) * prm.n + n0;
    const int ncols = row < prm.tokens ? min(kPfTileN, prm.n - n0) : 0;
#pragma unroll 1
    for (int c = 0; c < kPfTileN; c += 16) {
      float r16[16];
      pf_acc16(tm_row + uint32_t(c), r16);
      if (c < ncols) {
        uint4 pk;
        pk.x = h2_bits(__floats2half2_rn(r16[0], r16[1]));
        pk.y = h2_bits(__floats2half2_rn(r16[2], r16[3]));
        pk.z = h2_bits(__floats2half2_rn(r16[4], r16[5]));
        pk.w = h2_bits(__floats2half2_rn(r16[6], r16[7]));
        *reinterpret_cast<uint4*>(y + c) = pk;
      }
      if (c + 8 < ncols) {
        uint4 pk;
        pk.x = h2_bits(__floats2half2_rn(r16[8], r16[9]));
        pk.y = h2_bits(__floats2half2_rn(r16[10], r16[11]));
        pk.z = h2_bits(__floats2half2_rn(r16[12], r16[13]));
        pk.w = h2_bits(__floats2half2_rn(r16[14], r16[15]));
        *reinterpret_cast<uint4*>(y + c + 8) = pk;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPfIssuers * kPfTileN));
  }
}

// ---------------------------------------------------------------- host side
inline SmemAttrOnce g_prefill_attr;

}  // namespace bqg

extern "C" int qgemm_prefill(int fmt, const void* W, const void* X, void* Y, int tokens, int n, int k, void* stream) {
  using namespace bqg;
  if (W == nullptr || X == nullptr || Y == nullptr || tokens < 1 || n < 1 || k < 1) return BQG_ERR_ARG;
  if (fmt != BQG_Q4_0) return BQG_ERR_FMT;
  if (tokens > kPfTileM || n % 16 != 0 || k % kPfRawK != 0 || k > BQG_MAX_COLS) return BQG_ERR_SHAPE;
  if (!aligned(W, 16) || !aligned(X, 16) || !aligned(Y, 16)) return BQG_ERR_ALIGN;
  int dev;
  DeviceInfo* info;
  int st = current_device(&dev, &info);
  if (st != BQG_OK) return st;
  EncodeTiledFn encode = encode_tiled_fn();
  if (encode == nullptr) return BQG_ERR_CUDA;
  st = g_prefill_attr.ensure(dev, k_prefill_q4, kPfSmemBytes);
  if (st != BQG_OK) return st;

  // X: fp16 [tokens x k], tiles of 64 k x 128 rows, 128-byte swizzle; rows >= tokens read as 0
  CUtensorMap tx, tw;
  {
    const cuuint64_t dims[2] = {cuuint64_t(k), cuuint64_t(tokens)};
    const cuuint64_t strides[1] = {cuuint64_t(k) * 2};
    const cuuint32_t box[2] = {cuuint32_t(kPfStageK), cuuint32_t(kPfTileM)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return BQG_ERR_CUDA;
  }
  // W: the Q4_0 bytes as a [n x row_bytes] byte matrix, tiles of 144 bytes (256 k) x 128 rows;
  // rows >= n read as 0 (scale 0: weights 0)
  {
    const cuuint64_t rb = cuuint64_t(k / 32) * 18;
    const cuuint64_t dims[2] = {rb, cuuint64_t(n)};
    const cuuint64_t strides[1] = {rb};
    const cuuint32_t box[2] = {cuuint32_t(kPfRawBytesRow), cuuint32_t(kPfTileN)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(W), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return BQG_ERR_CUDA;
  }

  // Split k across a cluster of CTAs when the output tiles alone would leave SMs idle.
  const int ntiles = (n + kPfTileN - 1) / kPfTileN;
  const int kchunks = k / kPfRawK;
  int ksplit = 1;
  while (ksplit * 2 <= kPfMaxSplit && ntiles * ksplit * 2 <= info->sm_count && kchunks >= ksplit * 2) ksplit *= 2;
  PfParams prm{};
  prm.Y = Y;
  prm.tokens = tokens;
  prm.n = n;
  prm.k = k;
  prm.ksplit = ksplit;
  prm.kchunks = kchunks;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(ntiles * ksplit), 1, 1);
  cfg.blockDim = dim3(kPfThreads, 1, 1);
  cfg.dynamicSmemBytes = kPfSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(ksplit);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, k_prefill_q4, tx, tw, prm) != cudaSuccess) {
    (void)cudaGetLastError();  // not left behind for a later call's status check
    return BQG_ERR_CUDA;
  }
  return launch_status();
}
