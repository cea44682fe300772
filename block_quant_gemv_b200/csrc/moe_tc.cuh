// Grouped expert GEMM of the MoE layer on the 5th-generation tensor cores (tcgen05), for steps
// with many tokens (a prefill chunk, or a decode batch whose experts each serve several tokens):
//   gate/up phase:  h[p, i] = act(G_e[i, :] x_t) * (U_e[i, :] x_t)   for every routed pair p = (t, j)
//   down phase:     out[p, c] = D_e[c, :] h[p, :]
// and the same for the shared expert over all tokens.
//
// Sources: TurboFieldfare wiki, "메모리·전문가 스트리밍" (prefill in chunks of at most 128 tokens;
// each expert read serves every row routed to it; routed experts split from the dense shared
// branch); Camelid README, "Gemma 4" (GeGLU experts; dense shared expert + sparse top-8 branch).
//
// Two variants of one kernel template: kind::f16 (Q8_0, Q4_0 and int4 weights as fp16, fp16
// activation rows, fp32 accumulation, 128 k per stage) and kind::i8 (int4 and int2 weights as
// unsigned bytes, activations as pairs of int8 digit rows, int32 accumulation, 256 k per stage).
//
// One work item = up to 64 activation rows (64 tokens in kind::f16; 32 tokens of two digit rows
// each in kind::i8) of one expert (or of the shared expert) times two 128-row weight tiles: the
// gate and up tiles of the same rows (gate/up phase), or two consecutive tiles of the down matrix
// (down phase).  Weight rows sit on the MMA's M side (128), the activation rows on N (16..64,
// padded to 16), k along the matrix columns.  Each CTA (one per SM) runs items claimed from a
// counter, with warp-specialised roles:
//   warp 0      TMA: raw weight chunks (128 rows of each tile, 192 to 288 bytes of each row, in
//               their block format) through a ring in shared memory.  A 3-D tensor map with 8-byte
//               elements views each family as [expert][super-row][bytes], a super-row being g = 1,
//               2 or 4 consecutive rows so that its byte length is a multiple of 16 (Q4_0 rows of
//               704 values are 396 bytes); each row's chunk is fetched in a 16-byte-aligned window.
//               Each chunk takes a long piece of every row, so that one producer/consumer round
//               through the raw ring covers two to four MMA stages.
//               Rows land in shared memory an odd multiple of 16 bytes apart (208, 272 or 304), so the
//               dequantizing threads' 16-byte loads of consecutive rows hit distinct bank groups
//               (a 64- or 256-byte pitch put 4 or 8 rows on the same banks).
//   warp 14     TMA: the item's activation rows (128-byte swizzle, k-major), one stage at a time
//               into the slot of the matching A stage.
//   warps 2-9   dequantize: thread (tile f, row r) turns its row's weights of a stage into fp16
//               or bytes and stores them with tcgen05.st straight into TENSOR MEMORY (lane r),
//               where the MMA reads its A operand.  Keeping A out of shared memory matters:
//               4-bit weights expanded in shared memory would cost 2-4 bytes of shared-memory
//               traffic per weight (store + MMA read), more than the SM moves at the HBM rate.
//               The first of these threads also waits for the stage's activation rows before it
//               arrives, so the stage barrier covers both operands.
//   warp 1      allocates all 512 tensor-memory columns; it and warps 15-21 issue tcgen05.mma
//               (A from tensor memory, B from shared memory): two A stages of 2 x 64 columns
//               (128 fp16 or 256 byte weights of each row), and
//               two accumulator buffers of 2 x 64 columns, so the epilogue of one item overlaps
//               the MMAs of the next.  The MMAs of one thread run back to back (~115-200 cycles
//               each for any N up to 128, measured on B200), while those of different warps
//               overlap; so each tile's k steps are spread over up to four chains, each issued by
//               its own warp into its own partial accumulator.
//   warps 10-13 epilogue: read the accumulators (tcgen05.ld), add the partials, apply row scales
//               (and, in kind::i8, the digit recombination), and write h = act(g) * u (gate/up)
//               or the fp32 per-pair outputs (down).
//
// kind::f16 weights become fp16 exactly as stored values allow: Q4_0 (q - 8) and Q8_0 q exactly
// via the fp16 exponent-bias identity (0x6400 | byte = 1024 + byte), then one rounding of the
// product by d; int4 values -8..7 exactly (its row scale is applied to the fp32 accumulator).
// Within each group of 8 k, nibble formats store the weights in the order their bytes yield them
// (elements 0,4,1,5,2,6,3,7 in kind::f16; 0,2,4,6,1,3,5,7 in kind::i8; int2 groups of 16 in
// kind::i8); the activation rows are written in the same order, which leaves every dot product
// unchanged.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "host_common.h"
#include "moe.cuh"
#include "tcgen05.cuh"

namespace bqg {

#ifndef BQG_TC_MMA_WARPS
#define BQG_TC_MMA_WARPS 8
#endif
constexpr int kTcWarpRaw = 0, kTcWarpMma = 1, kTcWarpDq = 2, kTcWarpEpi = 10, kTcWarpB = 14, kTcWarpMma2 = 15;
constexpr int kTcMmaWarps = BQG_TC_MMA_WARPS;  // MMA issuers: warp 1 and warps 15, 16, ...
constexpr int kTcThreads = 32 * (14 + kTcMmaWarps);
constexpr int kTcDqThreads = 256;          // 2 tiles x 128 rows
#ifndef BQG_TC_NMAX
#define BQG_TC_NMAX 64
#endif
#ifndef BQG_TC_I8_STAGE_K
#define BQG_TC_I8_STAGE_K 256
#endif
constexpr int kTcNMax = BQG_TC_NMAX;       // MMA N per item (tokens; two digit rows per token in kind::i8)
constexpr int kTcACols = 256;              // tensor-memory columns of the A stage ring
constexpr int kTcAStages = 4;              // barrier slots (the most stages a variant uses)
constexpr int kTcBStages = kTcAStages;
constexpr int kTcBRing = 32 * 1024;        // shared memory of the activation ring (all variants)
// Stage geometry of a variant.  kind::f16: BQG_TC_F16_STAGE_K (64 or 128) k per stage, 2 tiles x 32
// or 64 columns, 4 or 2 stages, 4 or 8 MMAs of 16 k per tile; the activation rows of a stage are
// one or two 128-byte-swizzled blocks of 64 k.  kind::i8: BQG_TC_I8_STAGE_K (128 or 256) k per
// stage, 2 tiles x 32 or 64 columns, 4 or 2 stages, 4 or 8 MMAs of 32 k per tile; one or two
// blocks of 128 k.  Blocks of one stage sit kTcNMax * 128 bytes apart.  Bigger stages halve the
// handoffs through the stage barriers per weight, which bound this loop.
#ifndef BQG_TC_F16_STAGE_K
#define BQG_TC_F16_STAGE_K 128
#endif
template <bool I8>
struct TcCfg {
  static constexpr int kStageK = I8 ? BQG_TC_I8_STAGE_K : BQG_TC_F16_STAGE_K;
  static constexpr int kTileCols = I8 ? kStageK / 4 : kStageK / 2;  // 4 bytes (or two fp16) per column
  static constexpr int kStageCols = 2 * kTileCols;
  static constexpr int kAStages = kTcACols / kStageCols;
  static constexpr int kKSteps = I8 ? kStageK / 32 : kStageK / 16;  // MMAs per tile and stage
  static constexpr int kBBlocks = I8 ? kStageK / 128 : kStageK / 64;  // 128-byte swizzle blocks per B row
  static constexpr int kBStageBytes = kBBlocks * kTcNMax * 128;
};
static_assert(TcCfg<true>::kAStages <= kTcAStages && TcCfg<false>::kAStages <= kTcAStages, "barrier slots");
static_assert(TcCfg<true>::kAStages * TcCfg<true>::kBStageBytes <= kTcBRing &&
                  TcCfg<false>::kAStages * TcCfg<false>::kBStageBytes <= kTcBRing,
              "activation ring");
constexpr int kTcAccTile = kTcNMax;        // accumulator columns per tile of one buffer
constexpr int kTcAccBuf = 2 * kTcAccTile;  // columns per accumulator buffer (two tiles)
#ifndef BQG_TC_ACC_BUFS
#define BQG_TC_ACC_BUFS 2
#endif
constexpr int kTcAccBufs = BQG_TC_ACC_BUFS;  // accumulator buffers (2: an item's epilogue overlaps the next one's MMAs)
constexpr int kTcDescs = 8;                // item descriptor ring
constexpr int kTcRawMax = 12;              // raw weight ring depth (runtime, by window size)
constexpr int kTcAccCol = kTcACols;       // first accumulator column (after the A stages)
static_assert(kTcAccBufs >= 1 && kTcAccBufs <= 2, "one or two accumulator buffers");
static_assert(kTcAccCol + kTcAccBufs * kTcAccBuf <= 512, "tensor memory: A stages + accumulator buffers");
constexpr int kTcDescReaders = 1 + kTcMmaWarps + 8 + 4;  // B producer, MMA, dequant and epilogue warps
// smem: [1 KB alignment slack][B ring][raw ring][barriers + descriptors]
constexpr int kTcBarBytes = 1024;
constexpr size_t kTcFixedSmem = 1024 + size_t(kTcBRing) + kTcBarBytes;
constexpr size_t kTcMaxSmem = 227 * 1024;
static_assert(kTcBStages == kTcAStages, "activation stage i shares the A stage's barriers");
static_assert((2 * kTcRawMax + 2 * kTcAStages + kTcBStages + 4 + 2 * kTcDescs + 1) * 8 + 16 + kTcDescs * 32 <=
                  kTcBarBytes,
              "barrier area");

// One family of stacked matrices as the kernel sees it (rows on M, cols = k).
struct TcFam {
  const uint8_t* base;  // expert 0's matrix (the shared expert: its only matrix)
  long long stride;     // bytes between experts
  int fmt, rows, cols;
  int row_bytes;
  int g;                // rows per super-row of the tensor map
  int win;              // bytes fetched per row and raw chunk (a 16-byte-aligned window)
  int cb;               // bytes of one raw chunk of one row
  int raw_k;            // weights per raw chunk (int4 512 or 384, int2 768, Q4_0 512, Q8_0 256)
  int scale_off;        // int4: byte offset of the row scales in one matrix
  int m_off;            // row offset of this tile inside an item (0, or 128 for the second down tile)
};

struct alignas(64) TcParams {
  CUtensorMap amap[4];  // weight maps: 0, 1 routed tiles; 2, 3 shared tiles
  CUtensorMap bmap[2];  // activation maps: 0 routed (rows in expert-grouped order), 1 shared (token order)
  TcFam fam[4];
  int phase;            // 0 gate/up, 1 down
  int act;
  int tokens, has_shared;
  int tiles_r, tiles_s; // items' tile pairs per routed expert / for the shared expert
  int raw_stages, raw_stage_bytes;
  const int4* act_info; // per touched expert: (expert, count, offset, first pair)
  const int32_t* n_active;
  const int32_t* perm;  // pair ids in expert-grouped order
  uint32_t* ctr;        // item counter (zeroed by the route kernel)
  __half* hout[2];      // gate/up: h rows (routed: grouped order; shared: token order)
  int hstride[2];       // inter, shared_inter
  int hperm[2];         // 1: the down matrix is a nibble format (store h in nibble order)
  float* yout[2];       // down: per-pair outputs [pairs][hidden], shared [tokens][hidden]
  int ystride;          // hidden
  // kind::i8 variant (int4 / int2 weights): activation rows are pairs of int8 digit rows
  // (X = 256 H + L, x ~= scale * X); per activation row its scale and the digit sum of X.
  int nmax;             // tokens per item: kTcNMax (fp16) or kTcNMax / 2 (int8 digit rows)
  const float* bscale[2];
  const int32_t* bsum[2];
  float* h32[2];        // gate/up of the kind::i8 variant: h rows in fp32 (natural order)
};

// ---------------------------------------------------------------- dequantization of one stage
// Four fp16 pairs of the 8 nibbles of word w (element 2m = low nibble of byte m), in the order
// the bytes yield them: (e0, e4) (e1, e5) (e2, e6) (e3, e7); values (q - 8) * d.
__device__ __forceinline__ void tc_nib8(uint32_t w, __half2 d2, uint32_t* o) {
  const __half2 bias = __half2half2(__ushort_as_half(0x6408));  // 1032
  uint32_t p[4] = {(w & 0x000F000Fu) | 0x64006400u, ((w >> 4) & 0x000F000Fu) | 0x64006400u,
                   ((w >> 8) & 0x000F000Fu) | 0x64006400u, ((w >> 12) & 0x000F000Fu) | 0x64006400u};
#pragma unroll
  for (int i = 0; i < 4; ++i)  // (1024 + q) - 1032 = q - 8 exactly; times d rounds once
    o[i] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<__half2*>(&p[i]), bias), d2));
}
// Same for two's-complement nibbles without a scale: t ^ 8 = t + 8, so (1024 + (t + 8)) - 1032 = t.
__device__ __forceinline__ void tc_i4nib8(uint32_t w, uint32_t* o) {
  const __half2 bias = __half2half2(__ushort_as_half(0x6408));
  w ^= 0x88888888u;
  uint32_t p[4] = {(w & 0x000F000Fu) | 0x64006400u, ((w >> 4) & 0x000F000Fu) | 0x64006400u,
                   ((w >> 8) & 0x000F000Fu) | 0x64006400u, ((w >> 12) & 0x000F000Fu) | 0x64006400u};
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = h2_bits(__hsub2(*reinterpret_cast<__half2*>(&p[i]), bias));
}
// Four int8 values of word w as two fp16 pairs (e0, e1) (e2, e3), values q * d:
// q ^ 0x80 = q + 128 as an unsigned byte, 0x64 high byte gives 1024 + q + 128, minus 1152 is q.
__device__ __forceinline__ void tc_q8x4(uint32_t w, __half2 d2, uint32_t* o) {
  const __half2 bias = __half2half2(__ushort_as_half(0x6480));  // 1152
  const uint32_t u = w ^ 0x80808080u;
  uint32_t p0 = __byte_perm(u, 0x64646464u, 0x5140), p1 = __byte_perm(u, 0x64646464u, 0x7362);
  o[0] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<__half2*>(&p0), bias), d2));
  o[1] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<__half2*>(&p1), bias), d2));
}

// ---------------------------------------------------------------- kind::i8 operands (int4 / int2)
// Weights as unsigned bytes t + 8 (int4) or t + 2 (int2): flipping the sign bit of each
// two's-complement field adds the offset, and masks spread the fields over bytes.  The epilogue
// removes the offset exactly: sum (t + z) X = sum t X + z sum X.
// Offset z of the unsigned weight bytes of a family (t + z).
__host__ __device__ __forceinline__ int tc_i8_zero(int fmt) { return fmt == BQG_I2_ROW ? 2 : 8; }

// Position of element k inside its int8 digit row: int4 groups of 8 in the order 0,2,4,6,1,3,5,7;
// int2 groups of 16 with element 4j + k at position 4k + j.
__host__ __device__ __forceinline__ int tc_i8_kpos(int k, int fmt) {
  if (fmt == BQG_I2_ROW) {
    const int i = k & 15;
    return (k & ~15) | ((i & 3) << 2) | (i >> 2);
  }
  const int i = k & 7;
  return (k & ~7) | ((i & 1) << 2) | (i >> 1);
}

// Position of element k inside its activation row: nibble formats hold each group of 8 in
// the order 0,4,1,5,2,6,3,7, i.e. element i of a group sits at position {0,2,4,6,1,3,5,7}[i].
__host__ __device__ __forceinline__ int tc_kpos(int k, int nibble) {
  if (!nibble) return k;
  const int i = k & 7;
  return (k & ~7) | ((i & 3) << 1) | (i >> 2);
}

// Partial accumulators per tile for an item of N (padded) tokens: 4 x 16, 2 x 32 or 1 x N columns,
// so that both tiles of an accumulator buffer fit its 128 columns.  Partial p takes the k steps
// p, p + parts, ... and is initialised by its first one, so every partial needs at least one k step
// in an item's first stage: the shortest possible stage (a matrix of 64 columns in kind::f16, 128
// in kind::i8, the smallest widths either variant accepts) has 4 k steps, the most partials used.
constexpr int kTcMaxPartials = 4;
static_assert(64 / 16 >= kTcMaxPartials && 128 / 32 >= kTcMaxPartials,
              "every partial accumulator gets a k step of the first stage");
__host__ __device__ __forceinline__ int tc_partials(int N) {
  const int cap = kTcMmaWarps >= 2 ? kTcMmaWarps / 2 : 1;  // issuers per tile
  int p = 1;
  while (p < kTcMaxPartials && p < cap && 2 * p * N <= kTcAccTile) p *= 2;
  return p;
}

// 8 accumulator columns of this warp's lanes at taddr, summed over the tile's `parts` partial
// accumulators (stride columns apart) in a fixed order.  Warp-uniform arguments.
__device__ __forceinline__ void tc_acc8(uint32_t taddr, int stride, int parts, float (&o)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;
  for (int p = 0; p < parts; ++p) {
    uint32_t v[8];
    tmem_ld8_nowait(taddr + uint32_t(p * stride), v);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] += __uint_as_float(v[i]);
  }
}

// The same for int32 accumulators (kind::i8): exact integer sums.
__device__ __forceinline__ void tc_acc8i(uint32_t taddr, int stride, int parts, int (&o)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0;
  for (int p = 0; p < parts; ++p) {
    uint32_t v[8];
    tmem_ld8_nowait(taddr + uint32_t(p * stride), v);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] += int(v[i]);
  }
}

// Raw chunk geometry per weight format: weights and bytes of one row per chunk, and the shared-
// memory pitch of the rows (an odd multiple of 16 bytes; the chunk plus up to 12 bytes of
// misalignment for the 18- and 34-byte block formats).
// int4 takes 512 k (256 bytes, pitch 272) when the kind::i8 stage is 256 k, else 384 k.
__host__ __device__ constexpr int tc_raw_k(int fmt) {
  return fmt == BQG_I2_ROW ? 768 : fmt == BQG_I4_ROW ? (BQG_TC_I8_STAGE_K == 256 ? 512 : 384)
                                 : fmt == BQG_Q4_0 ? 512 : 256;
}
__host__ __device__ constexpr int tc_raw_cb(int fmt) {
  return fmt == BQG_I2_ROW ? 192 : fmt == BQG_I4_ROW ? tc_raw_k(fmt) / 2 : fmt == BQG_Q4_0 ? 288 : 272;
}
__host__ __device__ constexpr int tc_raw_win(int fmt) { return fmt == BQG_I2_ROW || fmt == BQG_I4_ROW ? tc_raw_cb(fmt) + 16 : 304; }
// Geometry checks per format: the window holds the chunk plus the largest misalignment (12 bytes
// for the block formats, whose rows are multiples of 4 bytes; none for int4 / int2, whose chunks
// start 16-byte aligned), its pitch is an odd multiple of 16 bytes, chunks hold whole stages of
// both variants, and at least two raw stages of the widest window fit beside the fixed areas.
constexpr bool tc_raw_geometry_ok(int fmt, int stage_k, int fixed_smem, int max_smem) {
  return tc_raw_win(fmt) >= tc_raw_cb(fmt) + (fmt == BQG_Q4_0 || fmt == BQG_Q8_0 ? 12 : 0) &&
         tc_raw_win(fmt) % 16 == 0 && (tc_raw_win(fmt) / 16) % 2 == 1 && tc_raw_k(fmt) % stage_k == 0 &&
         fixed_smem + 2 * (2 * 128 * tc_raw_win(fmt)) <= max_smem;
}

static_assert(tc_raw_geometry_ok(BQG_Q4_0, TcCfg<false>::kStageK, int(kTcFixedSmem), int(kTcMaxSmem)) &&
                  tc_raw_geometry_ok(BQG_Q8_0, TcCfg<false>::kStageK, int(kTcFixedSmem), int(kTcMaxSmem)) &&
                  tc_raw_geometry_ok(BQG_I4_ROW, TcCfg<false>::kStageK, int(kTcFixedSmem), int(kTcMaxSmem)) &&
                  tc_raw_geometry_ok(BQG_I4_ROW, TcCfg<true>::kStageK, int(kTcFixedSmem), int(kTcMaxSmem)) &&
                  tc_raw_geometry_ok(BQG_I2_ROW, TcCfg<true>::kStageK, int(kTcFixedSmem), int(kTcMaxSmem)),
              "raw chunk geometry");

// 64 k of one row (32 tensor-memory columns), loaded first and converted after: all its shared-
// memory words are read before the tensor-memory store, so the loads of the second half do not
// wait behind it.  Q4_0: 36 bytes (two blocks), Q8_0: 68 bytes, int4 (kind::f16): 32 bytes.
template <int FMT>
__device__ __forceinline__ void tc_f16_sub(uint32_t src, uint32_t taddr) {
  uint32_t o[32];  // both halves, stored with one tensor-memory instruction
  if constexpr (FMT == BQG_Q4_0) {  // block A: d at bytes 0-1, qs 2..17; block B: d at 18-19, qs 20..35
    uint32_t v[9];
#pragma unroll
    for (int i = 0; i < 9; ++i) v[i] = lds32(src + 4 * i);
    const __half2 dA = __half2half2(__ushort_as_half(static_cast<unsigned short>(v[0] & 0xFFFFu)));
    const __half2 dB = __half2half2(__ushort_as_half(static_cast<unsigned short>(v[4] >> 16)));
#pragma unroll
    for (int m = 0; m < 4; ++m) tc_nib8(__funnelshift_r(v[m], v[m + 1], 16), dA, &o[4 * m]);
#pragma unroll
    for (int m = 0; m < 4; ++m) tc_nib8(v[5 + m], dB, &o[16 + 4 * m]);
  } else if constexpr (FMT == BQG_Q8_0) {  // block A: d 0-1, q 2..33; block B: d 34-35, q 36..67
    uint32_t v[17];
#pragma unroll
    for (int i = 0; i < 17; ++i) v[i] = lds32(src + 4 * i);
    const __half2 dA = __half2half2(__ushort_as_half(static_cast<unsigned short>(v[0] & 0xFFFFu)));
    const __half2 dB = __half2half2(__ushort_as_half(static_cast<unsigned short>(v[8] >> 16)));
#pragma unroll
    for (int m = 0; m < 8; ++m) tc_q8x4(__funnelshift_r(v[m], v[m + 1], 16), dA, &o[2 * m]);
#pragma unroll
    for (int m = 0; m < 8; ++m) tc_q8x4(v[9 + m], dB, &o[16 + 2 * m]);
  } else {  // int4: 16-byte aligned
    const uint4 p0 = lds128(src), p1 = lds128(src + 16);
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
    for (int m = 0; m < 8; ++m) tc_i4nib8(w[m], &o[4 * m]);
  }
  tmem_st32(taddr, o);
}
template <int FMT>
__device__ __forceinline__ void tc_f16_stage(uint32_t src, uint32_t taddr) {
  constexpr int kSub = FMT == BQG_Q4_0 ? 36 : FMT == BQG_Q8_0 ? 68 : 32;  // bytes per 64 k
#pragma unroll
  for (int g = 0; g < TcCfg<false>::kStageK / 64; ++g) tc_f16_sub<FMT>(src + kSub * g, taddr + 32 * g);
}

// kind::i8: int4 64 bytes (128 k), int2 32 bytes; 16-byte aligned.  Each int4 word yields two
// words of bytes t + 8: elements 0,2,4,6 then 1,3,5,7 of its group of 8; each int2 word yields four
// words of bytes t + 2, byte j of word k holding element 4j + k of its group of 16.
__device__ __forceinline__ void tc_i4_bytes(uint4 a, uint4 b, uint32_t (&o)[16]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint32_t u = w[m] ^ 0x88888888u;
    o[2 * m] = u & 0x0F0F0F0Fu;
    o[2 * m + 1] = (u >> 4) & 0x0F0F0F0Fu;
  }
}
__device__ __forceinline__ void tc_i2_bytes(uint4 a, uint32_t (&o)[16]) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t u = w[m] ^ 0xAAAAAAAAu;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[4 * m + k] = (u >> (2 * k)) & 0x03030303u;
  }
}
template <int FMT>
__device__ __forceinline__ void tc_i8_stage(uint32_t src, uint32_t taddr) {
  constexpr int kStageK = TcCfg<true>::kStageK;
  uint32_t o[32];
  uint32_t (&lo)[16] = *reinterpret_cast<uint32_t(*)[16]>(&o[0]);
  uint32_t (&hi)[16] = *reinterpret_cast<uint32_t(*)[16]>(&o[16]);
#pragma unroll
  for (int g = 0; g < kStageK / 128; ++g) {  // 128 k = 32 tensor-memory columns per step
    if constexpr (FMT == BQG_I4_ROW) {       // 64 bytes per 128 k
      const uint32_t a = src + 64 * g;
      const uint4 p0 = lds128(a), p1 = lds128(a + 16), p2 = lds128(a + 32), p3 = lds128(a + 48);
      tc_i4_bytes(p0, p1, lo);
      tc_i4_bytes(p2, p3, hi);
    } else {                                 // int2: 32 bytes per 128 k
      const uint32_t a = src + 32 * g;
      tc_i2_bytes(lds128(a), lo);
      tc_i2_bytes(lds128(a + 16), hi);
    }
    tmem_st32(taddr + 32 * g, o);
  }
}

// One item's stages for this thread's row of a tile: wait for each raw chunk, dequantize every
// stage of it (TcCfg<I8>::kStageK weights) into the A stage ring in tensor memory, and
// hand the stages to the MMA issuers.  The format is a template argument, so the block layout
// and every offset are constants.  Returns false when a bounded wait gave up.
//   row_base  shared address of this row's window in raw stage 0;  mis0  j * row_bytes (the
//   row's byte offset inside its super-row, for the 16-byte misalignment of each chunk)
//   tcol      tensor-memory address of this lane, tile column offset included
//   wait_b    this thread also waits for the stage's activation rows (b_full) before it arrives,
//             so that a_full completes only once both operands of the stage are in place
template <bool I8, int FMT>
__device__ __forceinline__ bool tc_dq_item(int nst, bool row_on, uint32_t row_base, int mis0, int raw_stages,
                                           int raw_stage_bytes, uint64_t* raw_full, uint64_t* raw_empty,
                                           uint64_t* a_full, uint64_t* a_empty, uint64_t* b_full, bool wait_b,
                                           uint32_t tcol, int& slot_r, uint32_t& ph_r, int& as) {
  using C = TcCfg<I8>;
  constexpr int kStageK = C::kStageK;
  constexpr int kSpr = tc_raw_k(FMT) / kStageK;      // stages per raw chunk
  static_assert(tc_raw_k(FMT) % kStageK == 0, "raw chunks hold whole stages");
  constexpr int kCb = tc_raw_cb(FMT);
  constexpr int kStageBytes = kCb / kSpr;
  const int nraw = (nst + kSpr - 1) / kSpr;
  for (int kc = 0; kc < nraw; ++kc) {
    if (!mbar_wait(&raw_full[slot_r], ph_r)) return false;
    const uint32_t base = row_base + uint32_t(slot_r * raw_stage_bytes) + (uint32_t(mis0 + kc * kCb) & 15u);
    const int nh = min(kSpr, nst - kc * kSpr);
    for (int h = 0; h < nh; ++h, ++as) {
      const int aslot = as % C::kAStages;
      if (as >= C::kAStages && !mbar_wait(&a_empty[aslot], uint32_t(as / C::kAStages - 1) & 1u)) return false;
      tc_fence_after();
      if (row_on) {
        const uint32_t src = base + uint32_t(h * kStageBytes);
        const uint32_t taddr = tcol + uint32_t(aslot * C::kStageCols);
        if constexpr (I8) tc_i8_stage<FMT>(src, taddr);
        else tc_f16_stage<FMT>(src, taddr);
        tmem_wait_st();
      }
      tc_fence_before();
      if (wait_b && !mbar_wait(&b_full[aslot], uint32_t(as / C::kAStages) & 1u)) return false;
      mbar_arrive(&a_full[aslot]);
    }
    mbar_arrive(&raw_empty[slot_r]);
    if (++slot_r == raw_stages) {
      slot_r = 0;
      ph_r ^= 1u;
    }
  }
  return true;
}

// ---------------------------------------------------------------- the kernel
// Item descriptor: d0 = (flags: bit0 shared, bit1 second tile present; expert; m0; tokens),
//                  d1 = (first activation row; N; first output row; stages).
// I8: kind::i8 variant (int4 / int2 weights as unsigned bytes in tensor memory, activations as
// int8 digit rows, int32 accumulators); the stage geometry of each variant is TcCfg<I8>.
template <bool I8>
__global__ void __launch_bounds__(kTcThreads, 1) k_moe_tc(const __grid_constant__ TcParams P) {
  using C = TcCfg<I8>;
  constexpr int kStageK = C::kStageK;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_s & 1023)) & 1023);
  uint8_t* bring = smem;                                            // C::kAStages x C::kBStageBytes
  uint8_t* wring = bring + size_t(kTcBRing);                        // raw_stages x raw_stage_bytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(wring + size_t(P.raw_stages) * P.raw_stage_bytes);
  uint64_t* raw_full = bars;                        // [kTcRawMax] TMA bytes
  uint64_t* raw_empty = raw_full + kTcRawMax;       // [kTcRawMax] 256 dequant threads
  uint64_t* a_full = raw_empty + kTcRawMax;         // [kTcAStages] 256 dequant threads
  uint64_t* a_empty = a_full + kTcAStages;          // [kTcAStages] MMA commits (one per issuer)
  uint64_t* b_full = a_empty + kTcAStages;          // [kTcBStages] TMA bytes (B slot i is freed by a_empty[i])
  uint64_t* acc_full = b_full + kTcBStages;         // [2] MMA commits
  uint64_t* acc_empty = acc_full + 2;               // [2] 128 epilogue threads
  uint64_t* d_full = acc_empty + 2;                 // [kTcDescs] producer
  uint64_t* d_empty = d_full + kTcDescs;            // [kTcDescs] reader warps
  uint64_t* done = d_empty + kTcDescs;              // final MMA commits
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int4* descs = reinterpret_cast<int4*>(bars + (kTcBarBytes - kTcDescs * 32) / 8);  // [kTcDescs][2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcRawMax; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], kTcDqThreads);
    }
    for (int i = 0; i < kTcAStages; ++i) {
      mbar_init(&a_full[i], kTcDqThreads);
      mbar_init(&a_empty[i], kTcMmaWarps);
    }
    for (int i = 0; i < kTcBStages; ++i) {
      mbar_init(&b_full[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], kTcMmaWarps);
      mbar_init(&acc_empty[i], 128);
    }
    for (int i = 0; i < kTcDescs; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kTcDescReaders);
    }
    mbar_init(done, kTcMmaWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTcWarpRaw && lane == 0) {
    for (int i = 0; i < 4; ++i) prefetch_tensormap(&P.amap[i]);
    prefetch_tensormap(&P.bmap[0]);
    prefetch_tensormap(&P.bmap[1]);
  }
  if (warp == kTcWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // routing tables and activation rows come from earlier kernels

  // Readers of the descriptor ring: wait for slot ds, copy, release (lane 0 of each reader warp).
  // Called by lane 0 of a reader warp only (the other lanes get the values by shuffles).
  auto read_desc = [&](int ds, int4& d0, int4& d1) -> bool {
    const int slot = ds % kTcDescs;
    if (!mbar_wait(&d_full[slot], uint32_t(ds / kTcDescs) & 1u)) {
      *abort_flag = 1;
      return false;
    }
    d0 = ld_desc(&descs[2 * slot]);
    d1 = ld_desc(&descs[2 * slot + 1]);
    mbar_arrive(&d_empty[slot]);
    return true;
  };

  if (warp == kTcWarpRaw) {
    // ------------------------------------------------ item claims + raw weight TMA
    if (lane == 0) {
      const int na = *P.n_active;
      const int nmax = P.nmax;
      const int nch = (P.tokens + nmax - 1) / nmax;
      const int n_sh = P.has_shared ? P.tiles_s * nch : 0;
      const int per_e = P.tiles_r * nch;
      const int n_items = n_sh + na * per_e;
      const int tile_rows = P.phase == 0 ? 128 : 256;
      int ds = 0, rp = 0;
      bool ok = true;
      int item = int(atomicAdd(P.ctr, 1u));
      while (ok) {
        const int next = item < n_items ? int(atomicAdd(P.ctr, 1u)) : n_items;  // one claim ahead
        int4 d0, d1;
        bool end = item >= n_items;
        if (!end) {
          int shared, e = 0, t, c, cnt, off;
          if (item < n_sh) {
            shared = 1;
            t = item / nch;
            c = item - t * nch;
            cnt = P.tokens;
            off = 0;
          } else {
            shared = 0;
            const int r = item - n_sh;
            const int a = r / per_e;
            const int rem = r - a * per_e;
            t = rem / nch;
            c = rem - t * nch;
            const int4 ai = __ldg(P.act_info + a);
            e = ai.x;
            cnt = ai.y;
            off = ai.z;
          }
          const int ntok = min(nmax, cnt - c * nmax);
          if (ntok <= 0) {  // an empty token chunk of a lightly routed expert
            item = next;
            continue;
          }
          const int fb = shared ? 2 : 0;
          const int m0 = t * tile_rows;
          const int two = (P.phase == 0 || m0 + 128 < P.fam[fb].rows) ? 1 : 0;
          d0 = make_int4(shared | (two << 1), e, m0, ntok);
          const int brow = I8 ? 2 * (off + c * nmax) : off + c * nmax;  // first B row
          const int nb = I8 ? 2 * ntok : ntok;                                // B rows
          d1 = make_int4(brow, (nb + 15) & ~15, off + c * nmax, (P.fam[fb].cols + kStageK - 1) / kStageK);
        } else {
          d0 = make_int4(-1, 0, 0, 0);
          d1 = make_int4(0, 0, 0, 0);
        }
        const int slot = ds % kTcDescs;
        if (ds >= kTcDescs && !mbar_wait(&d_empty[slot], uint32_t(ds / kTcDescs - 1) & 1u)) {
          ok = false;
          break;
        }
        descs[2 * slot] = d0;
        descs[2 * slot + 1] = d1;
        mbar_arrive(&d_full[slot]);
        ++ds;
        if (end) break;
        // raw chunks of this item: both tiles' rows, k range [kc * raw_k, (kc + 1) * raw_k)
        const int fb = (d0.x & 1) ? 2 : 0;
        const int ntiles = 1 + ((d0.x >> 1) & 1);
        const TcFam& F0 = P.fam[fb];
        const int nraw = (d1.w * kStageK + F0.raw_k - 1) / F0.raw_k;
        for (int kc = 0; kc < nraw; ++kc, ++rp) {
          const int slot_r = rp % P.raw_stages;
          if (rp >= P.raw_stages && !mbar_wait(&raw_empty[slot_r], uint32_t(rp / P.raw_stages - 1) & 1u)) {
            ok = false;
            break;
          }
          if (*abort_flag) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&raw_full[slot_r], uint32_t(ntiles * 128 * F0.win));
          uint8_t* dst0 = wring + size_t(slot_r) * P.raw_stage_bytes;
          for (int f = 0; f < ntiles; ++f) {
            const TcFam& F = P.fam[fb + f];
            const int y = (d0.z + F.m_off) / F.g;
            for (int j = 0; j < F.g; ++j) {
              const int xb = (j * F.row_bytes + kc * F.cb) & ~15;
              tma_load_3d(dst0 + size_t(f) * 128 * F.win + size_t(j) * (128 / F.g) * F.win, &P.amap[fb + f], xb / 8, y,
                          d0.y, &raw_full[slot_r]);
            }
          }
        }
        item = next;
      }
      if (!ok) {
        *abort_flag = 1;
        // bounded wait for the copies already issued, so none lands after the CTA exits
        for (int q = (rp > P.raw_stages ? rp - P.raw_stages : 0); q < rp; ++q)
          mbar_wait(&raw_full[q % P.raw_stages], uint32_t(q / P.raw_stages) & 1u);
      }
    }
  } else if (warp == kTcWarpB) {
    // ------------------------------------------------ activation rows (B operand) TMA
    if (lane == 0) {
      int bs = 0;
      bool ok = true;
      for (int ds = 0; ok; ++ds) {
        int4 d0, d1;
        if (!read_desc(ds, d0, d1)) break;
        if (d0.x < 0) break;
        const int sh = d0.x & 1;
        const int N = d1.y;
        for (int s = 0; s < d1.w; ++s, ++bs) {
          const int slot = bs % C::kAStages;
          if (bs >= C::kAStages && !mbar_wait(&a_empty[slot], uint32_t(bs / C::kAStages - 1) & 1u)) {
            ok = false;
            break;
          }
          if (*abort_flag) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&b_full[slot], uint32_t(N * 128 * C::kBBlocks));
          uint8_t* dst = bring + size_t(slot) * C::kBStageBytes;
          for (int blk = 0; blk < C::kBBlocks; ++blk)  // 128 k (kind::i8) or 64 k (fp16) per swizzle block
            for (int nb = 0; nb < N / 16; ++nb)
              tma_load_2d(dst + blk * (kTcNMax * 128) + nb * 2048, &P.bmap[sh],
                          s * kStageK + blk * (I8 ? 128 : 64), d1.x + 16 * nb, &b_full[slot]);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int q = (bs > C::kAStages ? bs - C::kAStages : 0); q < bs; ++q)
          mbar_wait(&b_full[q % C::kAStages], uint32_t(q / C::kAStages) & 1u);
      }
    }
  } else if (warp == kTcWarpMma || warp >= kTcWarpMma2) {
    // ------------------------------------------------ MMA issuers
    // One thread's tcgen05.mma instructions run one after another, each taking ~170 cycles at
    // N <= 128 whatever N is, while several issuing warps overlap theirs.  So the MMAs of a stage
    // are spread over kTcMmaWarps issuers: issuer (tile f, partial p) owns the chain of k steps
    // kk = p, p + P, ... of tile f into its own accumulator, P = 64 / N partial accumulators per
    // tile (4 at N = 16, 2 at N = 32, else 1); the epilogue adds the P partials.
    if (lane == 0) {
      const int mi = warp == kTcWarpMma ? 0 : warp - kTcWarpMma2 + 1;
      constexpr int kTileStep = kTcMmaWarps >= 2 ? 2 : 1;  // one issuer per tile, or one for both
      const int f0 = mi % kTileStep, p = mi / kTileStep;
      int as = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        int4 d0, d1;
        if (!read_desc(it, d0, d1)) break;
        if (d0.x < 0) break;
        const int two = (d0.x >> 1) & 1;
        const int N = d1.y;
        const int kcols = P.fam[(d0.x & 1) ? 2 : 0].cols;
        const int parts = tc_partials(N);
        const int buf = it % kTcAccBufs;
        if (it >= kTcAccBufs && !mbar_wait(&acc_empty[buf], uint32_t(it / kTcAccBufs - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = I8 ? umma_idesc_i8(128, N) : umma_idesc_f16(128, N);
        const uint32_t dbase = tmem + uint32_t(kTcAccCol + buf * kTcAccBuf + p * N);
        for (int s = 0; s < d1.w; ++s, ++as) {
          const int aslot = as % C::kAStages;  // B uses the same slot
          if (!mbar_wait(&a_full[aslot], uint32_t(as / C::kAStages) & 1u)) {  // A and B of the stage
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_s = smem_u32(bring + size_t(aslot) * C::kBStageBytes);
          // k steps of this stage: all of them, or only those inside the row (a last stage of 128 k
          // when the stage is 256 k)
          const int ksteps = s == d1.w - 1 && (kcols % kStageK) != 0 ? (kcols % kStageK) / (I8 ? 32 : 16) : C::kKSteps;
          for (int f = f0; f < 1 + two && p < parts; f += kTileStep) {
            const uint32_t acol = tmem + uint32_t(aslot * C::kStageCols + f * C::kTileCols);
            const uint32_t dcol = dbase + uint32_t(f * kTcAccTile);
            for (int kk = p; kk < ksteps; kk += parts) {  // 8 tensor-memory columns, 32 bytes of B per MMA
              const uint64_t bdesc = umma_desc_sw128(b_s + (kk >> 2) * (kTcNMax * 128) + 32 * (kk & 3));
              const uint32_t acc = (s > 0 || kk != p) ? 1u : 0u;
              if constexpr (I8) umma_i8_ts(dcol, acol + 8 * kk, bdesc, idesc, acc);  // 32 k
              else umma_f16_ts(dcol, acol + 8 * kk, bdesc, idesc, acc);               // 16 k
            }
          }
          umma_commit(&a_empty[aslot]);  // frees the A and the B stage
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(done);  // every MMA this thread issued has completed once all issuers' commits arrive
      mbar_wait(done, 0);
    }
  } else if (warp >= kTcWarpDq && warp < kTcWarpEpi) {
    // ------------------------------------------------ dequantize into tensor memory
    const int f = (warp - kTcWarpDq) >> 2;    // tile 0 (warps 2-5) or tile 1 (warps 6-9)
    const int qw = warp & 3;                  // tensor-memory lane quarter this warp may access
    const int r = 32 * qw + lane;             // row of the tile = tensor-memory lane
    const uint32_t tlane = uint32_t(32 * qw) << 16;
    const uint32_t wring_s = smem_u32(wring);
    const int raw_stages = P.raw_stages, raw_stage_bytes = P.raw_stage_bytes;
    int slot_r = 0, as = 0;
    uint32_t ph_r = 0;
    bool ok = true;
    for (int ds = 0; ok; ++ds) {
      int4 d0, d1;
      int4 dd0 = make_int4(0, 0, 0, 0), dd1 = dd0;
      if (lane == 0 && !read_desc(ds, dd0, dd1)) dd0.x = -2;
      d0.x = __shfl_sync(0xffffffffu, dd0.x, 0);
      d0.y = __shfl_sync(0xffffffffu, dd0.y, 0);
      d0.z = __shfl_sync(0xffffffffu, dd0.z, 0);
      d1.w = __shfl_sync(0xffffffffu, dd1.w, 0);
      if (d0.x < 0) break;
      const int fb = (d0.x & 1) ? 2 : 0;
      const bool tile_on = f == 0 || ((d0.x >> 1) & 1);
      const TcFam& F = P.fam[fb + f];
      const bool row_on = tile_on && d0.z + F.m_off + r < F.rows;  // warp-uniform (rows % 32 == 0)
      const int fmt = F.fmt, win = F.win, g = F.g, j = r % g, q = r / g;
      const uint32_t row_base = wring_s + uint32_t(f * 128 * win + j * (128 / g) * win + q * win);
      const int mis0 = j * F.row_bytes;
      const uint32_t tcol = tmem + tlane + uint32_t(f * C::kTileCols);
      const int nst = d1.w;
      const bool wait_b = warp == kTcWarpDq && lane == 0;
      if constexpr (I8) {
        ok = fmt == BQG_I2_ROW
                 ? tc_dq_item<true, BQG_I2_ROW>(nst, row_on, row_base, mis0, raw_stages, raw_stage_bytes, raw_full,
                                                raw_empty, a_full, a_empty, b_full, wait_b, tcol, slot_r, ph_r, as)
                 : tc_dq_item<true, BQG_I4_ROW>(nst, row_on, row_base, mis0, raw_stages, raw_stage_bytes, raw_full,
                                                raw_empty, a_full, a_empty, b_full, wait_b, tcol, slot_r, ph_r, as);
      } else {
        ok = fmt == BQG_Q4_0
                 ? tc_dq_item<false, BQG_Q4_0>(nst, row_on, row_base, mis0, raw_stages, raw_stage_bytes, raw_full,
                                               raw_empty, a_full, a_empty, b_full, wait_b, tcol, slot_r, ph_r, as)
             : fmt == BQG_Q8_0
                 ? tc_dq_item<false, BQG_Q8_0>(nst, row_on, row_base, mis0, raw_stages, raw_stage_bytes, raw_full,
                                               raw_empty, a_full, a_empty, b_full, wait_b, tcol, slot_r, ph_r, as)
                 : tc_dq_item<false, BQG_I4_ROW>(nst, row_on, row_base, mis0, raw_stages, raw_stage_bytes, raw_full,
                                                 raw_empty, a_full, a_empty, b_full, wait_b, tcol, slot_r, ph_r, as);
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= kTcWarpEpi && warp < kTcWarpB) {
    // ------------------------------------------------ epilogue
    const int qw = warp & 3;
    const int r = 32 * qw + lane;
    const uint32_t tlane = uint32_t(32 * qw) << 16;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int4 d0, d1;
      int4 dd0 = make_int4(0, 0, 0, 0), dd1 = dd0;
      if (lane == 0 && !read_desc(it, dd0, dd1)) dd0.x = -2;
      d0 = make_int4(__shfl_sync(0xffffffffu, dd0.x, 0), __shfl_sync(0xffffffffu, dd0.y, 0),
                     __shfl_sync(0xffffffffu, dd0.z, 0), __shfl_sync(0xffffffffu, dd0.w, 0));
      d1 = make_int4(__shfl_sync(0xffffffffu, dd1.x, 0), __shfl_sync(0xffffffffu, dd1.y, 0),
                     __shfl_sync(0xffffffffu, dd1.z, 0), __shfl_sync(0xffffffffu, dd1.w, 0));
      if (d0.x < 0) break;
      const int sh = d0.x & 1, two = (d0.x >> 1) & 1;
      const int fb = sh ? 2 : 0;
      const int ntok = d0.w, N = d1.y, obase = d1.z;
      const int parts = tc_partials(N);
      const int buf = it % kTcAccBufs;
      if (!mbar_wait(&acc_full[buf], uint32_t(it / kTcAccBufs) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + tlane + uint32_t(kTcAccCol + buf * kTcAccBuf);
      if constexpr (I8) {
        // columns 2n and 2n + 1: digit sums D_H, D_L of token n; x W^T = s (256 D_H + D_L - z SX)
        const float* bsc = P.bscale[sh] + obase;
        const int32_t* bsm = P.bsum[sh] + obase;
        if (P.phase == 0) {
          const TcFam& G = P.fam[fb];
          const TcFam& U = P.fam[fb + 1];
          const int row = d0.z + r;
          const bool on = row < G.rows;
          float sg = 0.f, su = 0.f;
          if (on) {
            sg = __ldg(reinterpret_cast<const float*>(G.base + (sh ? 0 : size_t(d0.y) * G.stride) + G.scale_off) + row);
            su = __ldg(reinterpret_cast<const float*>(U.base + (sh ? 0 : size_t(d0.y) * U.stride) + U.scale_off) + row);
          }
          const long long z = tc_i8_zero(G.fmt);
          float* hrow = P.h32[sh] + row;
          const int hs = P.hstride[sh];
          for (int c0 = 0; c0 < N; c0 += 8) {
            int gv[8], uv[8];
            tc_acc8i(acc + uint32_t(c0), N, parts, gv);
            tc_acc8i(acc + uint32_t(kTcAccTile + c0), N, parts, uv);
            if (on) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int n = c0 / 2 + i;
                if (n < ntok) {
                  const float st = __ldg(bsc + n);
                  const long long zx = z * __ldg(bsm + n);
                  const float g = float(256LL * gv[2 * i] + gv[2 * i + 1] - zx) * st * sg;
                  const float u = float(256LL * uv[2 * i] + uv[2 * i + 1] - zx) * st * su;
                  hrow[size_t(obase + n) * hs] = act_fn(P.act, g) * u;
                }
              }
            }
          }
        } else {
          for (int f = 0; f <= two; ++f) {
            const TcFam& D = P.fam[fb + f];
            const int row = d0.z + D.m_off + r;
            const bool on = row < D.rows;
            float sd = 0.f;
            if (on)
              sd = __ldg(reinterpret_cast<const float*>(D.base + (sh ? 0 : size_t(d0.y) * D.stride) + D.scale_off) + row);
            const long long z = tc_i8_zero(D.fmt);
            for (int c0 = 0; c0 < N; c0 += 8) {
              int v[8];
              tc_acc8i(acc + uint32_t(f * kTcAccTile + c0), N, parts, v);
              if (on) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int n = c0 / 2 + i;
                  if (n < ntok) {
                    const float st = __ldg(bsc + n);
                    const long long zx = z * __ldg(bsm + n);
                    const int orow = sh ? obase + n : __ldg(P.perm + obase + n);
                    P.yout[sh][size_t(orow) * P.ystride + row] =
                        float(256LL * v[2 * i] + v[2 * i + 1] - zx) * st * sd;
                  }
                }
              }
            }
          }
        }
      } else if (P.phase == 0) {
        const TcFam& G = P.fam[fb];
        const TcFam& U = P.fam[fb + 1];
        const int row = d0.z + r;
        const bool on = row < G.rows;
        float sg = 1.f, su = 1.f;
        if (on && G.fmt == BQG_I4_ROW) {
          sg = __ldg(reinterpret_cast<const float*>(G.base + (sh ? 0 : size_t(d0.y) * G.stride) + G.scale_off) + row);
          su = __ldg(reinterpret_cast<const float*>(U.base + (sh ? 0 : size_t(d0.y) * U.stride) + U.scale_off) + row);
        }
        __half* hrow = P.hout[sh] + tc_kpos(row, P.hperm[sh]);
        const int hs = P.hstride[sh];
        for (int c0 = 0; c0 < N; c0 += 8) {
          float gv[8], uv[8];
          tc_acc8(acc + uint32_t(c0), N, parts, gv);
          tc_acc8(acc + uint32_t(kTcAccTile + c0), N, parts, uv);
          if (on) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int n = c0 + i;
              if (n < ntok) {
                const float hv = act_fn(P.act, gv[i] * sg) * (uv[i] * su);
                hrow[size_t(obase + n) * hs] = __float2half_rn(hv);
              }
            }
          }
        }
      } else {
        for (int f = 0; f <= two; ++f) {
          const TcFam& D = P.fam[fb + f];
          const int row = d0.z + D.m_off + r;
          const bool on = row < D.rows;
          float sd = 1.f;
          if (on && D.fmt == BQG_I4_ROW)
            sd = __ldg(reinterpret_cast<const float*>(D.base + (sh ? 0 : size_t(d0.y) * D.stride) + D.scale_off) + row);
          for (int c0 = 0; c0 < N; c0 += 8) {
            float v[8];
            tc_acc8(acc + uint32_t(f * kTcAccTile + c0), N, parts, v);
            if (on) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int n = c0 + i;
                if (n < ntok) {
                  const int orow = sh ? obase + n : __ldg(P.perm + obase + n);
                  P.yout[sh][size_t(orow) * P.ystride + row] = v[i] * sd;
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------- activation rows in fp16
// Routed rows in expert-grouped order (row i = x of token perm[i] / top_k) and, with a shared
// expert, its rows in token order; each group of 8 values in the order of the family's format.
__global__ void __launch_bounds__(256) k_moe_xprep(const float* __restrict__ x, const int32_t* __restrict__ perm,
                                                 const int32_t* __restrict__ offsets, int n_experts, int top_k,
                                                 int tokens, int hidden, __half* __restrict__ xg, int nib_r,
                                                 __half* __restrict__ xs, int nib_s) {
  griddep_launch_dependents();
  griddep_wait();
  const int routed_rows = offsets[n_experts];  // pairs with a valid expert id
  const int groups = hidden / 8;
  const long long total = (long long)(routed_rows + (xs != nullptr ? tokens : 0)) * groups;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int row = int(i / groups), m = int(i - (long long)row * groups);
    int src;
    __half* dst;
    int nib;
    if (row < routed_rows) {
      src = __ldg(perm + row) / top_k;
      dst = xg + size_t(row) * hidden + 8 * m;
      nib = nib_r;
    } else {
      src = row - routed_rows;
      dst = xs + size_t(src) * hidden + 8 * m;
      nib = nib_s;
    }
    const float4 a = __ldg(reinterpret_cast<const float4*>(x + size_t(src) * hidden + 8 * m));
    const float4 b = __ldg(reinterpret_cast<const float4*>(x + size_t(src) * hidden + 8 * m) + 1);
    uint4 o;
    if (nib) {  // order 0,4,1,5,2,6,3,7
      o.x = h2_bits(__floats2half2_rn(a.x, b.x));
      o.y = h2_bits(__floats2half2_rn(a.y, b.y));
      o.z = h2_bits(__floats2half2_rn(a.z, b.z));
      o.w = h2_bits(__floats2half2_rn(a.w, b.w));
    } else {
      o.x = h2_bits(__floats2half2_rn(a.x, a.y));
      o.y = h2_bits(__floats2half2_rn(a.z, a.w));
      o.z = h2_bits(__floats2half2_rn(b.x, b.y));
      o.w = h2_bits(__floats2half2_rn(b.z, b.w));
    }
    *reinterpret_cast<uint4*>(dst) = o;
  }
}

// ---------------------------------------------------------------- int8 digit rows (kind::i8 operand B)
// One group of G values (G = 8 for int4, 16 for int2 weights): X = rint(v * inv), clamped to
// |X| <= 32639, split into H = (X + 128) >> 8 and L = X - 256 H (both within [-128, 127]), placed at
// the positions tc_i8_kpos gives.  Returns the sum of the group's X.
template <int G>
__device__ __forceinline__ int tc_digits_group(const float* __restrict__ v, float inv, int8_t* dh, int8_t* dl) {
  float a[G];
#pragma unroll
  for (int q = 0; q < G / 4; ++q) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(v) + q);
    a[4 * q] = t.x;
    a[4 * q + 1] = t.y;
    a[4 * q + 2] = t.z;
    a[4 * q + 3] = t.w;
  }
  uint32_t wh[G / 4], wl[G / 4];
#pragma unroll
  for (int q = 0; q < G / 4; ++q) wh[q] = wl[q] = 0u;
  int sx = 0;
#pragma unroll
  for (int e = 0; e < G; ++e) {
    const int X = max(-32639, min(32639, __float2int_rn(a[e] * inv)));
    const int H = (X + 128) >> 8;
    const int L = X - 256 * H;
    const int pos = tc_i8_kpos(e, G == 16 ? BQG_I2_ROW : BQG_I4_ROW);
    wh[pos >> 2] |= uint32_t(H & 0xFF) << (8 * (pos & 3));
    wl[pos >> 2] |= uint32_t(L & 0xFF) << (8 * (pos & 3));
    sx += X;
  }
  if constexpr (G == 8) {
    *reinterpret_cast<uint2*>(dh) = make_uint2(wh[0], wh[1]);
    *reinterpret_cast<uint2*>(dl) = make_uint2(wl[0], wl[1]);
  } else {
    *reinterpret_cast<uint4*>(dh) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4*>(dl) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
  return sx;
}

// Activation rows of the kind::i8 variant, one warp per row: row i reads source row
// gather[i] / gdiv (or i without gather) of `cols` fp32 values, takes s = max|v| / 32639 and
// writes its digit rows 2i (H) and 2i + 1 (L) to dst [2 rows][cols] bytes, scale[i] = s and
// sum[i] = sum of X, so that v ~= s X = s (256 H + L).  Rows: *rows_ptr if given, else rows.
__global__ void __launch_bounds__(256) k_moe_digits(const float* __restrict__ src, const int32_t* __restrict__ gather,
                                                  int gdiv, const int32_t* __restrict__ rows_ptr, int rows, int cols,
                                                  int fmt, int8_t* __restrict__ dst, float* __restrict__ scale,
                                                  int32_t* __restrict__ sum) {
  griddep_launch_dependents();
  griddep_wait();
  const int n = rows_ptr != nullptr ? *rows_ptr : rows;
  const int lane = threadIdx.x & 31;
  const int nwarps = int((gridDim.x * blockDim.x) >> 5);
  for (int i = int((blockIdx.x * blockDim.x + threadIdx.x) >> 5); i < n; i += nwarps) {
    const int sr = gather != nullptr ? __ldg(gather + i) / gdiv : i;
    const float* v = src + size_t(sr) * cols;
    float m = 0.f;
    for (int k = 4 * lane; k < cols; k += 128) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(v + k));
      m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float inv = m > 0.f ? 32639.f / m : 0.f;
    int8_t* dh = dst + size_t(2 * i) * cols;
    int8_t* dl = dh + cols;
    int sx = 0;
    if (fmt == BQG_I2_ROW) {
      for (int g0 = 16 * lane; g0 < cols; g0 += 512) sx += tc_digits_group<16>(v + g0, inv, dh + g0, dl + g0);
    } else {
      for (int g0 = 8 * lane; g0 < cols; g0 += 256) sx += tc_digits_group<8>(v + g0, inv, dh + g0, dl + g0);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    if (lane == 0) {
      scale[i] = m / 32639.f;
      sum[i] = sx;
    }
  }
}

// ---------------------------------------------------------------- host side
inline int tc_row_bytes(int fmt, int cols) {
  return fmt == BQG_Q8_0 ? cols / 32 * 34 : fmt == BQG_Q4_0 ? cols / 32 * 18 : fmt == BQG_I2_ROW ? cols / 4 : cols / 2;
}

// Geometry of one family on the tensor-core path; false when the shape is not supported there
// (k not a multiple of the stage, or rows not a whole number of super-rows).  i8: the kind::i8
// variant (int4 and int2 only, k a multiple of 128); otherwise kind::f16 (Q8_0, Q4_0, int4).
inline bool tc_fam(int fmt, const void* base, size_t stride, int rows, int cols, int m_off, TcFam* out,
                   bool i8 = false) {
  if (i8 ? (fmt != BQG_I4_ROW && fmt != BQG_I2_ROW) : fmt == BQG_I2_ROW) return false;
  if (cols % (i8 ? 128 : 64) != 0 || rows % 32 != 0) return false;
  TcFam F{};
  F.base = static_cast<const uint8_t*>(base);
  F.stride = (long long)stride;
  F.fmt = fmt;
  F.rows = rows;
  F.cols = cols;
  F.row_bytes = tc_row_bytes(fmt, cols);
  F.g = (F.row_bytes % 16 == 0) ? 1 : (F.row_bytes % 8 == 0) ? 2 : (F.row_bytes % 4 == 0) ? 4 : 0;
  if (F.g == 0 || rows % F.g != 0) return false;
  if (fmt == BQG_I4_ROW || fmt == BQG_I2_ROW) {
    F.raw_k = tc_raw_k(fmt);
    F.cb = tc_raw_cb(fmt);
    F.win = tc_raw_win(fmt);  // rows are multiples of 32 (int4) or 16 (int2) bytes: chunks start 16-byte aligned
    F.scale_off = int((size_t(rows) * F.row_bytes + 15) / 16 * 16);
  } else {
    F.raw_k = tc_raw_k(fmt);
    F.cb = tc_raw_cb(fmt);
    F.win = tc_raw_win(fmt);  // chunk (288 or 272 bytes) + up to 12 bytes of misalignment
  }
  F.m_off = m_off;
  *out = F;
  return true;
}

// [expert][super-row][bytes] view of a family, 8-byte elements, boxes of one window x 128/g
// super-rows of one expert.
inline int tc_encode_amap(CUtensorMap* map, const TcFam& F, int n_experts) {
  EncodeTiledFn encode = encode_tiled_fn();
  if (encode == nullptr) return BQG_ERR_CUDA;
  const cuuint64_t srow = cuuint64_t(F.g) * F.row_bytes;
  const cuuint64_t mat = (cuuint64_t(F.rows) * F.row_bytes + 15) / 16 * 16;
  const cuuint64_t estride = n_experts > 1 ? cuuint64_t(F.stride) : mat;
  const cuuint64_t dims[3] = {srow / 8, cuuint64_t(F.rows / F.g), cuuint64_t(n_experts)};
  const cuuint64_t strides[2] = {srow, estride};
  const cuuint32_t box[3] = {cuuint32_t(F.win / 8), cuuint32_t(128 / F.g), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<uint8_t*>(F.base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return BQG_ERR_CUDA;
  return BQG_OK;
}

// fp16 [rows x cols] activation rows, boxes of 64 k x 16 rows with 128-byte swizzle.
inline int tc_encode_bmap(CUtensorMap* map, const __half* base, int rows, int cols) {
  EncodeTiledFn encode = encode_tiled_fn();
  if (encode == nullptr) return BQG_ERR_CUDA;
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows < 1 ? 1 : rows)};
  const cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return BQG_ERR_CUDA;
  return BQG_OK;
}

// int8 digit rows [rows x cols] bytes (kind::i8 operand B), boxes of 128 k x 16 rows, 128-byte swizzle.
inline int tc_encode_bmap_i8(CUtensorMap* map, const int8_t* base, int rows, int cols) {
  EncodeTiledFn encode = encode_tiled_fn();
  if (encode == nullptr) return BQG_ERR_CUDA;
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows < 1 ? 1 : rows)};
  const cuuint64_t strides[1] = {cuuint64_t(cols)};
  const cuuint32_t box[2] = {128, 16};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return BQG_ERR_CUDA;
  return BQG_OK;
}

inline size_t tc_smem_bytes(int raw_stages, int raw_stage_bytes) {
  return kTcFixedSmem + size_t(raw_stages) * raw_stage_bytes;
}

// Ring depth for a window size: as many raw stages as fit the shared memory.
inline void tc_raw_ring(int win, int* stages, int* stage_bytes) {
  *stage_bytes = 2 * 128 * win;
  int n = int((kTcMaxSmem - kTcFixedSmem) / size_t(*stage_bytes));
  *stages = n > kTcRawMax ? kTcRawMax : n;
}

inline SmemAttrOnce g_tc_attr;     // k_moe_tc<false>
inline SmemAttrOnce g_tc_attr_i8;  // k_moe_tc<true>

}  // namespace bqg
