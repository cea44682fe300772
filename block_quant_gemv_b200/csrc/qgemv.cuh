// Dequantize-fused GEMV over block-quantized weights (Q8_0, Q4_0, packed int4 with per-row
// scale), one persistent kernel for a single matrix or for a whole decode step's list.
//
// What it computes (Camelid README, "Engine status" and "Gemma 4"; colibri wiki summary,
// "구현 범위"):  y_r = sum_b d_rb * sum_i q_rbi x_{32b+i}  (Q8_0; Q4_0 with q-8),
//                y_r = s_r * sum_i q_ri x_i                 (int4 with per-row scale).
//
// Design (B200):
//  * The problem list is one byte stream.  Each CTA (one per SM) owns a contiguous,
//    byte-balanced range of rows, cut into stages of whole rows (<= 24 KB).
//  * A producer warp streams the stages with 1-D bulk copies (TMA) into a 4-deep shared
//    memory ring, completing on mbarriers; rows keep their canonical byte layout (18/34-byte
//    blocks), unaligned starts are handled by copying from the 16-byte boundary below.
//  * 16 consumer warps: thread t owns "unit" p = t % P of every row (a pair of blocks, one
//    block, or 32/64 int4 weights) and row group g = t / P.  Its 64 x values stay in
//    registers for the whole matrix, so each weight byte is read once from shared memory and
//    x costs no shared-memory traffic.
//  * Dequantization uses byte permutes into the fp32 mantissa: a nibble q becomes the float
//    128+q exactly (bits 0x43qq0000), an int8 becomes 2^23+128+q; sums are fp32 FMAs and the
//    constant offset is removed with a per-unit sum of x.
//  * Per-(row, unit) partials go to shared memory; one stage later each consumer warp sums a
//    few rows in a fixed order (warp butterfly) and writes y.  Results are deterministic.
#pragma once

#include "common.cuh"

namespace bqg {

constexpr int kGemvConsumerWarps = 15;  // + 1 producer = 16 warps: 4 per SM sub-partition, 128 registers each
constexpr int kGemvCompute = kGemvConsumerWarps * 32;       // consumer threads
constexpr int kGemvThreads = kGemvCompute + 32;             // + one producer warp
constexpr int kGemvStages = 4;
constexpr int kGemvStageBytes = 24576;                      // payload of one stage (whole rows)
constexpr int kGemvStageAlloc = kGemvStageBytes + 48;       // + slack for unaligned head / tail
constexpr int kGemvPartSlots = kGemvStages + 2;             // partial buffers (see reduce lag)
constexpr int kGemvPartFloats = kGemvStageBytes / 16;       // units per stage <= bytes / 16
constexpr size_t kGemvSmemBytes = size_t(kGemvStages) * kGemvStageAlloc +
                                  size_t(kGemvPartSlots) * kGemvPartFloats * sizeof(float) +
                                  2 * kGemvStages * sizeof(uint64_t);

// Unit kinds: how many weights a consumer thread handles per row, and their byte size.
enum UnitKind : int {
  kQ8Pair = 0,   // two Q8_0 blocks, 68 bytes, 64 weights (cols/32 even)
  kQ8One = 1,    // one Q8_0 block, 34 bytes, 32 weights (cols/32 odd)
  kQ4Pair = 2,   // two Q4_0 blocks, 36 bytes, 64 weights
  kQ4One = 3,    // one Q4_0 block, 18 bytes, 32 weights
  kI4x64 = 4,    // 64 int4 weights, 32 bytes (cols % 64 == 0)
  kI4x32 = 5     // 32 int4 weights, 16 bytes
};

struct GemvProb {
  const uint8_t* W;
  const float* x;
  float* y;
  long long byte_start;  // offset of this matrix's rows in the concatenated stream
  int rows;
  int cols;
  int kind;       // UnitKind
  int row_bytes;  // bytes of one row of packed weights
  int units;      // units per row (P)
  int scale_off;  // I4: byte offset of the fp32 row scales, else 0
};

template <int MAXP>
struct GemvParams {
  int n;
  int pad;
  long long total_bytes;
  GemvProb p[MAXP];
};

__host__ __device__ constexpr int unit_bytes(int kind) {
  return kind == kQ8Pair ? 68 : kind == kQ8One ? 34 : kind == kQ4Pair ? 36 : kind == kQ4One ? 18 : kind == kI4x64 ? 32 : 16;
}
__host__ __device__ constexpr int unit_weights(int kind) {
  return (kind == kQ8Pair || kind == kQ4Pair || kind == kI4x64) ? 64 : 32;
}

// ---------------------------------------------------------------- dequant + dot helpers
// Nibbles: bytes of `lo` hold elements 0,2,4,6 and bytes of `hi` elements 1,3,5,7 (each 0..15).
// __byte_perm(v, 0x43, 0x4k55) = 0x43 << 24 | byte_k(v) << 16, the float 128 + byte_k(v).
__device__ __forceinline__ void dot8_nib(uint32_t lo, uint32_t hi, const float* x, float& a0, float& a1) {
  a0 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4055u)), x[0], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4055u)), x[1], a1);
  a0 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4155u)), x[2], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4155u)), x[3], a1);
  a0 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4255u)), x[4], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4255u)), x[5], a1);
  a0 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4355u)), x[6], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4355u)), x[7], a1);
}

// Q4_0 word (8 unsigned nibbles, element 2m low / 2m+1 high nibble of byte m): adds (128+q)*x.
__device__ __forceinline__ void dot8_q4(uint32_t w, const float* x, float& a0, float& a1) {
  dot8_nib(w & 0x0F0F0F0Fu, (w >> 4) & 0x0F0F0F0Fu, x, a0, a1);
}

// int4 word (two's-complement nibbles): xor 8 maps q to q+8 in 0..15; adds (136+q)*x.
__device__ __forceinline__ void dot8_i4(uint32_t w, const float* x, float& a0, float& a1) {
  dot8_nib((w ^ 0x08080808u) & 0x0F0F0F0Fu, ((w >> 4) ^ 0x08080808u) & 0x0F0F0F0Fu, x, a0, a1);
}

// Q8_0 word (4 int8): xor 0x80 gives q+128 in 0..255; __byte_perm(u, 0x4B, 0x455k) is the
// float 2^23 + q + 128, so subtracting 2^23 + 128 recovers q exactly.
__device__ __forceinline__ void dot4_q8(uint32_t w, const float* x, float& a0, float& a1) {
  const uint32_t u = w ^ 0x80808080u;
  const float off = 8388736.0f;  // 2^23 + 128
  a0 = fmaf(__uint_as_float(__byte_perm(u, 0x4Bu, 0x4550u)) - off, x[0], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(u, 0x4Bu, 0x4551u)) - off, x[1], a1);
  a0 = fmaf(__uint_as_float(__byte_perm(u, 0x4Bu, 0x4552u)) - off, x[2], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(u, 0x4Bu, 0x4553u)) - off, x[3], a1);
}

// Partial dot product of one unit (bytes at `u` in shared memory) with the thread's x.
// c0/c1: 136 * (sum of x over block 0 / block 1 of the unit) for the nibble formats.
template <int KIND>
__device__ __forceinline__ float unit_dot(const uint8_t* u, const float (&x)[64], float c0, float c1) {
  if constexpr (KIND == kQ4Pair) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(u);  // 4-byte aligned
    uint32_t v[9];
#pragma unroll
    for (int i = 0; i < 9; ++i) v[i] = w[i];
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      dot8_q4(__funnelshift_r(v[k], v[k + 1], 16), &x[8 * k], a0, a1);  // block A: bytes 2..17
      dot8_q4(v[5 + k], &x[32 + 8 * k], b0, b1);                          // block B: bytes 20..35
    }
    const float dA = half_bits_to_float(v[0]);
    const float dB = half_bits_to_float(v[4] >> 16);
    return dA * ((a0 + a1) - c0) + dB * ((b0 + b1) - c1);
  } else if constexpr (KIND == kQ4One) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(u);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
    const uint32_t sh = uint32_t(a & 2) * 8;  // 0 or 16
    uint32_t v[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) v[i] = w[i];
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) dot8_q4(__funnelshift_rc(v[k], v[k + 1], 16 + sh), &x[8 * k], a0, a1);
    const float d = half_bits_to_float(__funnelshift_r(v[0], v[1], sh));
    return d * ((a0 + a1) - c0);
  } else if constexpr (KIND == kQ8Pair) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(u);
    uint32_t v[17];
#pragma unroll
    for (int i = 0; i < 17; ++i) v[i] = w[i];
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      dot4_q8(__funnelshift_r(v[k], v[k + 1], 16), &x[4 * k], a0, a1);  // block A: bytes 2..33
      dot4_q8(v[9 + k], &x[32 + 4 * k], b0, b1);                          // block B: bytes 36..67
    }
    const float dA = half_bits_to_float(v[0]);
    const float dB = half_bits_to_float(v[8] >> 16);
    return dA * (a0 + a1) + dB * (b0 + b1);
  } else if constexpr (KIND == kQ8One) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(u);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
    const uint32_t sh = uint32_t(a & 2) * 8;
    uint32_t v[9];
#pragma unroll
    for (int i = 0; i < 9; ++i) v[i] = w[i];
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) dot4_q8(__funnelshift_rc(v[k], v[k + 1], 16 + sh), &x[4 * k], a0, a1);
    const float d = half_bits_to_float(__funnelshift_r(v[0], v[1], sh));
    return d * (a0 + a1);
  } else if constexpr (KIND == kI4x64) {
    const uint4* w = reinterpret_cast<const uint4*>(u);  // 16-byte aligned
    const uint4 p0 = w[0], p1 = w[1];
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    dot8_i4(p0.x, &x[0], a0, a1);
    dot8_i4(p0.y, &x[8], b0, b1);
    dot8_i4(p0.z, &x[16], a0, a1);
    dot8_i4(p0.w, &x[24], b0, b1);
    dot8_i4(p1.x, &x[32], a0, a1);
    dot8_i4(p1.y, &x[40], b0, b1);
    dot8_i4(p1.z, &x[48], a0, a1);
    dot8_i4(p1.w, &x[56], b0, b1);
    return ((a0 + a1) + (b0 + b1)) - (c0 + c1);
  } else {  // kI4x32
    const uint4 p0 = *reinterpret_cast<const uint4*>(u);
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    dot8_i4(p0.x, &x[0], a0, a1);
    dot8_i4(p0.y, &x[8], b0, b1);
    dot8_i4(p0.z, &x[16], a0, a1);
    dot8_i4(p0.w, &x[24], b0, b1);
    return ((a0 + a1) + (b0 + b1)) - c0;
  }
}

// ---------------------------------------------------------------- CTA work range
// Rows of problem p owned by this CTA: those whose first byte lies in [lo, hi).
__device__ __forceinline__ void owned_rows(const GemvProb& P, long long lo, long long hi, int& r0, int& r1) {
  const long long rb = P.row_bytes;
  long long a = lo - P.byte_start, b = hi - P.byte_start;
  a = a <= 0 ? 0 : (a + rb - 1) / rb;
  b = b <= 0 ? 0 : (b + rb - 1) / rb;
  r0 = int(a < P.rows ? a : P.rows);
  r1 = int(b < P.rows ? b : P.rows);
}

__device__ __forceinline__ int stage_rows(const GemvProb& P) {
  const int sr = kGemvStageBytes / P.row_bytes;
  return sr < 1 ? 1 : sr;
}

// ---------------------------------------------------------------- consumer helpers
struct StageRef {
  int prob;  // -1: none
  int r0, r1;
  int slot_part;
};

template <int MAXP>
__device__ __forceinline__ void reduce_stage(const GemvParams<MAXP>& prm, const StageRef& st, const float* parts,
                                             int warp, int lane) {
  if (st.prob < 0) return;
  const GemvProb& P = prm.p[st.prob];
  const float* part = parts + size_t(st.slot_part) * kGemvPartFloats;
  const int nrows = st.r1 - st.r0;
  for (int i = warp; i < nrows; i += kGemvConsumerWarps) {
    float v = 0.f;
    for (int q = lane; q < P.units; q += 32) v += part[i * P.units + q];
    v = warp_sum(v);
    if (lane == 0) {
      const int row = st.r0 + i;
      if (P.kind == kI4x64 || P.kind == kI4x32)
        v *= __ldg(reinterpret_cast<const float*>(P.W + P.scale_off) + row);
      P.y[row] = v;
    }
  }
}

// One unit's partial dot product, the format chosen at run time (uniform across the CTA).
__device__ __forceinline__ float unit_dot_any(int kind, const uint8_t* u, const float (&x)[64], float c0, float c1) {
  switch (kind) {
    case kQ4Pair: return unit_dot<kQ4Pair>(u, x, c0, c1);
    case kQ8Pair: return unit_dot<kQ8Pair>(u, x, c0, c1);
    case kI4x64: return unit_dot<kI4x64>(u, x, c0, c1);
    case kQ4One: return unit_dot<kQ4One>(u, x, c0, c1);
    case kQ8One: return unit_dot<kQ8One>(u, x, c0, c1);
    default: return unit_dot<kI4x32>(u, x, c0, c1);
  }
}

template <int MAXP>
__global__ void __launch_bounds__(kGemvThreads, 1) k_qgemv(const __grid_constant__ GemvParams<MAXP> prm) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  float* parts = reinterpret_cast<float*>(smem + size_t(kGemvStages) * kGemvStageAlloc);
  uint64_t* full = reinterpret_cast<uint64_t*>(parts + size_t(kGemvPartSlots) * kGemvPartFloats);
  uint64_t* empty = full + kGemvStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemvStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kGemvConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const long long lo = prm.total_bytes * blockIdx.x / gridDim.x;
  const long long hi = prm.total_bytes * (blockIdx.x + 1) / gridDim.x;

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------ producer warp (one elected lane)
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    int s = 0;
    bool ok = true;
    for (int pi = 0; pi < prm.n && ok; ++pi) {
      const GemvProb& P = prm.p[pi];
      int ra, rbnd;
      owned_rows(P, lo, hi, ra, rbnd);
      const int sr = stage_rows(P);
      const uintptr_t wbeg = reinterpret_cast<uintptr_t>(P.W);
      const uintptr_t wend = wbeg + size_t(P.rows) * P.row_bytes;
      for (int r0 = ra; r0 < rbnd; r0 += sr, ++s) {
        const int r1 = min(r0 + sr, rbnd);
        const int slot = s % kGemvStages;
        if (s >= kGemvStages && !mbar_wait(&empty[slot], uint32_t(s / kGemvStages - 1) & 1u)) {
          ok = false;
          break;
        }
        const uintptr_t src = wbeg + size_t(r0) * P.row_bytes;
        const uintptr_t end = src + size_t(r1 - r0) * P.row_bytes;
        const uintptr_t a0 = src & ~uintptr_t(15);
        const uintptr_t lim = wend & ~uintptr_t(15);
        uintptr_t a1 = (end + 15) & ~uintptr_t(15);
        if (a1 > lim) a1 = lim;
        if (a1 < a0) a1 = a0;
        uint8_t* dst = ring + size_t(slot) * kGemvStageAlloc;
        // bytes past the last 16-byte boundary of the matrix: plain loads
        for (uintptr_t b = (a1 > src ? a1 : src); b < end; ++b)
          dst[b - a0] = *reinterpret_cast<const uint8_t*>(b);
        const uint32_t nb = uint32_t(a1 - a0);
        if (nb > 0) {
          mbar_arrive_expect_tx(&full[slot], nb);
          bulk_g2s(dst, reinterpret_cast<const void*>(a0), nb, &full[slot], pol);
        } else {
          mbar_arrive(&full[slot]);
        }
      }
    }
    if (!ok) {
      // wait (bounded) for the copies already issued so none lands after the CTA exits
      for (int q = (s > kGemvStages ? s - kGemvStages : 0); q < s; ++q)
        mbar_wait(&full[q % kGemvStages], uint32_t(q / kGemvStages) & 1u);
    }
    return;
  }

  // ------------------------------------------------ consumer warps
  const int t = warp * 32 + lane;
  int s = 0;
  StageRef prev{-1, 0, 0, 0};
  float x[64];
  for (int pi = 0; pi < prm.n; ++pi) {
    const GemvProb& P = prm.p[pi];
    int ra, rbnd;
    owned_rows(P, lo, hi, ra, rbnd);
    if (ra >= rbnd) continue;
    const int kind = P.kind;
    const int units = P.units;
    const int groups = kGemvCompute / units;
    const int g = t / units;
    const int p = t - g * units;
    const bool active = g < groups;
    const int uw = unit_weights(kind);
    const int ub = unit_bytes(kind);

    // this thread's x values stay in registers for the whole matrix
    float c0 = 0.f, c1 = 0.f;
    if (active) {
      const float4* xs = reinterpret_cast<const float4*>(P.x + size_t(p) * uw);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < uw / 4) v = __ldg(xs + i);
        x[4 * i] = v.x;
        x[4 * i + 1] = v.y;
        x[4 * i + 2] = v.z;
        x[4 * i + 3] = v.w;
      }
      if (kind != kQ8Pair && kind != kQ8One) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) s0 += x[i];
#pragma unroll
        for (int i = 32; i < 64; ++i) s1 += x[i];
        c0 = 136.f * s0;
        c1 = 136.f * s1;
      }
    }

    const int sr = stage_rows(P);
    for (int r0 = ra; r0 < rbnd; r0 += sr, ++s) {
      const int r1 = min(r0 + sr, rbnd);
      const int slot = s % kGemvStages;
      if (!mbar_wait(&full[slot], uint32_t(s / kGemvStages) & 1u)) return;
      const uintptr_t src = reinterpret_cast<uintptr_t>(P.W) + size_t(r0) * P.row_bytes;
      const uint8_t* base = ring + size_t(slot) * kGemvStageAlloc + (src & 15);
      const int pslot = s % kGemvPartSlots;
      float* part = parts + size_t(pslot) * kGemvPartFloats;
      if (active) {
        // rows of this stage owned by group g: (r - ra) % groups == g
        int r = r0 + ((g - (r0 - ra) % groups) % groups + groups) % groups;
        for (; r < r1; r += groups) {
          const int i = r - r0;
          part[i * units + p] = unit_dot_any(kind, base + size_t(i) * P.row_bytes + size_t(p) * ub, x, c0, c1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      // reduce the previous stage once every consumer warp has released it
      if (prev.prob >= 0) {
        const int ps = s - 1;
        if (!mbar_wait(&empty[ps % kGemvStages], uint32_t(ps / kGemvStages) & 1u)) return;
        reduce_stage(prm, prev, parts, warp, lane);
      }
      prev.prob = pi;
      prev.r0 = r0;
      prev.r1 = r1;
      prev.slot_part = pslot;
    }
  }
  if (prev.prob >= 0) {
    const int ps = s - 1;
    if (!mbar_wait(&empty[ps % kGemvStages], uint32_t(ps / kGemvStages) & 1u)) return;
    reduce_stage(prm, prev, parts, warp, lane);
  }
}

}  // namespace bqg
