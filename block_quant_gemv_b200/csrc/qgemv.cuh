// Dequantize-fused GEMV over block-quantized weights (Q8_0, Q4_0, packed int4 with per-row
// scale), one persistent kernel for a single matrix or for a whole decode step's list.
//
// What it computes (Camelid README, "Engine status" and "Gemma 4"; colibri wiki summary,
// "구현 범위"):  y_r = sum_b d_rb * sum_i q_rbi x_{32b+i}  (Q8_0; Q4_0 with q-8),
//                y_r = s_r * sum_i q_ri x_i                 (int4 with per-row scale).
//
// Design (B200):
//  * The problem list is one byte stream.  Each CTA (one per SM) owns a contiguous,
//    byte-balanced range of rows (computed on the host), cut into stages of whole rows.
//  * A producer warp streams the stages with 1-D bulk copies (TMA) into two 72 KB shared-memory
//    slots (double buffering), completing on mbarriers.  Rows keep their canonical byte
//    layout (18/34-byte blocks); an unaligned start is copied from the 16-byte boundary below.
//  * 15 consumer warps.  A row is split into "units" (a pair of blocks, one block, or 32/64
//    int4 weights); a row group of W = ceil(units/32) warps owns whole rows, lane l of its
//    warp j handling unit 32j+l.  Each thread keeps its unit's 64 x values (fp32) in registers
//    for the whole matrix: each weight byte is read once from shared memory and x costs no
//    shared-memory traffic in the loop.  x itself is bulk-copied into shared memory by the
//    producer one matrix ahead.  Two rows are processed together for more independent FMAs.
//  * Dequantization uses byte permutes into the fp32 mantissa: a nibble q becomes the float
//    128+q exactly (bits 0x43qq0000), an int8 becomes 2^23+128+q (then minus 2^23+128); sums
//    are fp32 FMAs and the constant offset of the nibble formats is removed with a per-block
//    sum of x.  All products are exact; only the fp32 sums round.
//  * Each row is reduced with a warp butterfly (plus a fixed-order sum over the W warps of a
//    group through shared memory), so results are deterministic.
#pragma once

#include "common.cuh"

namespace bqg {

constexpr int kGemvConsumerWarps = 15;  // + 1 producer = 16 warps: 4 per SM sub-partition, 128 registers each
constexpr int kGemvCompute = kGemvConsumerWarps * 32;       // consumer threads
constexpr int kGemvThreads = kGemvCompute + 32;             // + one producer warp
#ifndef BQG_GEMV_STAGES
#define BQG_GEMV_STAGES 2
#endif
#ifndef BQG_GEMV_STAGE_BYTES
#define BQG_GEMV_STAGE_BYTES 73728
#endif
constexpr int kGemvStages = BQG_GEMV_STAGES;
constexpr int kGemvStageBytes = BQG_GEMV_STAGE_BYTES;       // payload of one stage (whole rows)
constexpr int kGemvStageAlloc = kGemvStageBytes + 48;       // + slack for unaligned head / tail
constexpr int kGemvMaxCols = BQG_MAX_COLS;
constexpr int kGemvRedRows = 40;                            // rows per group per stage when W > 1
constexpr size_t kGemvSmemBytes = size_t(kGemvStages) * kGemvStageAlloc +            // weight ring
                                  size_t(kGemvMaxCols) * sizeof(float) +              // x staging
                                  size_t(2 * kGemvConsumerWarps * kGemvRedRows) * sizeof(float) +
                                  (2 * kGemvStages + 2) * sizeof(uint64_t);

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

constexpr int kGemvMaxGrid = 160;  // >= SM count of a B200 (148)

// Rows owned by one CTA: from row r0 of problem p0 up to (not including) row r1 of problem
// p1, in problem order.  Computed on the host so that the kernel does no 64-bit divisions.
struct CtaRange {
  int p0, r0, p1, r1;
};

template <int MAXP>
struct GemvParams {
  int n;
  int pad;
  long long total_bytes;
  GemvProb p[MAXP];
  CtaRange cta[kGemvMaxGrid];
};

__host__ __device__ constexpr int unit_bytes(int kind) {
  return kind == kQ8Pair ? 68 : kind == kQ8One ? 34 : kind == kQ4Pair ? 36 : kind == kQ4One ? 18 : kind == kI4x64 ? 32 : 16;
}
__host__ __device__ constexpr int unit_weights(int kind) {
  return (kind == kQ8Pair || kind == kQ4Pair || kind == kI4x64) ? 64 : 32;
}
__host__ __device__ constexpr bool is_i4(int kind) { return kind == kI4x64 || kind == kI4x32; }
__host__ __device__ constexpr bool is_q8(int kind) { return kind == kQ8Pair || kind == kQ8One; }

// Geometry shared by host and device: warps per row group, groups, rows per stage.
__host__ __device__ constexpr int gemv_group_warps(int units) { return (units + 31) / 32; }
__host__ __device__ constexpr int gemv_groups(int units) { return kGemvConsumerWarps / gemv_group_warps(units); }
// The most whole rows that fit a stage, rounded down to a multiple of the number of groups so
// that every group owns the same number of rows of each stage.  (groups * row_bytes <= 15 *
// 32 * largest unit <= the stage size, so one row per group always fits.)
__host__ __device__ constexpr int gemv_stage_rows(int units, int row_bytes) {
  return (kGemvStageBytes / row_bytes) / gemv_groups(units) * gemv_groups(units);
}
static_assert(kGemvStageBytes >= kGemvCompute * 68, "a stage must hold one row per row group");

// ---------------------------------------------------------------- dequant + dot helpers
// Nibbles: bytes of `lo` hold elements 0,2,4,6 and bytes of `hi` elements 1,3,5,7 (each 0..15).
// __byte_perm(v, 0x43, 0x4k55) = 0x43 << 24 | byte_k(v) << 16, the float 128 + byte_k(v).
__device__ __forceinline__ void dot8_nib(uint32_t lo, uint32_t hi, const float* x, float& a0, float& a1, float& a2,
                                         float& a3) {
  a0 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4055u)), x[0], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4055u)), x[1], a1);
  a2 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4155u)), x[2], a2);
  a3 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4155u)), x[3], a3);
  a0 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4255u)), x[4], a0);
  a1 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4255u)), x[5], a1);
  a2 = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4355u)), x[6], a2);
  a3 = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4355u)), x[7], a3);
}

// Q4_0 word (8 unsigned nibbles, element 2m low / 2m+1 high nibble of byte m): adds (128+q)*x.
__device__ __forceinline__ void dot8_q4(uint32_t w, const float* x, float& a0, float& a1, float& a2, float& a3) {
  dot8_nib(w & 0x0F0F0F0Fu, (w >> 4) & 0x0F0F0F0Fu, x, a0, a1, a2, a3);
}

// int4 word (two's-complement nibbles): xor 8 maps q to q+8 in 0..15; adds (136+q)*x.
__device__ __forceinline__ void dot8_i4(uint32_t w, const float* x, float& a0, float& a1, float& a2, float& a3) {
  dot8_nib((w ^ 0x08080808u) & 0x0F0F0F0Fu, ((w >> 4) ^ 0x08080808u) & 0x0F0F0F0Fu, x, a0, a1, a2, a3);
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

// Loads one unit's x values from xs into registers and the per-block offset constants of the
// nibble formats: c[b] = 136 * sum of x over block b (sum_i (128+u_i) x_i - c = sum (u_i-8) x_i).
__device__ __forceinline__ void build_x(int kind, const float* xs, float (&x)[64], float& c0, float& c1) {
  const int uw = unit_weights(kind);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < uw / 4) v = reinterpret_cast<const float4*>(xs)[i];
    x[4 * i] = v.x;
    x[4 * i + 1] = v.y;
    x[4 * i + 2] = v.z;
    x[4 * i + 3] = v.w;
  }
  c0 = c1 = 0.f;
  if (!is_q8(kind)) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) s0 += x[i];
#pragma unroll
    for (int i = 32; i < 64; ++i) s1 += x[i];
    c0 = 136.f * s0;
    c1 = 136.f * s1;
  }
}

// Partial dot products of the same unit of NR rows (shared-memory byte addresses u[n]) with
// the thread's x registers.  Two rows at once give twice the independent FMA chains per thread.
template <int KIND, int NR>
__device__ __forceinline__ void units_dot(const uint32_t (&u)[NR], const float (&x)[64], float c0, float c1,
                                          float (&out)[NR]) {
  if constexpr (KIND == kQ4Pair) {
    uint32_t v[NR][9];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 9; ++i) v[n][i] = lds32(u[n] + 4 * i);  // 4-byte aligned
    float a[NR][4], b[NR][4];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) a[n][i] = b[n][i] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        dot8_q4(__funnelshift_r(v[n][m], v[n][m + 1], 16), &x[8 * m], a[n][0], a[n][1], a[n][2], a[n][3]);  // block A
        dot8_q4(v[n][5 + m], &x[32 + 8 * m], b[n][0], b[n][1], b[n][2], b[n][3]);                          // block B
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = half_bits_to_float(v[n][0]) * (((a[n][0] + a[n][1]) + (a[n][2] + a[n][3])) - c0) +
               half_bits_to_float(v[n][4] >> 16) * (((b[n][0] + b[n][1]) + (b[n][2] + b[n][3])) - c1);
  } else if constexpr (KIND == kQ4One) {
    uint32_t v[NR][5], sh[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      const uint32_t w = u[n] & ~3u;
      sh[n] = (u[n] & 2u) * 8;  // 0 or 16
#pragma unroll
      for (int i = 0; i < 5; ++i) v[n][i] = lds32(w + 4 * i);
    }
    float a[NR][4];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) a[n][i] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n)
        dot8_q4(__funnelshift_rc(v[n][m], v[n][m + 1], 16 + sh[n]), &x[8 * m], a[n][0], a[n][1], a[n][2], a[n][3]);
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = half_bits_to_float(__funnelshift_r(v[n][0], v[n][1], sh[n])) *
               (((a[n][0] + a[n][1]) + (a[n][2] + a[n][3])) - c0);
  } else if constexpr (KIND == kQ8Pair) {
    uint32_t v[NR][17];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 17; ++i) v[n][i] = lds32(u[n] + 4 * i);
    float a[NR][2], b[NR][2];
#pragma unroll
    for (int n = 0; n < NR; ++n) a[n][0] = a[n][1] = b[n][0] = b[n][1] = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        dot4_q8(__funnelshift_r(v[n][m], v[n][m + 1], 16), &x[4 * m], a[n][0], a[n][1]);  // block A: bytes 2..33
        dot4_q8(v[n][9 + m], &x[32 + 4 * m], b[n][0], b[n][1]);                          // block B: bytes 36..67
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = half_bits_to_float(v[n][0]) * (a[n][0] + a[n][1]) + half_bits_to_float(v[n][8] >> 16) * (b[n][0] + b[n][1]);
  } else if constexpr (KIND == kQ8One) {
    uint32_t v[NR][9], sh[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      const uint32_t w = u[n] & ~3u;
      sh[n] = (u[n] & 2u) * 8;
#pragma unroll
      for (int i = 0; i < 9; ++i) v[n][i] = lds32(w + 4 * i);
    }
    float a[NR][2];
#pragma unroll
    for (int n = 0; n < NR; ++n) a[n][0] = a[n][1] = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) dot4_q8(__funnelshift_rc(v[n][m], v[n][m + 1], 16 + sh[n]), &x[4 * m], a[n][0], a[n][1]);
#pragma unroll
    for (int n = 0; n < NR; ++n) out[n] = half_bits_to_float(__funnelshift_r(v[n][0], v[n][1], sh[n])) * (a[n][0] + a[n][1]);
  } else {  // int4 with per-row scale (applied by the caller): kI4x64 (8 words) or kI4x32 (4 words)
    constexpr int NW = (KIND == kI4x64) ? 8 : 4;
    uint32_t q[NR][8];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      const uint4 p0 = lds128(u[n]);  // 16-byte aligned
      q[n][0] = p0.x; q[n][1] = p0.y; q[n][2] = p0.z; q[n][3] = p0.w;
      if constexpr (NW == 8) {
        const uint4 p1 = lds128(u[n] + 16);
        q[n][4] = p1.x; q[n][5] = p1.y; q[n][6] = p1.z; q[n][7] = p1.w;
      }
    }
    float a[NR][4], b[NR][4];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) a[n][i] = b[n][i] = 0.f;
#pragma unroll
    for (int k = 0; k < NW; k += 2)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        dot8_i4(q[n][k], &x[8 * k], a[n][0], a[n][1], a[n][2], a[n][3]);
        dot8_i4(q[n][k + 1], &x[8 * k + 8], b[n][0], b[n][1], b[n][2], b[n][3]);
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = (((a[n][0] + a[n][1]) + (a[n][2] + a[n][3])) + ((b[n][0] + b[n][1]) + (b[n][2] + b[n][3]))) - (c0 + c1);
  }
}

// ---------------------------------------------------------------- CTA work range
// Rows [ra, rb) of problem pi owned by this CTA (empty when ra >= rb).
__device__ __forceinline__ void cta_rows(const CtaRange& c, const GemvProb& P, int pi, int& ra, int& rb) {
  ra = pi == c.p0 ? c.r0 : 0;
  rb = pi < c.p1 ? P.rows : (pi == c.p1 ? c.r1 : 0);
  if (pi < c.p0) rb = 0;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// One matrix's rows [ra, rbnd) on the consumer side, specialised for its unit kind.
// Returns false if a bounded wait gave up.
template <int KIND, int MAXP>
__device__ __forceinline__ bool gemv_matrix(const GemvParams<MAXP>& prm, int pi, int ra, int rbnd, uint8_t* ring,
                                            float* xs, float* red, uint64_t* full, uint64_t* xfull, uint64_t* xfree,
                                            uint64_t* empty, int& s, int& xs_n, float (&X)[64]) {
  const GemvProb& P = prm.p[pi];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = P.units, row_bytes = P.row_bytes;
  const int gw = gemv_group_warps(units);
  const int groups = gemv_groups(units);
  const int g = warp / gw, j = warp - g * gw;  // row group, warp within the group
  const int p = 32 * j + lane;                 // this thread's unit
  const bool in_group = g < groups;
  const bool active = in_group && p < units;
  constexpr int UB = unit_bytes(KIND), UW = unit_weights(KIND);

  // x was bulk-copied into xs by the producer; load this thread's x values into registers
  if (!mbar_wait(xfull, uint32_t(xs_n) & 1u)) return false;
  float c0 = 0.f, c1 = 0.f;
  if (active) build_x(KIND, xs + size_t(p) * UW, X, c0, c1);
  mbar_arrive(xfree);
  ++xs_n;

  const uint32_t ring_s = smem_u32(ring);
  const int sr = gemv_stage_rows(units, row_bytes);
  for (int r0 = ra; r0 < rbnd; r0 += sr, ++s) {
    const int r1 = min(r0 + sr, rbnd);
    const int slot = s % kGemvStages;
    if (!mbar_wait(&full[slot], uint32_t(s / kGemvStages) & 1u)) return false;
    const uint32_t src_lo = uint32_t(reinterpret_cast<uintptr_t>(P.W) + size_t(r0) * row_bytes) & 15u;
    const uint32_t base = ring_s + uint32_t(slot) * kGemvStageAlloc + src_lo + uint32_t(p) * UB;
    const int nrows = r1 - r0;
    const int par = s & 1;  // group reduction buffer of this stage (same in every warp)
    int nmine = 0;
    if (in_group) {
      // group g owns rows g, g + groups, ... of the stage; two of them are done together
      const float* scales = reinterpret_cast<const float*>(P.W + P.scale_off) + r0;
      for (int i = g; i < nrows; i += 2 * groups) {
        const bool two = i + groups < nrows;
        float v[2] = {0.f, 0.f};
        if (active) {
          if (two) {
            const uint32_t u2[2] = {base + uint32_t(i) * row_bytes, base + uint32_t(i + groups) * row_bytes};
            units_dot<KIND, 2>(u2, X, c0, c1, v);
          } else {
            const uint32_t u1[1] = {base + uint32_t(i) * row_bytes};
            float o1[1];
            units_dot<KIND, 1>(u1, X, c0, c1, o1);
            v[0] = o1[0];
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {  // two interleaved butterflies
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
          v[1] += __shfl_xor_sync(0xffffffffu, v[1], o);
        }
        if (lane == 0) {
          if (gw == 1) {
            if (is_i4(KIND)) v[0] *= __ldg(scales + i);
            P.y[r0 + i] = v[0];
            if (two) {
              if (is_i4(KIND)) v[1] *= __ldg(scales + i + groups);
              P.y[r0 + i + groups] = v[1];
            }
          } else {
            red[(par * kGemvConsumerWarps + warp) * kGemvRedRows + nmine] = v[0];
            if (two) red[(par * kGemvConsumerWarps + warp) * kGemvRedRows + nmine + 1] = v[1];
          }
        }
        nmine += two ? 2 : 1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (gw > 1 && in_group) {
      // fixed-order sum over the group's warps, by the group's first warp
      named_bar_sync(2 + g, 32 * gw);
      if (j == 0 && lane < nmine) {
        float v = 0.f;
        for (int jj = 0; jj < gw; ++jj) v += red[(par * kGemvConsumerWarps + g * gw + jj) * kGemvRedRows + lane];
        const int row = r0 + g + lane * groups;
        if (is_i4(KIND)) v *= __ldg(reinterpret_cast<const float*>(P.W + P.scale_off) + row);
        P.y[row] = v;
      }
    }
  }
  return true;
}

template <int MAXP>
__global__ void __launch_bounds__(kGemvThreads, 1) k_qgemv(const __grid_constant__ GemvParams<MAXP> prm) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  float* xs = reinterpret_cast<float*>(smem + size_t(kGemvStages) * kGemvStageAlloc);
  float* red = xs + kGemvMaxCols;  // [2][kGemvConsumerWarps][kGemvRedRows]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * kGemvConsumerWarps * kGemvRedRows);
  uint64_t* empty = full + kGemvStages;
  uint64_t* xfull = empty + kGemvStages;  // x of the current problem landed in xs
  uint64_t* xfree = xfull + 1;            // every consumer warp has read xs

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemvStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kGemvConsumerWarps);
    }
    mbar_init(xfull, 1);
    mbar_init(xfree, kGemvCompute);  // every consumer thread releases its own reads of xs
    fence_barrier_init();
  }
  __syncthreads();

  const CtaRange cr = prm.cta[blockIdx.x];
  const int p_last = min(cr.p1, prm.n - 1);

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------ producer warp (one elected lane)
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    int s = 0;
    int xs_n = 0;  // problems whose x has been staged
    bool ok = true;
    for (int pi = cr.p0; pi <= p_last && ok; ++pi) {
      const GemvProb& P = prm.p[pi];
      int ra, rbnd;
      cta_rows(cr, P, pi, ra, rbnd);
      if (ra >= rbnd) continue;
      // stage this problem's x once the consumers have read the previous one
      if (xs_n > 0 && !mbar_wait(xfree, uint32_t(xs_n - 1) & 1u)) {
        ok = false;
        break;
      }
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(xfull, uint32_t(P.cols) * 4u);
      bulk_g2s(xs, P.x, uint32_t(P.cols) * 4u, xfull, pol_x);
      ++xs_n;
      const int sr = gemv_stage_rows(P.units, P.row_bytes);
      const uintptr_t wbeg = reinterpret_cast<uintptr_t>(P.W);
      const uintptr_t wend = wbeg + size_t(P.rows) * P.row_bytes;
      for (int r0 = ra; r0 < rbnd; r0 += sr, ++s) {
        const int r1 = min(r0 + sr, rbnd);
        const int slot = s % kGemvStages;
        if (s >= kGemvStages && !mbar_wait(&empty[slot], uint32_t(s / kGemvStages - 1) & 1u)) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();
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
      if (xs_n > 0) mbar_wait(xfull, uint32_t(xs_n - 1) & 1u);
    }
    return;
  }

  // ------------------------------------------------ consumer warps
  int s = 0;     // stage counter (same sequence as the producer's, and in every consumer warp)
  int xs_n = 0;  // problems whose x has been read
  float X[64];
  for (int pi = cr.p0; pi <= p_last; ++pi) {
    const GemvProb& P = prm.p[pi];
    int ra, rbnd;
    cta_rows(cr, P, pi, ra, rbnd);
    if (ra >= rbnd) continue;
    // Every consumer warp has finished the previous matrix (including the group reductions
    // that read `red`): row groups may be composed differently from one matrix to the next.
    named_bar_sync(1, kGemvCompute);
    bool ok;
    switch (P.kind) {
      case kQ4Pair: ok = gemv_matrix<kQ4Pair, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X); break;
      case kQ8Pair: ok = gemv_matrix<kQ8Pair, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X); break;
      case kI4x64: ok = gemv_matrix<kI4x64, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X); break;
      case kQ4One: ok = gemv_matrix<kQ4One, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X); break;
      case kQ8One: ok = gemv_matrix<kQ8One, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X); break;
      default: ok = gemv_matrix<kI4x32, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X); break;
    }
    if (!ok) return;
  }
}

}  // namespace bqg
