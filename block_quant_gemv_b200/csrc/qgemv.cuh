// Dequantize-fused GEMV over block-quantized weights (Q8_0, Q4_0, packed int4 with per-row
// scale), one persistent kernel for a single matrix or for a whole decode step's list.
//
// What it computes (Camelid README, "Engine status" and "Gemma 4"; colibri wiki summary,
// "구현 범위"):  y_r = sum_b d_rb * sum_i q_rbi x_{32b+i}  (Q8_0; Q4_0 with q-8),
//                y_r = s_r * sum_i q_ri x_i                 (int4 with per-row scale).
//
// Design (B200):
//  * The problem list is one stream of rows.  Each CTA (one per SM) owns a contiguous range of
//    rows of about equal cost (bytes, with nibble-format bytes weighted 1.5; computed on the
//    host), cut into stages of whole rows.
//  * A producer warp streams the stages with 1-D bulk copies (TMA) into two 72 KB shared-memory
//    slots (double buffering), completing on mbarriers.  Rows keep their canonical byte
//    layout (18/34-byte blocks); an unaligned start is copied from the 16-byte boundary below.
//  * 15 consumer warps.  A row is split into "units" (a pair of blocks, one block, or 32/64
//    int4 weights); a row group of W = ceil(units/32) warps owns whole rows, lane l of its
//    warp j handling unit 32j+l.  Each thread keeps its unit's x (in the integer form below) in
//    registers for the whole matrix: each weight byte is read once from shared memory and x
//    costs no shared-memory traffic in the loop.  x itself is bulk-copied into shared memory by the
//    producer one matrix ahead.  Two rows are processed together for more independent chains.
//  * Integer dot products: each thread converts its unit of x once per matrix to 16-bit fixed
//    point (per-unit scale), split into high and low bytes; a 4-byte weight word then costs two
//    dp4a (Q8_0), or two masks and four dp4a (nibble formats), with exact int32 sums per block.  The block
//    scale and the sum over blocks are fp32.  (dp4a has about 2.4x the throughput per weight of
//    an fp32 decode by byte permutes plus FMAs on B200, which keeps the kernel memory-bound.)
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
  kI4x32 = 5,    // 32 int4 weights, 16 bytes
  kI2x64 = 6     // 64 int2 weights, 16 bytes (cols % 64 == 0)
};

struct GemvProb {
  const uint8_t* W;
  const float* x;
  float* y;
  long long byte_start;  // host: the matrix's first cost unit in the whole list (partitioning)
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
  int am_p;                    // problem whose y is reduced to its argmax (greedy token), or -1
  long long total_bytes;
  int am_ctas;                 // CTAs that hold rows of problem am_p (they alone take part)
  int am_pad;
  int32_t* am_token;           // argmax index of y[am_p] (ties: the lower index)
  float* am_value;             // its value (may be null)
  unsigned long long* am_state;  // [2]: packed running maximum, CTA completion count (zero between calls)
  GemvProb p[MAXP];
  CtaRange cta[kGemvMaxGrid];
};

// ---------------------------------------------------------------- greedy argmax of one output
// A running (value, row) maximum: equal values keep the lower row.
__device__ __forceinline__ void am_take(float& bv, int& bi, float v, int i) {
  if (v > bv || (v == bv && i < bi)) {
    bv = v;
    bi = i;
  }
}
// 64-bit key whose unsigned order is (value, then lower row first): the value's bits made
// order-preserving (sign flipped for positives, all bits for negatives; -0.0 taken as +0.0) in
// the high word, the complemented row in the low word.
__device__ __forceinline__ unsigned long long am_pack(float v, int i) {
  if (v == 0.f) v = 0.f;
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(i));
}
__device__ __forceinline__ void am_unpack(unsigned long long key, float& v, int& i) {
  const uint32_t u = static_cast<uint32_t>(key >> 32);
  v = __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
  i = static_cast<int>(~static_cast<uint32_t>(key & 0xffffffffu));
}

__host__ __device__ constexpr int unit_bytes(int kind) {
  return kind == kQ8Pair ? 68 : kind == kQ8One ? 34 : kind == kQ4Pair ? 36 : kind == kQ4One ? 18 : kind == kI4x64 ? 32 : 16;
}
__host__ __device__ constexpr int unit_weights(int kind) {
  return (kind == kQ8Pair || kind == kQ4Pair || kind == kI4x64 || kind == kI2x64) ? 64 : 32;
}
__host__ __device__ constexpr bool is_i2(int kind) { return kind == kI2x64; }
// Formats with one fp32 scale per row (int4 and int2): applied to the row's sum by the caller.
__host__ __device__ constexpr bool is_i4(int kind) { return kind == kI4x64 || kind == kI4x32 || kind == kI2x64; }
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
// x of one unit (32 or 64 values) in 16-bit fixed point: x_i ~= s * X_i with X_i =
// round(x_i * 32767 / max|x|) (per unit, so |X_i| <= 32767), split into a signed high byte and
// an unsigned low byte, X_i = 256 * H_i + L_i, packed four per word in the order in which the
// weight bytes hold their elements.  The integer dot products sum_i q_i X_i are then exact
// (dp4a, int32) for every block, and only the per-block scaling and the sum over blocks use
// fp32.  The quantization of x is the only approximation: |x_i - s X_i| <= max|x| / 65534,
// about 3e-5 of a typical |y| for Gaussian x.
//   nibble formats: word 2m holds elements 8m, 8m+2, 8m+4, 8m+6 (low nibbles of bytes 4m..4m+3),
//                   word 2m+1 holds 8m+1, 8m+3, 8m+5, 8m+7 (high nibbles);
//   Q8_0:           word m holds elements 4m..4m+3.
struct XUnit {
  uint32_t h[16];  // high bytes (signed)
  uint32_t l[16];  // low bytes (unsigned)
  int c0, c1;      // nibble formats: -8 * sum of X over block 0 / block 1 (the q - 8 offset)
  float s;         // x_i ~= s * X_i
};

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {  // a unsigned bytes, b signed
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {  // a signed bytes, b unsigned
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Bytes k of four integers as one word (k = 0: low bytes, k = 1: second bytes).
__device__ __forceinline__ uint32_t pack_byte(int a, int b, int c, int d, int k) {
  const uint32_t sel = k == 0 ? 0x0040u : 0x0051u;
  return __byte_perm(__byte_perm(uint32_t(a), uint32_t(b), sel), __byte_perm(uint32_t(c), uint32_t(d), sel), 0x5410u);
}

// Converts one unit's x values (see XUnit).
template <int KIND>
__device__ __forceinline__ void quantize_unit(const float (&xv)[unit_weights(KIND)], XUnit& X) {
  constexpr int UW = unit_weights(KIND);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < UW; ++i) amax = fmaxf(amax, fabsf(xv[i]));
  const float inv = amax > 0.f ? 32767.f / amax : 0.f;
  X.s = amax * (1.f / 32767.f);
  int xi[UW];
#pragma unroll
  for (int i = 0; i < UW; ++i) xi[i] = __float2int_rn(xv[i] * inv);
  if constexpr (is_q8(KIND)) {
#pragma unroll
    for (int m = 0; m < UW / 4; ++m) {
      X.h[m] = pack_byte(xi[4 * m], xi[4 * m + 1], xi[4 * m + 2], xi[4 * m + 3], 1);
      X.l[m] = pack_byte(xi[4 * m], xi[4 * m + 1], xi[4 * m + 2], xi[4 * m + 3], 0);
    }
    X.c0 = X.c1 = 0;
  } else if constexpr (is_i2(KIND)) {
    // word 4m + k: elements 16m + k, 16m + 4 + k, 16m + 8 + k, 16m + 12 + k (the 2-bit values in
    // bits 2k..2k+1 of the four bytes of weight word m); the -2 offset of t ^ 2 = t + 2 goes to c0
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        X.h[4 * m + k] = pack_byte(xi[16 * m + k], xi[16 * m + 4 + k], xi[16 * m + 8 + k], xi[16 * m + 12 + k], 1);
        X.l[4 * m + k] = pack_byte(xi[16 * m + k], xi[16 * m + 4 + k], xi[16 * m + 8 + k], xi[16 * m + 12 + k], 0);
      }
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 64; ++i) sum += xi[i];
    X.c0 = -2 * sum;
    X.c1 = 0;
  } else {
#pragma unroll
    for (int m = 0; m < UW / 8; ++m) {
      X.h[2 * m] = pack_byte(xi[8 * m], xi[8 * m + 2], xi[8 * m + 4], xi[8 * m + 6], 1);
      X.l[2 * m] = pack_byte(xi[8 * m], xi[8 * m + 2], xi[8 * m + 4], xi[8 * m + 6], 0);
      X.h[2 * m + 1] = pack_byte(xi[8 * m + 1], xi[8 * m + 3], xi[8 * m + 5], xi[8 * m + 7], 1);
      X.l[2 * m + 1] = pack_byte(xi[8 * m + 1], xi[8 * m + 3], xi[8 * m + 5], xi[8 * m + 7], 0);
    }
    int s0 = 0, s1 = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) s0 += xi[i];
#pragma unroll
    for (int i = 32; i < UW; ++i) s1 += xi[i];
    X.c0 = -8 * s0;
    X.c1 = -8 * s1;
  }
}

// Loads one unit's x from xs (shared or global memory, 16-byte aligned) and converts it.
template <int KIND>
__device__ __forceinline__ void build_x(const float* xs, XUnit& X) {
  constexpr int UW = unit_weights(KIND);
  float xv[UW];
#pragma unroll
  for (int i = 0; i < UW / 4; ++i) {
    const float4 v = reinterpret_cast<const float4*>(xs)[i];
    xv[4 * i] = v.x;
    xv[4 * i + 1] = v.y;
    xv[4 * i + 2] = v.z;
    xv[4 * i + 3] = v.w;
  }
  quantize_unit<KIND>(xv, X);
}

// sum over the 8 elements of one nibble word of u * X (u the unsigned nibble), into (h, l).
__device__ __forceinline__ void dot8_nib(uint32_t lo, uint32_t hi, uint32_t xh0, uint32_t xh1, uint32_t xl0,
                                         uint32_t xl1, int& h, int& l) {
  h = dp4a_us(lo, xh0, h);
  h = dp4a_us(hi, xh1, h);
  l = dp4a_uu(lo, xl0, l);
  l = dp4a_uu(hi, xl1, l);
}

// Partial dot products of the same unit of NR rows (shared-memory byte addresses u[n]) with
// the thread's x.  Two rows at once give twice the independent chains per thread.
template <int KIND, int NR>
__device__ __forceinline__ void units_dot(const uint32_t (&u)[NR], const XUnit& X, float (&out)[NR]) {
  if constexpr (KIND == kQ4Pair) {
    uint32_t v[NR][9];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 9; ++i) v[n][i] = lds32(u[n] + 4 * i);  // 4-byte aligned
    int ha[NR], la[NR], hb[NR], lb[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      ha[n] = hb[n] = 0;
      la[n] = X.c0;
      lb[n] = X.c1;
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const uint32_t wa = __funnelshift_r(v[n][m], v[n][m + 1], 16);  // block A: qs bytes 2..17
        dot8_nib(wa & 0x0F0F0F0Fu, (wa >> 4) & 0x0F0F0F0Fu, X.h[2 * m], X.h[2 * m + 1], X.l[2 * m], X.l[2 * m + 1],
                 ha[n], la[n]);
        const uint32_t wb = v[n][5 + m];  // block B: qs bytes 20..35
        dot8_nib(wb & 0x0F0F0F0Fu, (wb >> 4) & 0x0F0F0F0Fu, X.h[8 + 2 * m], X.h[9 + 2 * m], X.l[8 + 2 * m],
                 X.l[9 + 2 * m], hb[n], lb[n]);
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = X.s * fmaf(half_bits_to_float(v[n][0]), float(ha[n] * 256 + la[n]),
                          half_bits_to_float(v[n][4] >> 16) * float(hb[n] * 256 + lb[n]));
  } else if constexpr (KIND == kQ4One) {
    uint32_t v[NR][5], sh[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      const uint32_t w = u[n] & ~3u;
      sh[n] = (u[n] & 2u) * 8;  // 0 or 16
#pragma unroll
      for (int i = 0; i < 5; ++i) v[n][i] = lds32(w + 4 * i);
    }
    int h[NR], l[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      h[n] = 0;
      l[n] = X.c0;
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const uint32_t w = __funnelshift_rc(v[n][m], v[n][m + 1], 16 + sh[n]);
        dot8_nib(w & 0x0F0F0F0Fu, (w >> 4) & 0x0F0F0F0Fu, X.h[2 * m], X.h[2 * m + 1], X.l[2 * m], X.l[2 * m + 1], h[n],
                 l[n]);
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = X.s * half_bits_to_float(__funnelshift_r(v[n][0], v[n][1], sh[n])) * float(h[n] * 256 + l[n]);
  } else if constexpr (KIND == kQ8Pair) {
    uint32_t v[NR][17];
#pragma unroll
    for (int n = 0; n < NR; ++n)
#pragma unroll
      for (int i = 0; i < 17; ++i) v[n][i] = lds32(u[n] + 4 * i);
    int ha[NR], la[NR], hb[NR], lb[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) ha[n] = la[n] = hb[n] = lb[n] = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const uint32_t wa = __funnelshift_r(v[n][m], v[n][m + 1], 16);  // block A: q bytes 2..33
        ha[n] = dp4a_ss(wa, X.h[m], ha[n]);
        la[n] = dp4a_su(wa, X.l[m], la[n]);
        const uint32_t wb = v[n][9 + m];  // block B: q bytes 36..67
        hb[n] = dp4a_ss(wb, X.h[8 + m], hb[n]);
        lb[n] = dp4a_su(wb, X.l[8 + m], lb[n]);
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = X.s * fmaf(half_bits_to_float(v[n][0]), float(ha[n] * 256 + la[n]),
                          half_bits_to_float(v[n][8] >> 16) * float(hb[n] * 256 + lb[n]));
  } else if constexpr (KIND == kQ8One) {
    uint32_t v[NR][9], sh[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      const uint32_t w = u[n] & ~3u;
      sh[n] = (u[n] & 2u) * 8;
#pragma unroll
      for (int i = 0; i < 9; ++i) v[n][i] = lds32(w + 4 * i);
    }
    int h[NR], l[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) h[n] = l[n] = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const uint32_t w = __funnelshift_rc(v[n][m], v[n][m + 1], 16 + sh[n]);
        h[n] = dp4a_ss(w, X.h[m], h[n]);
        l[n] = dp4a_su(w, X.l[m], l[n]);
      }
#pragma unroll
    for (int n = 0; n < NR; ++n)
      out[n] = X.s * half_bits_to_float(__funnelshift_r(v[n][0], v[n][1], sh[n])) * float(h[n] * 256 + l[n]);
  } else if constexpr (KIND == kI2x64) {  // int2 with per-row scale (applied by the caller): 4 words
    uint32_t q[NR][4];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      const uint4 p0 = lds128(u[n]);  // 16-byte aligned
      q[n][0] = p0.x; q[n][1] = p0.y; q[n][2] = p0.z; q[n][3] = p0.w;
    }
    int h[NR], l[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      h[n] = 0;
      l[n] = X.c0;
    }
    // two's-complement 2-bit t: t ^ 2 = t + 2 in 0..3; plane k of a word = bits 2k..2k+1 of its bytes
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const uint32_t w = q[n][m] ^ 0xAAAAAAAAu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t c = (w >> (2 * k)) & 0x03030303u;
          h[n] = dp4a_us(c, X.h[4 * m + k], h[n]);
          l[n] = dp4a_uu(c, X.l[4 * m + k], l[n]);
        }
      }
#pragma unroll
    for (int n = 0; n < NR; ++n) out[n] = X.s * float(h[n] * 256 + l[n]);
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
    int h[NR], l[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
      h[n] = 0;
      l[n] = X.c0 + X.c1;
    }
    // two's-complement nibble t: t ^ 8 = t + 8 in 0..15, so the q - 8 offset applies as for Q4_0
#pragma unroll
    for (int k = 0; k < NW; ++k)
#pragma unroll
      for (int n = 0; n < NR; ++n)
        dot8_nib((q[n][k] ^ 0x08080808u) & 0x0F0F0F0Fu, ((q[n][k] >> 4) ^ 0x08080808u) & 0x0F0F0F0Fu, X.h[2 * k],
                 X.h[2 * k + 1], X.l[2 * k], X.l[2 * k + 1], h[n], l[n]);
#pragma unroll
    for (int n = 0; n < NR; ++n) out[n] = X.s * float(h[n] * 256 + l[n]);
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
                                            uint64_t* empty, int& s, int& xs_n, XUnit& X, float& am_v, int& am_i) {
  const GemvProb& P = prm.p[pi];
  const bool track = pi == prm.am_p;  // this matrix's rows also feed the greedy argmax
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
  if (active) build_x<KIND>(xs + size_t(p) * UW, X);
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
            units_dot<KIND, 2>(u2, X, v);
          } else {
            const uint32_t u1[1] = {base + uint32_t(i) * row_bytes};
            float o1[1];
            units_dot<KIND, 1>(u1, X, o1);
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
            if (track) am_take(am_v, am_i, v[0], r0 + i);
            if (two) {
              if (is_i4(KIND)) v[1] *= __ldg(scales + i + groups);
              P.y[r0 + i + groups] = v[1];
              if (track) am_take(am_v, am_i, v[1], r0 + i + groups);
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
        if (track) am_take(am_v, am_i, v, row);
      }
    }
  }
  return true;
}

// The CTA's problems in processing order.  A CTA holding rows of the argmax output takes that
// matrix first, so that its share of the greedy argmax is merged early, overlapping the rest of
// its rows, instead of adding a chain of global atomics after the last matrix.
__device__ __forceinline__ int cta_problem(const CtaRange& cr, int am_first, int q) {
  if (am_first < 0) return cr.p0 + q;
  if (q == 0) return am_first;
  const int pi = cr.p0 + q - 1;
  return pi >= am_first ? pi + 1 : pi;
}

// Greedy argmax of y[am_p] over the CTAs that wrote its rows (called by every consumer thread of
// such a CTA, right after those rows): warp, then CTA maximum; one 64-bit max reduction per CTA
// on the packed key, then a release/acquire count; the last of these CTAs decodes the key into
// the token and clears the state.
template <int MAXP>
__device__ __forceinline__ void argmax_merge(const GemvParams<MAXP>& prm, float am_v, int am_i) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, am_v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, am_i, o);
    am_take(am_v, am_i, ov, oi);
  }
  __shared__ float am_wv[kGemvConsumerWarps];
  __shared__ int am_wi[kGemvConsumerWarps];
  if (lane == 0) {
    am_wv[warp] = am_v;
    am_wi[warp] = am_i;
  }
  named_bar_sync(1, kGemvCompute);
  if (threadIdx.x == 0) {
    for (int w = 1; w < kGemvConsumerWarps; ++w) am_take(am_v, am_i, am_wv[w], am_wi[w]);
    unsigned int* count = reinterpret_cast<unsigned int*>(prm.am_state + 1);
    if (am_i != 0x7fffffff)
      asm volatile("red.relaxed.gpu.global.max.u64 [%0], %1;" ::"l"(prm.am_state), "l"(am_pack(am_v, am_i))
                   : "memory");
    unsigned int prev;
    // release: this CTA's maximum is visible before its count; acquire: the last CTA sees them all
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(count) : "memory");
    if (prev == unsigned(prm.am_ctas) - 1u) {
      unsigned long long key;
      asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(key) : "l"(prm.am_state) : "memory");
      float v;
      int i;
      am_unpack(key, v, i);
      *prm.am_token = i;
      if (prm.am_value != nullptr) *prm.am_value = v;
      prm.am_state[0] = 0ull;  // ready for the next call on this stream
      *count = 0u;
    }
  }
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
  const int nprob = p_last >= cr.p0 ? p_last - cr.p0 + 1 : 0;
  int am_first = -1;  // the argmax output, when this CTA holds rows of it
  if (prm.am_p >= cr.p0 && prm.am_p <= p_last) {
    int ra, rb;
    cta_rows(cr, prm.p[prm.am_p], prm.am_p, ra, rb);
    if (ra < rb) am_first = prm.am_p;
  }

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------ producer warp (one elected lane)
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    int s = 0;
    int xs_n = 0;  // problems whose x has been staged
    bool ok = true;
    for (int q = 0; q < nprob && ok; ++q) {
      const int pi = cta_problem(cr, am_first, q);
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
  XUnit X;
  float am_v = -INFINITY;  // greedy argmax: the best (value, row) this thread has written
  int am_i = 0x7fffffff;
  for (int q = 0; q < nprob; ++q) {
    const int pi = cta_problem(cr, am_first, q);
    const GemvProb& P = prm.p[pi];
    int ra, rbnd;
    cta_rows(cr, P, pi, ra, rbnd);
    if (ra >= rbnd) continue;
    // Every consumer warp has finished the previous matrix (including the group reductions
    // that read `red`): row groups may be composed differently from one matrix to the next.
    named_bar_sync(1, kGemvCompute);
    bool ok;
    switch (P.kind) {
      case kQ4Pair: ok = gemv_matrix<kQ4Pair, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
      case kQ8Pair: ok = gemv_matrix<kQ8Pair, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
      case kI4x64: ok = gemv_matrix<kI4x64, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
      case kQ4One: ok = gemv_matrix<kQ4One, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
      case kQ8One: ok = gemv_matrix<kQ8One, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
      case kI2x64: ok = gemv_matrix<kI2x64, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
      default: ok = gemv_matrix<kI4x32, MAXP>(prm, pi, ra, rbnd, ring, xs, red, full, xfull, xfree, empty, s, xs_n, X, am_v, am_i); break;
    }
    // the argmax output comes first: merge this CTA's share now (also after a failed wait, so
    // that the count of the CTAs stays whole)
    if (q == 0 && am_first >= 0) argmax_merge(prm, am_v, am_i);
    if (!ok) break;
  }
}

}  // namespace bqg
