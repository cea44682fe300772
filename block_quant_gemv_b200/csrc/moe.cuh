// Routed Mixture-of-Experts layer on block-quantized experts:
//   y_t = sum_{j<k} w_tj * D_e (act(G_e x_t) * (U_e x_t))  +  shared FFN(x_t),   e = idx[t, j]
//
// Sources: Camelid README, "Gemma 4" (GeGLU experts; dense shared expert + sparse top-8
// branch of the 128-expert MoE); TurboFieldfare wiki, "메모리·전문가 스트리밍" (routed experts
// split from the shared branch; an expert read serves every row routed to it); colibri wiki
// summary, "핵심 아이디어" and "구현 범위" (256 routed int4 experts with per-row scales).
//
// Steps (all on the caller's stream):
//   1. k_moe_prep     block 0: per-expert counts, offsets, the list of touched experts and a
//                     stable permutation of the (token, slot) pairs grouped by expert, in token
//                     order (expert ids outside [0, E) are skipped and flagged); it also zeroes
//                     the work counters.  Other blocks: x of every token in the integer form
//                     the GEMV kernel uses (16-bit fixed point per unit, see XUnit).
//   2. k_moe_gemv     (gate/up) a persistent grouped GEMV over work items = stages of up to
//                     72 KB of rows of one matrix of one touched expert (or of the shared
//                     expert).  Each stage is bulk-copied into shared memory ONCE and applied
//                     to every token routed to that expert, so each touched expert's bytes
//                     are read from HBM once per call.  Items are claimed from a counter, the
//                     shared expert's (all tokens) first.  Outputs g and u per pair.
//   3. k_moe_quant    h = act(g) * u per pair (and for the shared expert), in the integer form.
//   4. k_moe_gemv     (down) the same over the down matrices; one output row per pair.
//   5. k_moe_combine  y_t = sum_j w_tj * out_(t,j) in slot order, plus the shared output.
// Every sum has a fixed order, so results are deterministic.
#pragma once

#include "common.cuh"
#include "host_common.h"
#include "qgemv.cuh"

namespace bqg {

// ---------------------------------------------------------------- activations in integer form
// Records of XUnit in global memory: words [0, UW/4) high bytes, [UW/4, UW/2) low bytes, then
// c0, c1, s; padded to whole 16-byte chunks (9 chunks for 64-value units, 5 for 32).
__host__ __device__ constexpr int xrec_chunks(int kind) { return unit_weights(kind) == 64 ? 9 : 5; }

template <int KIND>
__device__ __forceinline__ void store_xunit(const XUnit& X, uint4* rec) {
  constexpr int UW = unit_weights(KIND), NW = UW / 4;
  uint32_t w[4 * xrec_chunks(KIND)];
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    w[i] = X.h[i];
    w[NW + i] = X.l[i];
  }
  w[2 * NW] = uint32_t(X.c0);
  w[2 * NW + 1] = uint32_t(X.c1);
  w[2 * NW + 2] = __float_as_uint(X.s);
#pragma unroll
  for (int i = 2 * NW + 3; i < 4 * xrec_chunks(KIND); ++i) w[i] = 0u;
#pragma unroll
  for (int c = 0; c < xrec_chunks(KIND); ++c) rec[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

template <int KIND>
__device__ __forceinline__ void load_xunit(const uint4* rec, XUnit& X) {
  constexpr int NW = unit_weights(KIND) / 4;
#pragma unroll
  for (int c = 0; c < xrec_chunks(KIND); ++c) {
    const uint4 v = __ldg(rec + c);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 4 * c + k;  // compile-time after unrolling
      if (i < NW) X.h[i] = w4[k];
      else if (i < 2 * NW) X.l[i - NW] = w4[k];
      else if (i == 2 * NW) X.c0 = int(w4[k]);
      else if (i == 2 * NW + 1) X.c1 = int(w4[k]);
      else if (i == 2 * NW + 2) X.s = __uint_as_float(w4[k]);
    }
  }
}

__device__ __forceinline__ float act_fn(int act, float g) {
  if (act == BQG_ACT_SILU) return g / (1.f + expf(-g));
  const float c = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * g * (1.f + tanhf(c * (g + 0.044715f * g * g * g)));
}

// One conversion job: rows x cols values (row stride cols) -> records [rows][cols / UW].
// With b != nullptr the values are act(a) * b (the gated FFN's hidden activation).
struct QuantJob {
  const float* a;
  const float* b;
  uint4* dst;
  int rows, cols, kind, act;
};
struct QuantJobs {
  QuantJob j[2];
  int n;
};

// One 8-value segment of a unit: the UW/8 segments of a unit sit on consecutive lanes of one
// warp, which share max|x| and the block sums by shuffles.  Every lane of the warp must call
// this (valid = false for lanes past the end).
template <int KIND>
__device__ __forceinline__ void quant_seg(const QuantJob& J, long long gs, bool valid) {
  constexpr int UW = unit_weights(KIND), G = UW / 8, NW = UW / 4;
  const int lane = threadIdx.x & 31;
  const int units = J.cols / UW;
  const long long unit = gs / G;
  const int m = int(gs - unit * G);
  float xv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) xv[i] = 0.f;
  if (valid) {
    const int row = int(unit / units), u = int(unit - (long long)row * units);
    const size_t off = size_t(row) * J.cols + size_t(u) * UW + 8 * m;
    const float4 v0 = *reinterpret_cast<const float4*>(J.a + off);
    const float4 v1 = *reinterpret_cast<const float4*>(J.a + off + 4);
    xv[0] = v0.x; xv[1] = v0.y; xv[2] = v0.z; xv[3] = v0.w;
    xv[4] = v1.x; xv[5] = v1.y; xv[6] = v1.z; xv[7] = v1.w;
    if (J.b != nullptr) {
      const float4 b0 = *reinterpret_cast<const float4*>(J.b + off);
      const float4 b1 = *reinterpret_cast<const float4*>(J.b + off + 4);
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) xv[i] = act_fn(J.act, xv[i]) * bv[i];
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(xv[i]));
#pragma unroll
  for (int o = 1; o < G; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float inv = amax > 0.f ? 32767.f / amax : 0.f;
  int xi[8];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    xi[i] = __float2int_rn(xv[i] * inv);
    sum += xi[i];
  }
  if constexpr (is_i2(KIND)) {
    // int2 record: h/l word 4w + k holds elements 16w + k + 4b (b = 0..3), the order of the 2-bit
    // values in bits 2k..2k+1 of weight word w.  Segment m = 2w + half holds b = 2 half, 2 half + 1
    // of every plane: each lane builds its 16-bit halves, the pair exchanges them, the even lane
    // stores the h words and the odd lane the l words.
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t hh = (uint32_t(xi[k] >> 8) & 0xFFu) | ((uint32_t(xi[4 + k] >> 8) & 0xFFu) << 8);
      const uint32_t ll = (uint32_t(xi[k]) & 0xFFu) | ((uint32_t(xi[4 + k]) & 0xFFu) << 8);
      const uint32_t ph = __shfl_xor_sync(0xffffffffu, hh, 1);
      const uint32_t pl = __shfl_xor_sync(0xffffffffu, ll, 1);
      hw[k] = (m & 1) ? (ph | (hh << 16)) : (hh | (ph << 16));
      lw[k] = (m & 1) ? (pl | (ll << 16)) : (ll | (pl << 16));
    }
    int tot = sum;  // all 64 values of the unit: the t ^ 2 = t + 2 offset
    tot += __shfl_xor_sync(0xffffffffu, tot, 1);
    tot += __shfl_xor_sync(0xffffffffu, tot, 2);
    tot += __shfl_xor_sync(0xffffffffu, tot, 4);
    if (valid) {
      uint32_t* rec = reinterpret_cast<uint32_t*>(J.dst + unit * xrec_chunks(KIND));
      const int w = m >> 1;
      if ((m & 1) == 0) *reinterpret_cast<uint4*>(rec + 4 * w) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      else *reinterpret_cast<uint4*>(rec + NW + 4 * w) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      if (m == 0)
        *reinterpret_cast<uint4*>(rec + 2 * NW) =
            make_uint4(uint32_t(-2 * tot), 0u, __float_as_uint(amax * (1.f / 32767.f)), 0u);
    }
    return;
  }
  uint32_t h0, h1, l0, l1;
  if constexpr (is_q8(KIND)) {  // words 2m, 2m+1 = elements 8m..8m+3, 8m+4..8m+7
    h0 = pack_byte(xi[0], xi[1], xi[2], xi[3], 1);
    h1 = pack_byte(xi[4], xi[5], xi[6], xi[7], 1);
    l0 = pack_byte(xi[0], xi[1], xi[2], xi[3], 0);
    l1 = pack_byte(xi[4], xi[5], xi[6], xi[7], 0);
  } else {  // words 2m, 2m+1 = even, odd elements of 8m..8m+7
    h0 = pack_byte(xi[0], xi[2], xi[4], xi[6], 1);
    h1 = pack_byte(xi[1], xi[3], xi[5], xi[7], 1);
    l0 = pack_byte(xi[0], xi[2], xi[4], xi[6], 0);
    l1 = pack_byte(xi[1], xi[3], xi[5], xi[7], 0);
  }
  // block sums: 4 segments of 32 values per block
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  const int sum_b1 = __shfl_sync(0xffffffffu, sum, (lane & ~(G - 1)) + (G == 8 ? 4 : 0));
  if (valid) {
    uint32_t* rec = reinterpret_cast<uint32_t*>(J.dst + unit * xrec_chunks(KIND));
    *reinterpret_cast<uint2*>(rec + 2 * m) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(rec + NW + 2 * m) = make_uint2(l0, l1);
    if (m == 0) {
      const int c0 = is_q8(KIND) ? 0 : -8 * sum;
      const int c1 = (is_q8(KIND) || G == 4) ? 0 : -8 * sum_b1;
      *reinterpret_cast<uint4*>(rec + 2 * NW) = make_uint4(uint32_t(c0), uint32_t(c1), __float_as_uint(amax * (1.f / 32767.f)), 0u);
    }
  }
}

// Converts every unit of the jobs: thread i of nthreads (a multiple of 32, warps aligned)
// takes segments i, i + nthreads, ...
__device__ __forceinline__ void quant_jobs(const QuantJobs& Q, long long i0, long long nthreads) {
  for (int jn = 0; jn < Q.n; ++jn) {
    const QuantJob& J = Q.j[jn];
    const int G = unit_weights(J.kind) / 8;
    const long long total = (long long)J.rows * (J.cols / unit_weights(J.kind)) * G;
    const long long padded = (total + 31) / 32 * 32;
    for (long long i = i0; i < padded; i += nthreads) {
      const bool valid = i < total;
      switch (J.kind) {
        case kQ4Pair: quant_seg<kQ4Pair>(J, i, valid); break;
        case kQ4One: quant_seg<kQ4One>(J, i, valid); break;
        case kQ8Pair: quant_seg<kQ8Pair>(J, i, valid); break;
        case kQ8One: quant_seg<kQ8One>(J, i, valid); break;
        case kI4x64: quant_seg<kI4x64>(J, i, valid); break;
        case kI2x64: quant_seg<kI2x64>(J, i, valid); break;
        default: quant_seg<kI4x32>(J, i, valid); break;
      }
    }
  }
}

__global__ void __launch_bounds__(256) k_moe_quant(const __grid_constant__ QuantJobs Q) {
  griddep_launch_dependents();
  griddep_wait();
  quant_jobs(Q, (long long)blockIdx.x * blockDim.x + threadIdx.x, (long long)gridDim.x * blockDim.x);
}

// ---------------------------------------------------------------- 1. route grouping
constexpr int kRouteThreads = 512;

struct RouteWs {
  int32_t* counts;    // [E]
  int32_t* offsets;   // [E + 1]
  int32_t* active;    // [E] touched experts in increasing id order
  int32_t* n_active;  // [1]
  int32_t* perm;      // [T * k] pair ids (t * k + j) grouped by expert, token order inside
  uint32_t* ctr;      // [2] work item counters of the two grouped GEMV launches
  int4* act_info;     // [E] per touched expert (in active order): (expert, count, offset, first pair)
  int skip_negative;  // 1: negative ids mark pairs left out of this call (skipped, not an error)
};

__device__ __forceinline__ void moe_route(const int32_t* __restrict__ idx, int pairs, int n_experts,
                                          const RouteWs& ws) {
  __shared__ int cnt[BQG_MAX_EXPERTS];
  __shared__ int base[BQG_MAX_EXPERTS];
  __shared__ int wcnt[kRouteThreads / 32][BQG_MAX_EXPERTS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < 2) ws.ctr[tid] = 0u;
  for (int e = tid; e < n_experts; e += kRouteThreads) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int p = tid; p < pairs; p += kRouteThreads) {
    const int e = idx[p];
    if (e >= 0 && e < n_experts) atomicAdd(&cnt[e], 1);
    else if (!(ws.skip_negative && e < 0)) bad = true;
  }
  if (bad) flag_error(BQG_DEVERR_EXPERT_ID);
  __syncthreads();
  if (warp == 0) {
    // exclusive scan of the counts and the list of touched experts: lane l owns experts
    // 8l .. 8l+7 (n_experts <= 256)
    int c[8], tot = 0, nact = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = 8 * lane + i;
      c[i] = e < n_experts ? cnt[e] : 0;
      tot += c[i];
      nact += c[i] > 0 ? 1 : 0;
    }
    int incl = tot, ainc = nact;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      const int a = __shfl_up_sync(0xffffffffu, ainc, o);
      if (lane >= o) {
        incl += v;
        ainc += a;
      }
    }
    int off = incl - tot, na = ainc - nact;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = 8 * lane + i;
      if (e < n_experts) {
        ws.counts[e] = c[i];
        ws.offsets[e] = off;
        base[e] = off;
        if (c[i] > 0) ws.active[na++] = e;
      }
      off += c[i];
    }
    if (lane == 31) {
      ws.offsets[n_experts] = incl;
      ws.n_active[0] = ainc;
    }
  }
  __syncthreads();
  // stable placement, one chunk of kRouteThreads pairs at a time
  for (int c0 = 0; c0 < pairs; c0 += kRouteThreads) {
    for (int i = tid; i < (kRouteThreads / 32) * n_experts; i += kRouteThreads) (&wcnt[0][0])[i / n_experts * BQG_MAX_EXPERTS + i % n_experts] = 0;
    __syncthreads();
    const int p = c0 + tid;
    const int e = p < pairs ? idx[p] : -1;
    const bool ok = e >= 0 && e < n_experts;
    const unsigned okmask = __ballot_sync(0xffffffffu, ok);
    unsigned same = 0;
    int rank = 0;
    if (ok) {
      same = __match_any_sync(okmask, e);
      rank = __popc(same & ((1u << lane) - 1u));
      if (rank == 0) wcnt[warp][e] = __popc(same);
    }
    __syncthreads();
    if (ok) {
      int pos = base[e] + rank;
      for (int w = 0; w < warp; ++w) pos += wcnt[w][e];
      ws.perm[pos] = p;
    }
    __syncthreads();
    for (int e2 = tid; e2 < n_experts; e2 += kRouteThreads) {
      int s = 0;
      for (int w = 0; w < kRouteThreads / 32; ++w) s += wcnt[w][e2];
      base[e2] += s;
    }
    __syncthreads();
  }
  // one record per touched expert, so a work item needs a single load to find its tokens
  const int na = ws.n_active[0];
  for (int a = tid; a < na; a += kRouteThreads) {
    const int e = ws.active[a];
    const int off = ws.offsets[e];
    ws.act_info[a] = make_int4(e, ws.counts[e], off, ws.perm[off]);
  }
}

// Block 0 groups the routes; the other blocks convert x (jobs in Q).
__global__ void __launch_bounds__(kRouteThreads, 1) k_moe_prep(const int32_t* __restrict__ idx, int pairs,
                                                            int n_experts, RouteWs ws,
                                                            const __grid_constant__ QuantJobs Q) {
  griddep_launch_dependents();
  griddep_wait();
  if (blockIdx.x == 0) {
    moe_route(idx, pairs, n_experts, ws);
  } else {
    quant_jobs(Q, (long long)(blockIdx.x - 1) * blockDim.x + threadIdx.x, (long long)(gridDim.x - 1) * blockDim.x);
  }
}

// ---------------------------------------------------------------- 2/4. grouped GEMV
// The same producer/consumer structure, stage ring and integer dot products as k_qgemv; a
// work item is one stage of rows of one matrix, applied to all the tokens routed to it.
struct MgMat {            // one family of stacked matrices (gate, up or down of all experts)
  const uint8_t* base;    // expert e's matrix at base + e * stride (stride 0: the shared expert)
  long long stride;
  int rows, cols;         // of one expert's matrix
  int kind, row_bytes, units, scale_off;
  int stage_rows, nstages;
};

struct MgPhase {
  MgMat m[4];             // 0, 1: routed families; 2, 3: shared families
  int nmat;               // routed families (1 or 2; they share one shape)
  int s_nmat;             // shared families (0, 1 or 2; they share one shape)
  const uint4* xq;        // routed input records [input rows][units of m[0]]
  const uint4* s_xq;      // shared input records [tokens][units of m[2]]
  float* out[4];          // per family: routed [pairs][rows], shared [tokens][rows]
  int x_by_token;         // routed input row = pair / top_k (gate/up) or the pair (down)
  int top_k, tokens;
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* n_active;
  const int32_t* perm;
  const int4* act_info;   // per touched expert: (expert, count, offset, first pair)
  uint32_t* ctr;          // work item counter (zeroed by k_moe_prep)
};

__device__ __forceinline__ int4 ld_desc(const int4* d) {
  int4 v;
  asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(d))
               : "memory");
  return v;
}

constexpr int kMgStages = 3;  // no x staging buffer here: room for a third 72 KB stage
// The 15 consumer warps form two teams of 7 that take alternate items of the ring (the 15th
// warp idles): two items are in progress per SM, so one team's x loads, barrier and
// descriptor waits overlap the other team's dot products.
constexpr int kMgTeams = 2;
constexpr int kMgTeamWarps = 7;
constexpr int kMgMaxUnits = 32 * kMgTeamWarps;  // units per row a team can cover
__host__ __device__ constexpr int mg_groups(int units) { return kMgTeamWarps / gemv_group_warps(units); }
// Rows per stage: as many whole rows as fit 72 KB, a multiple of the team's row groups, and
// (when a group spans several warps) at most 32 rows per group (one reducing lane per row).
__host__ __device__ constexpr int mg_stage_rows(int units, int row_bytes) {
  return ((gemv_group_warps(units) > 1 && kGemvStageBytes / row_bytes > 32 * mg_groups(units))
              ? 32 * mg_groups(units)
              : kGemvStageBytes / row_bytes) /
         mg_groups(units) * mg_groups(units);
}
constexpr size_t kMgSmemBytes = size_t(kMgStages) * kGemvStageAlloc +
                                size_t(2 * kGemvConsumerWarps * kGemvRedRows) * sizeof(float) +
                                (3 * kMgStages) * sizeof(uint64_t) + size_t(2 * kMgStages) * sizeof(int4);
static_assert(kMgSmemBytes <= 227 * 1024, "grouped GEMV shared memory");
static_assert((size_t(kMgStages) * kGemvStageAlloc + size_t(2 * kGemvConsumerWarps * kGemvRedRows) * 4) % 16 == 0,
              "descriptors must be 16-byte aligned");

// Consumer side of one item (stage `slot` holds rows [r0, r1) of family fam, expert e).
// q counts token iterations (selects the group reduction buffer).
// The weight stage may still be in flight on entry: the first token's x is loaded before
// waiting for it (full, parity).  Returns false if that wait gave up.
// With `reuse` (a single token whose input record the team's previous item also used), X
// already holds it.
template <int KIND>
__device__ __forceinline__ bool mg_item(const MgPhase& P, const MgMat& M, int4 d, int4 dt, uint32_t stage_s,
                                        float* red, int& q, uint64_t* full, uint32_t parity, XUnit& X, bool reuse,
                                        int team) {
  const int fam = d.x, e = d.y, r0 = d.z, r1 = d.w;
  const bool shared = fam >= 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tw = warp - team * kMgTeamWarps;  // warp within the team
  const int units = M.units, row_bytes = M.row_bytes;
  const int gw = gemv_group_warps(units);
  const int groups = mg_groups(units);
  const int g = tw / gw, j = tw - g * gw;
  const int p = 32 * j + lane;
  const bool in_group = g < groups;
  const bool active = in_group && p < units;
  constexpr int UB = unit_bytes(KIND);
  const uint8_t* wbase = M.base + (shared ? 0 : size_t(e) * M.stride);
  const uint32_t src_lo = uint32_t(reinterpret_cast<uintptr_t>(wbase) + size_t(r0) * row_bytes) & 15u;
  const uint32_t base = stage_s + src_lo + uint32_t(p) * UB;
  const float* scales = reinterpret_cast<const float*>(wbase + M.scale_off);
  const int nrows = r1 - r0;
  const int ntok = dt.x;                   // tokens of this expert (all tokens: shared)
  const int32_t* list = P.perm + dt.y;     // their pairs, in token order
  const uint4* xq = shared ? P.s_xq : P.xq;
  float* out = P.out[fam];
  // int4 row scales: lane l of a group holds the scale of the group's l-th row of the stage
  float sc = 1.f;
  if constexpr (is_i4(KIND)) {
    const int rr = g + lane * groups;
    if (in_group && rr < nrows) sc = __ldg(scales + r0 + rr);
  }
  int pid = shared ? 0 : dt.z;
  for (int tt = 0; tt < ntok; ++tt, ++q) {
    int next_pid = tt + 1;  // prefetched for the next token
    if (!shared && tt + 1 < ntok) next_pid = __ldg(list + tt + 1);
    const int xrow = (shared || !P.x_by_token) ? pid : pid / P.top_k;
    if (active && !(reuse && ntok == 1)) load_xunit<KIND>(xq + (size_t(xrow) * units + p) * xrec_chunks(KIND), X);
    if (tt == 0 && !mbar_wait(full, parity)) return false;
    float* orow = out + size_t(pid) * M.rows + r0;
    const int par = q & 1;
    int nmine = 0;
    if (in_group) {
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
        for (int o = 16; o > 0; o >>= 1) {
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
          v[1] += __shfl_xor_sync(0xffffffffu, v[1], o);
        }
        float s0 = 1.f, s1 = 1.f;
        if constexpr (is_i4(KIND)) {
          if (gw == 1) {  // rows i and i + groups are the group's rows (i - g) / groups and + 1
            const int n0 = (i - g) / groups;
            s0 = __shfl_sync(0xffffffffu, sc, n0 & 31);
            s1 = __shfl_sync(0xffffffffu, sc, (n0 + 1) & 31);
            if (n0 >= 32) s0 = __ldg(scales + r0 + i);
            if (n0 + 1 >= 32) s1 = __ldg(scales + r0 + i + groups);
          }
        }
        if (lane == 0) {
          if (gw == 1) {
            orow[i] = v[0] * s0;
            if (two) orow[i + groups] = v[1] * s1;
          } else {
            red[(par * kGemvConsumerWarps + warp) * kGemvRedRows + nmine] = v[0];
            if (two) red[(par * kGemvConsumerWarps + warp) * kGemvRedRows + nmine + 1] = v[1];
          }
        }
        nmine += two ? 2 : 1;
      }
    }
    if (gw > 1 && in_group) {
      named_bar_sync(3 + 3 * team + g, 32 * gw);  // gw > 1: at most 3 groups per team
      if (j == 0 && lane < nmine) {
        float v = 0.f;
        for (int jj = 0; jj < gw; ++jj)
          v += red[(par * kGemvConsumerWarps + team * kMgTeamWarps + g * gw + jj) * kGemvRedRows + lane];
        const int i = g + lane * groups;
        orow[i] = v * sc;  // lane l writes the group's l-th row (its scale prefetched above)
      }
    }
    pid = next_pid;
  }
  if (ntok == 0) return mbar_wait(full, parity);
  return true;
}

// KR: unit kind of the routed families, KS: of the shared ones (one kernel per pair keeps each
// consumer path within the register budget).
template <int KR, int KS>
__global__ void __launch_bounds__(kGemvThreads, 1) k_moe_gemv(const __grid_constant__ MgPhase P) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(smem + size_t(kMgStages) * kGemvStageAlloc);
  // per slot: (family, expert, r0, r1), (tokens, offset in perm, first pair, 0)
  int4* desc = reinterpret_cast<int4*>(red + 2 * kGemvConsumerWarps * kGemvRedRows);
  __shared__ MgMat fams[4];  // the phase's matrix families, indexed per item from shared memory
  uint64_t* full = reinterpret_cast<uint64_t*>(desc + 2 * kMgStages);
  uint64_t* empty = full + kMgStages;
  uint64_t* dready = empty + kMgStages;  // the slot's descriptor is written (stage may be in flight)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMgStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kMgTeamWarps);  // the team that takes the slot's item
      mbar_init(&dready[i], 1);
    }
    for (int i = 0; i < 4; ++i) fams[i] = P.m[i];
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();
  griddep_wait();  // route lists, counters and input records come from earlier kernels

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------ producer (one elected lane)
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    const int na = *P.n_active;
    const int n_sh = P.s_nmat * fams[2].nstages;
    const int per_expert = P.nmat * fams[0].nstages;
    const int n_items = n_sh + na * per_expert;
    int s = 0;
    bool ok = true;
    // With one token every item costs about the same: items are claimed in runs (guided:
    // about 1/(2 * grid) of what is left, at least one), so a CTA mostly stays on one matrix
    // and keeps its x in registers.  With several tokens item costs differ (an expert's token
    // count, the shared expert's all tokens): one item per claim balances them.
    const int grid = int(gridDim.x);
    int est = 0;  // this CTA's estimate of the counter (end of its last claim)
    auto claim = [&](int& first) -> int {
      int want = (n_items - est) / (2 * grid);
      if (want < 1 || P.tokens > 1) want = 1;
      first = int(atomicAdd(P.ctr, unsigned(want)));
      est = first + want;
      return first >= n_items ? 0 : min(want, n_items - first);
    };
    int first = 0, nfirst = 0;
    int cnt = claim(first);
    int ncnt = cnt > 0 ? claim(nfirst) : 0;  // the next run, claimed one run ahead
    for (int item = first;; ++item) {
      if (item >= first + cnt) {
        first = nfirst;
        cnt = ncnt;
        if (cnt <= 0) break;
        ncnt = claim(nfirst);
        item = first;
      }
      int fam, e = 0, k;
      int4 tok = make_int4(P.tokens, 0, 0, 0);  // shared expert: all tokens in order
      if (item < n_sh) {
        fam = 2 + item / fams[2].nstages;
        k = item - (fam - 2) * fams[2].nstages;
      } else {
        int r = item - n_sh;
        const int a = r / per_expert;
        r -= a * per_expert;
        fam = r / fams[0].nstages;
        k = r - fam * fams[0].nstages;
        const int4 ai = __ldg(P.act_info + a);
        e = ai.x;
        tok = make_int4(ai.y, ai.z, ai.w, 0);
      }
      const MgMat& M = fams[fam];
      const int r0 = k * M.stage_rows;
      const int r1 = min(r0 + M.stage_rows, M.rows);
      const int slot = s % kMgStages;
      if (s >= kMgStages && !mbar_wait(&empty[slot], uint32_t(s / kMgStages - 1) & 1u)) {
        ok = false;
        break;
      }
      fence_proxy_async_smem();
      desc[2 * slot] = make_int4(fam, e, r0, r1);
      desc[2 * slot + 1] = tok;
      mbar_arrive(&dready[slot]);
      const uintptr_t wbeg = reinterpret_cast<uintptr_t>(M.base) + (fam >= 2 ? 0 : size_t(e) * M.stride);
      const uintptr_t wend = wbeg + size_t(M.rows) * M.row_bytes;
      const uintptr_t src = wbeg + size_t(r0) * M.row_bytes;
      const uintptr_t end = src + size_t(r1 - r0) * M.row_bytes;
      const uintptr_t a0 = src & ~uintptr_t(15);
      const uintptr_t lim = wend & ~uintptr_t(15);
      uintptr_t a1 = (end + 15) & ~uintptr_t(15);
      if (a1 > lim) a1 = lim;
      if (a1 < a0) a1 = a0;
      uint8_t* dst = ring + size_t(slot) * kGemvStageAlloc;
      for (uintptr_t b = (a1 > src ? a1 : src); b < end; ++b) dst[b - a0] = *reinterpret_cast<const uint8_t*>(b);
      const uint32_t nb = uint32_t(a1 - a0);
      if (nb > 0) {
        mbar_arrive_expect_tx(&full[slot], nb);
        bulk_g2s(dst, reinterpret_cast<const void*>(a0), nb, &full[slot], pol);
      } else {
        mbar_arrive(&full[slot]);
      }
      ++s;
    }
    // end markers, one for each team (the next item of each team)
    for (int t = 0; t < kMgTeams && ok; ++t, ++s) {
      const int slot = s % kMgStages;
      if (s >= kMgStages && !mbar_wait(&empty[slot], uint32_t(s / kMgStages - 1) & 1u)) {
        ok = false;
        break;
      }
      desc[2 * slot] = make_int4(-1, 0, 0, 0);
      mbar_arrive(&dready[slot]);
    }
    if (!ok) {
      for (int qq = (s > kMgStages ? s - kMgStages : 0); qq < s; ++qq)
        mbar_wait(&full[qq % kMgStages], uint32_t(qq / kMgStages) & 1u);
    }
    return;
  }

  // ------------------------------------------------ consumers
  const int team = warp / kMgTeamWarps;
  if (team >= kMgTeams) return;  // the odd warp out
  const uint32_t ring_s = smem_u32(ring);
  int q = 0;
  int prev_units = -1, prev_routed = -1;  // row shape of the team's previous item
  int prev_x = -1;                        // input record held in X (one-token items), else -1
  XUnit X;
  for (int s = team;; s += kMgTeams) {
    const int slot = s % kMgStages;
    const uint32_t par = uint32_t(s / kMgStages) & 1u;
    if (!mbar_wait(&dready[slot], par)) return;
    const int4 d = ld_desc(&desc[2 * slot]);
    if (d.x < 0) return;
    const int4 dt = ld_desc(&desc[2 * slot + 1]);
    // Another row shape (units per row or unit kind): row groups may change, so every consumer
    // warp of the team must have finished the previous item, including its group reductions.
    // Items of the same shape (another stage, gate after up, another expert) keep the groups,
    // and each group's own barrier orders its reduction buffers.
    const int routed = d.x < 2 ? 1 : 0;
    const int units = fams[d.x].units;
    if (units != prev_units || routed != prev_routed) named_bar_sync(1 + team, 32 * kMgTeamWarps);
    prev_units = units;
    prev_routed = routed;
    // One token: X may already hold its input record (the same token for every routed gate/up
    // item, the same pair for every stage of one expert's down matrix).
    int xkey = -1;
    if (dt.x == 1) {
      const int pid = routed ? dt.z : 0;
      xkey = 2 * ((routed && P.x_by_token) ? pid / P.top_k : pid) + routed;
    }
    const bool reuse = xkey >= 0 && xkey == prev_x;
    prev_x = xkey;
    const uint32_t stage_s = ring_s + uint32_t(slot) * kGemvStageAlloc;
    const bool ok = routed ? mg_item<KR>(P, fams[d.x], d, dt, stage_s, red, q, &full[slot], par, X, reuse, team)
                           : mg_item<KS>(P, fams[d.x], d, dt, stage_s, red, q, &full[slot], par, X, reuse, team);
    if (!ok) return;
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// ---------------------------------------------------------------- 4. combine
// y[t, c] = sum_{j<k} w[t, j] * part[t*k + j, c] in slot order (pairs with an invalid expert id
// contribute nothing), plus the shared output; with `accumulate`, added to y instead of stored.
__global__ void k_moe_combine(const float* __restrict__ part, const int32_t* __restrict__ idx,
                              const float* __restrict__ w, const float* __restrict__ sout, float* __restrict__ y,
                              int tokens, int top_k, int hidden, int n_experts, int accumulate) {
  griddep_wait();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)tokens * hidden) return;
  const int t = int(i / hidden), c = int(i - (long long)t * hidden);
  // all loads first (top_k <= BQG_MAX_TOPK), then the slot-order sum
  float wv[BQG_MAX_TOPK], pv[BQG_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < BQG_MAX_TOPK; ++j) {
    wv[j] = 0.f;
    pv[j] = 0.f;
    if (j < top_k) {
      const int e = __ldg(idx + t * top_k + j);
      if (e >= 0 && e < n_experts) {
        wv[j] = __ldg(w + t * top_k + j);
        pv[j] = part[(size_t(t) * top_k + j) * hidden + c];
      }
    }
  }
  const float s = sout != nullptr ? sout[size_t(t) * hidden + c] : 0.f;
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < BQG_MAX_TOPK; ++j)
    if (j < top_k) acc = fmaf(wv[j], pv[j], acc);
  y[i] = accumulate ? y[i] + (acc + s) : acc + s;
}

}  // namespace bqg
