// Routed Mixture-of-Experts layer on block-quantized experts:
//   y_t = sum_{j<k} w_tj * D_e (act(G_e x_t) * (U_e x_t))  +  shared FFN(x_t),   e = idx[t, j]
//
// Sources: Camelid README, "Gemma 4" (GeGLU experts; dense shared expert + sparse top-8
// branch of the 128-expert MoE); TurboFieldfare wiki, "메모리·전문가 스트리밍" (routed experts
// split from the shared branch; an expert read serves every row routed to it); colibri wiki
// summary, "핵심 아이디어" and "구현 범위" (256 routed int4 experts with per-row scales).
//
// Steps (all on the caller's stream):
//   1. k_moe_route    one CTA: per-expert counts, offsets, the list of touched experts and a
//                     stable permutation of the (token, slot) pairs grouped by expert, in token
//                     order.  Expert ids outside [0, E) are skipped and flagged.
//   2. k_moe_grouped  (phase gate/up) every touched expert's gate and up rows are streamed once
//                     (bulk copies into shared memory, next tile prefetched) and applied to all
//                     of its tokens; h = act(g) * u is written per pair.  The shared expert is
//                     one more work list over all tokens.
//   3. k_moe_grouped  (phase down) the same over the down matrices, x = h of each pair; writes
//                     one output row per pair (and the shared output).
//   4. k_moe_combine  y_t = sum_j w_tj * out_(t,j) in slot order, plus the shared output.
// Every sum has a fixed order, so results are deterministic.
#pragma once

#include "common.cuh"
#include "host_common.h"
#include "qgemv.cuh"

namespace bqg {

// ---------------------------------------------------------------- 1. route grouping
constexpr int kRouteThreads = 1024;

struct RouteWs {
  int32_t* counts;   // [E]
  int32_t* offsets;  // [E + 1]
  int32_t* active;   // [E] touched experts in increasing id order
  int32_t* n_active; // [1]
  int32_t* perm;     // [T * k] pair ids (t * k + j) grouped by expert, token order inside
};

__global__ void __launch_bounds__(kRouteThreads) k_moe_route(const int32_t* __restrict__ idx, int pairs,
                                                             int n_experts, RouteWs ws) {
  __shared__ int cnt[BQG_MAX_EXPERTS];
  __shared__ int base[BQG_MAX_EXPERTS];
  __shared__ int wcnt[kRouteThreads / 32][BQG_MAX_EXPERTS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < n_experts; e += kRouteThreads) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int p = tid; p < pairs; p += kRouteThreads) {
    const int e = idx[p];
    if (e >= 0 && e < n_experts) atomicAdd(&cnt[e], 1);
    else bad = true;
  }
  if (bad) flag_error(BQG_DEVERR_EXPERT_ID);
  __syncthreads();
  if (tid == 0) {
    int off = 0, na = 0;
    for (int e = 0; e < n_experts; ++e) {
      ws.counts[e] = cnt[e];
      ws.offsets[e] = off;
      base[e] = off;
      if (cnt[e] > 0) ws.active[na++] = e;
      off += cnt[e];
    }
    ws.offsets[n_experts] = off;
    ws.n_active[0] = na;
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
}

// ---------------------------------------------------------------- 2/3. grouped expert GEMM
constexpr int kMoeThreads = 256;                 // 8 warps
constexpr int kMoeSlotBytes = 72 * 1024;         // weight tile buffer (x2: current + prefetch)
constexpr int kMoeXBytes = 64 * 1024;            // token tile of activations
constexpr int kMoeMaxTok = 8;                    // tokens per token tile
constexpr int kMoeMaxVRows = 32;                 // rows per tile (both matrices together)
constexpr size_t kMoeSmemBytes = 2 * size_t(kMoeSlotBytes + 64) + kMoeXBytes +
                                 size_t(2 * kMoeMaxTok * kMoeMaxVRows) * sizeof(float) + 64;

struct MoeMat {          // one family of stacked matrices (gate, up or down of all experts)
  const uint8_t* base;   // expert e's matrix at base + e * stride
  long long stride;
  int rows, cols;        // of one expert's matrix
  int kind, row_bytes, units, scale_off;
};

struct MoePhase {
  // routed experts
  MoeMat m0, m1;         // gate/up phase: m0 = gate, m1 = up; down phase: m0 = down
  int nmat;              // 2 (gate/up) or 1 (down)
  int lpr;               // lanes per row: 8, 16 or 32
  int tile_rows;         // rows of one matrix per tile
  int tiles;             // tiles per expert
  int tb;                // tokens per token tile
  // shared expert (optional)
  MoeMat s0, s1;
  int s_present;
  int s_lpr, s_tile_rows, s_tiles, s_tb;
  // activations
  const float* xin;      // gate/up: x [T x hidden]; down: h [pairs x inter]
  const float* s_xin;    // down: shared h [T x shared_inter]
  float* out;            // gate/up: h [pairs x inter]; down: per-pair output [pairs x hidden]
  float* s_out;          // gate/up: shared h; down: shared output [T x hidden]
  int xin_stride, s_xin_stride, out_stride, s_out_stride;
  int gateup;            // 1: gate/up phase (epilogue act(g) * u), 0: down phase
  int act;
  int tokens, top_k;
  RouteWs route;
};

__device__ __forceinline__ float act_fn(int act, float g) {
  if (act == BQG_ACT_SILU) return g / (1.f + expf(-g));
  const float c = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * g * (1.f + tanhf(c * (g + 0.044715f * g * g * g)));
}

// Decodes one unit into exact fp32 weight values (without the I4 row scale).
template <int KIND>
__device__ __forceinline__ void unit_decode(const uint8_t* u, float (&w)[64]) {
  if constexpr (KIND == kQ4Pair || KIND == kQ4One) {
    uint32_t v[9];
    uint32_t q[8];
    float dA, dB = 0.f;
    if constexpr (KIND == kQ4Pair) {
      const uint32_t* p = reinterpret_cast<const uint32_t*>(u);
#pragma unroll
      for (int i = 0; i < 9; ++i) v[i] = p[i];
#pragma unroll
      for (int k = 0; k < 4; ++k) q[k] = __funnelshift_r(v[k], v[k + 1], 16);
#pragma unroll
      for (int k = 0; k < 4; ++k) q[4 + k] = v[5 + k];
      dA = half_bits_to_float(v[0]);
      dB = half_bits_to_float(v[4] >> 16);
    } else {
      const uintptr_t a = reinterpret_cast<uintptr_t>(u);
      const uint32_t* p = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
      const uint32_t sh = uint32_t(a & 2) * 8;
#pragma unroll
      for (int i = 0; i < 5; ++i) v[i] = p[i];
#pragma unroll
      for (int k = 0; k < 4; ++k) q[k] = __funnelshift_rc(v[k], v[k + 1], 16 + sh);
      dA = half_bits_to_float(__funnelshift_r(v[0], v[1], sh));
    }
    constexpr int NW = (KIND == kQ4Pair) ? 8 : 4;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const float d = k < 4 ? dA : dB;
      const float c = -136.f * d;
      const uint32_t lo = q[k] & 0x0F0F0F0Fu, hi = (q[k] >> 4) & 0x0F0F0F0Fu;
      // (128 + q) * d - 136 d = (q - 8) * d, exact in fp32
      w[8 * k + 0] = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4055u)), d, c);
      w[8 * k + 1] = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4055u)), d, c);
      w[8 * k + 2] = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4155u)), d, c);
      w[8 * k + 3] = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4155u)), d, c);
      w[8 * k + 4] = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4255u)), d, c);
      w[8 * k + 5] = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4255u)), d, c);
      w[8 * k + 6] = fmaf(__uint_as_float(__byte_perm(lo, 0x43u, 0x4355u)), d, c);
      w[8 * k + 7] = fmaf(__uint_as_float(__byte_perm(hi, 0x43u, 0x4355u)), d, c);
    }
  } else if constexpr (KIND == kQ8Pair || KIND == kQ8One) {
    uint32_t v[17];
    uint32_t q[16];
    float dA, dB = 0.f;
    if constexpr (KIND == kQ8Pair) {
      const uint32_t* p = reinterpret_cast<const uint32_t*>(u);
#pragma unroll
      for (int i = 0; i < 17; ++i) v[i] = p[i];
#pragma unroll
      for (int k = 0; k < 8; ++k) q[k] = __funnelshift_r(v[k], v[k + 1], 16);
#pragma unroll
      for (int k = 0; k < 8; ++k) q[8 + k] = v[9 + k];
      dA = half_bits_to_float(v[0]);
      dB = half_bits_to_float(v[8] >> 16);
    } else {
      const uintptr_t a = reinterpret_cast<uintptr_t>(u);
      const uint32_t* p = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
      const uint32_t sh = uint32_t(a & 2) * 8;
#pragma unroll
      for (int i = 0; i < 9; ++i) v[i] = p[i];
#pragma unroll
      for (int k = 0; k < 8; ++k) q[k] = __funnelshift_rc(v[k], v[k + 1], 16 + sh);
      dA = half_bits_to_float(__funnelshift_r(v[0], v[1], sh));
    }
    constexpr int NW = (KIND == kQ8Pair) ? 16 : 8;
    const float off = 8388736.0f;  // 2^23 + 128
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const float d = k < 8 ? dA : dB;
      const uint32_t s = q[k] ^ 0x80808080u;
      w[4 * k + 0] = (__uint_as_float(__byte_perm(s, 0x4Bu, 0x4550u)) - off) * d;
      w[4 * k + 1] = (__uint_as_float(__byte_perm(s, 0x4Bu, 0x4551u)) - off) * d;
      w[4 * k + 2] = (__uint_as_float(__byte_perm(s, 0x4Bu, 0x4552u)) - off) * d;
      w[4 * k + 3] = (__uint_as_float(__byte_perm(s, 0x4Bu, 0x4553u)) - off) * d;
    }
  } else {  // int4 with per-row scale (applied after the dot product)
    constexpr int NW = (KIND == kI4x64) ? 8 : 4;
    const uint4* p = reinterpret_cast<const uint4*>(u);
    uint32_t q[8];
    const uint4 a = p[0];
    q[0] = a.x; q[1] = a.y; q[2] = a.z; q[3] = a.w;
    if constexpr (NW == 8) {
      const uint4 b = p[1];
      q[4] = b.x; q[5] = b.y; q[6] = b.z; q[7] = b.w;
    }
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const uint32_t lo = (q[k] ^ 0x08080808u) & 0x0F0F0F0Fu, hi = ((q[k] >> 4) ^ 0x08080808u) & 0x0F0F0F0Fu;
      w[8 * k + 0] = __uint_as_float(__byte_perm(lo, 0x43u, 0x4055u)) - 136.f;
      w[8 * k + 1] = __uint_as_float(__byte_perm(hi, 0x43u, 0x4055u)) - 136.f;
      w[8 * k + 2] = __uint_as_float(__byte_perm(lo, 0x43u, 0x4155u)) - 136.f;
      w[8 * k + 3] = __uint_as_float(__byte_perm(hi, 0x43u, 0x4155u)) - 136.f;
      w[8 * k + 4] = __uint_as_float(__byte_perm(lo, 0x43u, 0x4255u)) - 136.f;
      w[8 * k + 5] = __uint_as_float(__byte_perm(hi, 0x43u, 0x4255u)) - 136.f;
      w[8 * k + 6] = __uint_as_float(__byte_perm(lo, 0x43u, 0x4355u)) - 136.f;
      w[8 * k + 7] = __uint_as_float(__byte_perm(hi, 0x43u, 0x4355u)) - 136.f;
    }
  }
}

__device__ __forceinline__ void unit_decode_any(int kind, const uint8_t* u, float (&w)[64]) {
  switch (kind) {
    case kQ4Pair: unit_decode<kQ4Pair>(u, w); break;
    case kQ8Pair: unit_decode<kQ8Pair>(u, w); break;
    case kI4x64: unit_decode<kI4x64>(u, w); break;
    case kQ4One: unit_decode<kQ4One>(u, w); break;
    case kQ8One: unit_decode<kQ8One>(u, w); break;
    default: unit_decode<kI4x32>(u, w); break;
  }
}

// Work item -> (which list, expert, tile).  Routed items first, then the shared expert's.
struct MoeItem {
  int shared;   // 0 routed, 1 shared
  int expert;   // routed expert id
  int tile;
  int ntok;     // tokens of this expert
  int tok0;     // offset into perm (routed)
};

__device__ __forceinline__ bool moe_item(const MoePhase& P, int n_active, int item, MoeItem& it) {
  const int routed = n_active * P.tiles;
  if (item < routed) {
    const int a = item / P.tiles;
    it.shared = 0;
    it.expert = P.route.active[a];
    it.tile = item - a * P.tiles;
    it.tok0 = P.route.offsets[it.expert];
    it.ntok = P.route.counts[it.expert];
    return true;
  }
  item -= routed;
  if (P.s_present && item < P.s_tiles) {
    it.shared = 1;
    it.expert = 0;
    it.tile = item;
    it.tok0 = 0;
    it.ntok = P.tokens;
    return true;
  }
  return false;
}

struct TileGeom {
  const MoeMat* m[2];
  int nmat, lpr, tile_rows, tb, r0, r1;
};

__device__ __forceinline__ TileGeom tile_geom(const MoePhase& P, const MoeItem& it) {
  TileGeom g;
  if (!it.shared) {
    g.m[0] = &P.m0; g.m[1] = &P.m1; g.nmat = P.nmat; g.lpr = P.lpr; g.tile_rows = P.tile_rows; g.tb = P.tb;
  } else {
    g.m[0] = &P.s0; g.m[1] = &P.s1; g.nmat = P.nmat; g.lpr = P.s_lpr; g.tile_rows = P.s_tile_rows; g.tb = P.s_tb;
  }
  g.r0 = it.tile * g.tile_rows;
  g.r1 = min(g.r0 + g.tile_rows, g.m[0]->rows);
  return g;
}

// Byte offset of matrix m's rows inside a slot (16-byte aligned sub-buffers).
__device__ __forceinline__ int slot_sub_offset(const TileGeom& g, int m) {
  return m == 0 ? 0 : ((g.tile_rows * g.m[0]->row_bytes + 47) / 16) * 16;
}

// Producer side: issue the bulk copies of one item's weight tile into `slot` (thread 0).
__device__ __forceinline__ void issue_tile(const MoeItem& it, const TileGeom& g, uint8_t* slot, uint64_t* bar,
                                           uint64_t pol) {
  uint32_t total = 0;
  for (int m = 0; m < g.nmat; ++m) {
    const MoeMat& M = *g.m[m];
    const uintptr_t wbeg = reinterpret_cast<uintptr_t>(M.base) + (it.shared ? 0 : size_t(it.expert) * M.stride);
    const uintptr_t wend = wbeg + size_t(M.rows) * M.row_bytes;
    const uintptr_t src = wbeg + size_t(g.r0) * M.row_bytes;
    const uintptr_t end = src + size_t(g.r1 - g.r0) * M.row_bytes;
    const uintptr_t a0 = src & ~uintptr_t(15);
    const uintptr_t lim = wend & ~uintptr_t(15);
    uintptr_t a1 = (end + 15) & ~uintptr_t(15);
    if (a1 > lim) a1 = lim;
    if (a1 < a0) a1 = a0;
    uint8_t* dst = slot + slot_sub_offset(g, m);
    for (uintptr_t b = (a1 > src ? a1 : src); b < end; ++b) dst[b - a0] = *reinterpret_cast<const uint8_t*>(b);
    total += uint32_t(a1 - a0);
  }
  mbar_arrive_expect_tx(bar, total);
  for (int m = 0; m < g.nmat; ++m) {
    const MoeMat& M = *g.m[m];
    const uintptr_t wbeg = reinterpret_cast<uintptr_t>(M.base) + (it.shared ? 0 : size_t(it.expert) * M.stride);
    const uintptr_t wend = wbeg + size_t(M.rows) * M.row_bytes;
    const uintptr_t src = wbeg + size_t(g.r0) * M.row_bytes;
    const uintptr_t end = src + size_t(g.r1 - g.r0) * M.row_bytes;
    const uintptr_t a0 = src & ~uintptr_t(15);
    const uintptr_t lim = wend & ~uintptr_t(15);
    uintptr_t a1 = (end + 15) & ~uintptr_t(15);
    if (a1 > lim) a1 = lim;
    if (a1 < a0) a1 = a0;
    if (a1 > a0) bulk_g2s(slot + slot_sub_offset(g, m), reinterpret_cast<const void*>(a0), uint32_t(a1 - a0), bar, pol);
  }
}

__global__ void __launch_bounds__(kMoeThreads, 1) k_moe_grouped(const __grid_constant__ MoePhase P) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* slots[2] = {smem, smem + kMoeSlotBytes + 64};
  float* xs = reinterpret_cast<float*>(smem + 2 * size_t(kMoeSlotBytes + 64));
  float* epi = xs + kMoeXBytes / 4;                       // [2][kMoeMaxTok][kMoeMaxVRows]
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + 2 * kMoeMaxTok * kMoeMaxVRows);
  __shared__ int s_tok[kMoeMaxTok];                       // token (or pair) of each tile slot

  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  const int n_active = *P.route.n_active;
  const uint64_t pol = policy_evict_first();

  int item = blockIdx.x;
  MoeItem it;
  bool have = moe_item(P, n_active, item, it);
  if (have && tid == 0) issue_tile(it, tile_geom(P, it), slots[0], &bars[0], pol);
  int phase[2] = {0, 0};
  int cur = 0;
  while (have) {
    const TileGeom g = tile_geom(P, it);
    // prefetch the next item into the other slot (its previous contents were consumed and
    // released by the __syncthreads at the end of the last iteration)
    MoeItem nx;
    const int nitem = item + gridDim.x;
    const bool nhave = moe_item(P, n_active, nitem, nx);
    if (nhave && tid == 0) issue_tile(nx, tile_geom(P, nx), slots[cur ^ 1], &bars[cur ^ 1], pol);

    if (!mbar_wait(&bars[cur], uint32_t(phase[cur]))) return;
    phase[cur] ^= 1;

    // geometry of this tile
    const MoeMat& M0 = *g.m[0];
    const int kind = M0.kind, units = M0.units, ub = unit_bytes(kind), uw = unit_weights(kind);
    const int xstride_u = uw + 4;                 // padded floats per unit in the x tile
    const int rows_per_pass = kMoeThreads / g.lpr;
    const int nrows = g.r1 - g.r0;
    const int vrows = nrows * g.nmat;             // rows of both matrices
    const int my_vr = tid / g.lpr, my_l = tid % g.lpr;
    const int cols = M0.cols;
    const float* xin = it.shared ? P.s_xin : P.xin;
    const int xin_stride = it.shared ? P.s_xin_stride : P.xin_stride;

    for (int j0 = 0; j0 < it.ntok; j0 += g.tb) {
      const int nt = min(g.tb, it.ntok - j0);
      // token ids of this token tile
      if (tid < nt) {
        const int jj = j0 + tid;
        s_tok[tid] = it.shared ? jj : P.route.perm[it.tok0 + jj];
      }
      __syncthreads();
      // stage x rows into the padded tile layout: unit u at u * (uw + 4) floats
      const int c4 = cols / 4;
      for (int i = tid; i < nt * c4; i += kMoeThreads) {
        const int j = i / c4, c = (i - j * c4) * 4;
        const int pid = s_tok[j];
        // gate/up reads x of the token; down reads h of the pair (or of the token if shared)
        const int row = (P.gateup && !it.shared) ? pid / P.top_k : pid;
        const float4 v = *reinterpret_cast<const float4*>(xin + size_t(row) * xin_stride + c);
        const int u = c / uw, o = c - u * uw;
        *reinterpret_cast<float4*>(xs + j * (units * xstride_u) + u * xstride_u + o) = v;
      }
      __syncthreads();

      // dot products: virtual row vr (matrix vr / nrows, row vr % nrows), lanes split units
      for (int vr0 = 0; vr0 < vrows; vr0 += rows_per_pass) {
        const int vr = vr0 + my_vr;
        float acc[kMoeMaxTok];
#pragma unroll
        for (int j = 0; j < kMoeMaxTok; ++j) acc[j] = 0.f;
        if (vr < vrows) {
          const int m = vr / nrows, r = vr - m * nrows;
          const MoeMat& M = *g.m[m];
          const uintptr_t wbeg = reinterpret_cast<uintptr_t>(M.base) + (it.shared ? 0 : size_t(it.expert) * M.stride);
          const uintptr_t src = wbeg + size_t(g.r0) * M.row_bytes;
          const uint8_t* rowp = slots[cur] + slot_sub_offset(g, m) + (src & 15) + size_t(r) * M.row_bytes;
          for (int u = my_l; u < units; u += g.lpr) {
            float w[64];
            unit_decode_any(kind, rowp + size_t(u) * ub, w);
#pragma unroll
            for (int j = 0; j < kMoeMaxTok; ++j) {
              if (j < nt) {
                const float4* xv = reinterpret_cast<const float4*>(xs + j * (units * xstride_u) + u * xstride_u);
                float a = acc[j];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                  if (q < uw / 4) {
                    const float4 x4 = xv[q];
                    a = fmaf(w[4 * q], x4.x, a);
                    a = fmaf(w[4 * q + 1], x4.y, a);
                    a = fmaf(w[4 * q + 2], x4.z, a);
                    a = fmaf(w[4 * q + 3], x4.w, a);
                  }
                }
                acc[j] = a;
              }
            }
          }
        }
        // reduce over the lanes of this row (fixed butterfly inside aligned lane groups)
#pragma unroll
        for (int j = 0; j < kMoeMaxTok; ++j) {
          float a = acc[j];
          for (int o = g.lpr / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          acc[j] = a;
        }
        if (vr < vrows && my_l == 0) {
          const int m = vr / nrows, r = vr - m * nrows;
          const MoeMat& M = *g.m[m];
          float sc = 1.f;
          if (M.kind == kI4x64 || M.kind == kI4x32) {
            const uint8_t* mb = M.base + (it.shared ? 0 : size_t(it.expert) * M.stride);
            sc = __ldg(reinterpret_cast<const float*>(mb + M.scale_off) + g.r0 + r);
          }
#pragma unroll
          for (int j = 0; j < kMoeMaxTok; ++j) {
            if (j >= nt) break;
            const float v = acc[j] * sc;
            if (P.gateup) {
              epi[(m * kMoeMaxTok + j) * kMoeMaxVRows + r] = v;
            } else {
              float* o = it.shared ? P.s_out : P.out;
              const int ostride = it.shared ? P.s_out_stride : P.out_stride;
              o[size_t(s_tok[j]) * ostride + g.r0 + r] = v;
            }
          }
        }
      }
      if (P.gateup) {
        __syncthreads();
        for (int i = tid; i < nt * nrows; i += kMoeThreads) {
          const int j = i / nrows, r = i - j * nrows;
          const float gv = epi[(0 * kMoeMaxTok + j) * kMoeMaxVRows + r];
          const float uv = epi[(1 * kMoeMaxTok + j) * kMoeMaxVRows + r];
          float* o = it.shared ? P.s_out : P.out;
          const int ostride = it.shared ? P.s_out_stride : P.out_stride;
          o[size_t(s_tok[j]) * ostride + g.r0 + r] = act_fn(P.act, gv) * uv;
        }
      }
      __syncthreads();
    }
    item = nitem;
    it = nx;
    have = nhave;
    cur ^= 1;
  }
}

// ---------------------------------------------------------------- 4. combine
// y[t, c] = sum_{j<k} w[t, j] * part[t*k + j, c] in slot order (pairs with an invalid expert id
// contribute nothing), plus the shared output.
__global__ void k_moe_combine(const float* __restrict__ part, const int32_t* __restrict__ idx,
                              const float* __restrict__ w, const float* __restrict__ sout, float* __restrict__ y,
                              int tokens, int top_k, int hidden, int n_experts) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)tokens * hidden) return;
  const int t = int(i / hidden), c = int(i - (long long)t * hidden);
  float acc = 0.f;
  for (int j = 0; j < top_k; ++j) {
    const int e = idx[t * top_k + j];
    if (e >= 0 && e < n_experts) acc = fmaf(w[t * top_k + j], part[(size_t(t) * top_k + j) * hidden + c], acc);
  }
  if (sout != nullptr) acc += sout[size_t(t) * hidden + c];
  y[i] = acc;
}

}  // namespace bqg
