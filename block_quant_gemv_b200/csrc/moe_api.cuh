// Host side of the MoE layer: workspace layout, argument checks, tile planning, launches.
#pragma once

#include "host_common.h"
#include "moe.cuh"
#include "moe_tc.cuh"
#include "qgemv_api.cuh"

namespace bqg {

constexpr int kMoeMaxCols = BQG_MAX_MOE_COLS;  // hidden / inter / shared_inter limit of moe_forward
static_assert(kMoeMaxCols / 32 <= kMgMaxUnits, "one-block units of the widest row must fit a consumer team");

inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Unit kind of a matrix format in the grouped GEMV: one block for Q8_0 and Q4_0 (a row of
// hidden/inter values then fills more lanes than pairs of blocks would: 88 units for 2816
// columns, 22 for 704), 64 values for int4 when the columns allow, else 32.  Rows of up to
// BQG_MAX_MOE_COLS values give at most 224 units, one per lane of a 7-warp consumer team.
inline int moe_kind(int fmt, int cols) {
  if (fmt == BQG_Q8_0) return kQ8One;
  if (fmt == BQG_Q4_0) return kQ4One;
  if (fmt == BQG_I2_ROW) return kI2x64;
  return cols % 64 == 0 ? kI4x64 : kI4x32;
}

// Kernel instance for a (routed kind, shared kind) pair.
using MgKernel = void (*)(MgPhase);
template <int KR>
inline MgKernel mg_kernel_ks(int ks) {
  switch (ks) {
    case kQ4One: return k_moe_gemv<KR, kQ4One>;
    case kQ8One: return k_moe_gemv<KR, kQ8One>;
    case kI4x64: return k_moe_gemv<KR, kI4x64>;
    case kI2x64: return k_moe_gemv<KR, kI2x64>;
    default: return k_moe_gemv<KR, kI4x32>;
  }
}
inline MgKernel mg_kernel(int kr, int ks) {
  switch (kr) {
    case kQ4One: return mg_kernel_ks<kQ4One>(ks);
    case kQ8One: return mg_kernel_ks<kQ8One>(ks);
    case kI4x64: return mg_kernel_ks<kI4x64>(ks);
    case kI2x64: return mg_kernel_ks<kI2x64>(ks);
    default: return mg_kernel_ks<kI4x32>(ks);
  }
}

inline int mg_row_bytes(int fmt, int cols) {
  return fmt == BQG_Q8_0 ? cols / 32 * 34 : fmt == BQG_Q4_0 ? cols / 32 * 18 : fmt == BQG_I2_ROW ? cols / 4 : cols / 2;
}

// One family of stacked matrices [rows x cols] (expert e at base + e * stride).
inline MgMat mg_mat(int fmt, const void* base, size_t stride, int rows, int cols) {
  MgMat M{};
  M.base = static_cast<const uint8_t*>(base);
  M.stride = (long long)stride;
  M.rows = rows;
  M.cols = cols;
  M.kind = moe_kind(fmt, cols);
  M.row_bytes = mg_row_bytes(fmt, cols);
  M.units = cols / unit_weights(M.kind);
  M.scale_off = (fmt == BQG_I4_ROW || fmt == BQG_I2_ROW) ? int((size_t(rows) * M.row_bytes + 15) / 16 * 16) : 0;
  M.stage_rows = mg_stage_rows(M.units, M.row_bytes);
  M.nstages = (rows + M.stage_rows - 1) / M.stage_rows;
  return M;
}

inline size_t xrec_bytes(int fmt, int rows, int cols) {
  const int kind = moe_kind(fmt, cols);
  return size_t(rows) * (cols / unit_weights(kind)) * xrec_chunks(kind) * 16;
}

struct MoeWsLayout {
  size_t counts, offsets, active, n_active, ctr, act_info, perm;
  size_t xq, s_xq, g, u, gs, us, hq, hsq, part, sout, total;
};

inline MoeWsLayout moe_ws_layout(const bqg_moe_layer* L, int tokens) {
  MoeWsLayout o{};
  const size_t E = size_t(L->n_experts), T = size_t(tokens), pairs = T * L->top_k;
  const bool sh = L->s_gate != nullptr;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  o.counts = take(4 * E);
  o.offsets = take(4 * (E + 1));
  o.active = take(4 * E);
  o.n_active = take(4);
  o.ctr = take(8);
  o.act_info = take(16 * E);
  o.perm = take(4 * pairs);
  o.xq = take(xrec_bytes(L->expert_fmt, tokens, L->hidden));
  o.s_xq = sh ? take(xrec_bytes(L->shared_fmt, tokens, L->hidden)) : 0;
  o.g = take(4 * pairs * L->inter);
  o.u = take(4 * pairs * L->inter);
  o.gs = sh ? take(4 * T * L->shared_inter) : 0;
  o.us = sh ? take(4 * T * L->shared_inter) : 0;
  o.hq = take(xrec_bytes(L->expert_fmt, int(pairs), L->inter));
  o.hsq = sh ? take(xrec_bytes(L->shared_fmt, tokens, L->shared_inter)) : 0;
  o.part = take(4 * pairs * L->hidden);
  o.sout = sh ? take(4 * T * L->hidden) : 0;
  o.total = off;
  return o;
}

// The families of a layer on the tensor-core path; false when a shape does not fit it.
// i8: the kind::i8 variant (every family int4 or int2 with k a multiple of 128).
struct TcLayer {
  TcFam gate, up, down0, down1, s_gate, s_up, s_down0, s_down1;
};

inline bool tc_layer(const bqg_moe_layer* L, TcLayer* T, bool i8) {
  TcLayer t{};
  if (!tc_fam(L->expert_fmt, L->gate, L->gate_stride, L->inter, L->hidden, 0, &t.gate, i8) ||
      !tc_fam(L->expert_fmt, L->up, L->up_stride, L->inter, L->hidden, 0, &t.up, i8) ||
      !tc_fam(L->expert_fmt, L->down, L->down_stride, L->hidden, L->inter, 0, &t.down0, i8) ||
      !tc_fam(L->expert_fmt, L->down, L->down_stride, L->hidden, L->inter, 128, &t.down1, i8))
    return false;
  if (L->s_gate != nullptr) {
    if (!tc_fam(L->shared_fmt, L->s_gate, 0, L->shared_inter, L->hidden, 0, &t.s_gate, i8) ||
        !tc_fam(L->shared_fmt, L->s_up, 0, L->shared_inter, L->hidden, 0, &t.s_up, i8) ||
        !tc_fam(L->shared_fmt, L->s_down, 0, L->hidden, L->shared_inter, 0, &t.s_down0, i8) ||
        !tc_fam(L->shared_fmt, L->s_down, 0, L->hidden, L->shared_inter, 128, &t.s_down1, i8))
      return false;
  }
  if (T != nullptr) *T = t;
  return true;
}

// Which tensor-core variant takes the layer: 1 kind::i8 (int4 / int2 layers), 0 kind::f16, -1 none.
inline int tc_variant(const bqg_moe_layer* L) {
  if (tc_layer(L, nullptr, true)) return 1;
  return tc_layer(L, nullptr, false) ? 0 : -1;
}

// Workspace of the tensor-core path: the same routing tables, then the activation rows (x in
// expert-grouped order, x of the shared expert in token order, the gated hidden rows h) and the
// fp32 per-pair and shared outputs that the combine sums.  kind::f16: fp16 rows.  kind::i8: two
// int8 digit rows per row (the same bytes), a scale and a digit sum per row, and h in fp32 as
// the gate/up epilogue writes it.
struct MoeTcLayout {
  bool i8;
  size_t counts, offsets, active, n_active, ctr, act_info, perm;
  size_t xg, xs, hg, hs, part, sout;
  size_t xg_sc, xg_sum, xs_sc, xs_sum, h32g, h32s, hg_sc, hg_sum, hs_sc, hs_sum;
  size_t total;
};

inline MoeTcLayout moe_ws_layout_tc(const bqg_moe_layer* L, int tokens) {
  MoeTcLayout o{};
  const size_t E = size_t(L->n_experts), T = size_t(tokens), pairs = T * L->top_k;
  const bool sh = L->s_gate != nullptr;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  o.counts = take(4 * E);
  o.offsets = take(4 * (E + 1));
  o.active = take(4 * E);
  o.n_active = take(4);
  o.ctr = take(8);
  o.act_info = take(16 * E);
  o.perm = take(4 * pairs);
  o.i8 = tc_variant(L) == 1;
  o.xg = take(2 * pairs * L->hidden);
  o.xs = sh ? take(2 * T * L->hidden) : 0;
  o.hg = take(2 * pairs * L->inter);
  o.hs = sh ? take(2 * T * L->shared_inter) : 0;
  o.part = take(4 * pairs * L->hidden);
  o.sout = sh ? take(4 * T * L->hidden) : 0;
  if (o.i8) {
    o.xg_sc = take(4 * pairs);
    o.xg_sum = take(4 * pairs);
    o.hg_sc = take(4 * pairs);
    o.hg_sum = take(4 * pairs);
    o.h32g = take(4 * pairs * L->inter);
    if (sh) {
      o.xs_sc = take(4 * T);
      o.xs_sum = take(4 * T);
      o.hs_sc = take(4 * T);
      o.hs_sum = take(4 * T);
      o.h32s = take(4 * T * L->shared_inter);
    }
  }
  o.total = off;
  return o;
}

// The automatic choice.  A tensor-core MMA instruction (M = 128 weight rows) costs the same
// whatever the number of tokens on its N side, so that path pays per weight read, while the
// CUDA-core path pays per (weight, token).  Measured on B200 (us per layer, CUDA cores / tensor
// cores): Gemma-like layer T = 4: 80 / 102, T = 8: 137 / 104; GLM-like layer T = 4: 157 / 167,
// T = 8: 290 / 245, T = 64: 2058 / 887.  So the tensor cores from 8 tokens on, even when the
// routed experts average well under one token each.
inline bool moe_tc_preferred(const bqg_moe_layer*, int tokens) { return tokens >= BQG_MOE_TC_MIN_TOKENS; }

// Path for `tokens` tokens: BQG_MOE_PATH_CUDA_CORES or BQG_MOE_PATH_TENSOR_CORES (negative: error).
inline int moe_path(const bqg_moe_layer* L, int tokens) {
  if (L->path == BQG_MOE_PATH_CUDA_CORES) return BQG_MOE_PATH_CUDA_CORES;
  const bool tc = tc_variant(L) >= 0;
  if (L->path == BQG_MOE_PATH_TENSOR_CORES) return tc ? int(BQG_MOE_PATH_TENSOR_CORES) : int(BQG_ERR_SHAPE);
  return (tc && moe_tc_preferred(L, tokens)) ? BQG_MOE_PATH_TENSOR_CORES : BQG_MOE_PATH_CUDA_CORES;
}

// Workspace for every call of up to `tokens` tokens (each path's layout grows with the tokens;
// with the automatic choice, fewer tokens may take the other path).
inline size_t moe_ws_total(const bqg_moe_layer* L, int tokens) {
  const int path = moe_path(L, tokens);
  if (path < 0) return 0;
  if (path == BQG_MOE_PATH_CUDA_CORES) return moe_ws_layout(L, tokens).total;
  size_t need = moe_ws_layout_tc(L, tokens).total;
  if (L->path == BQG_MOE_PATH_AUTO) {
    // the largest token count below `tokens` that the automatic choice sends to the CUDA cores
    int below = tokens - 1;
    while (below >= 1 && moe_tc_preferred(L, below)) --below;
    if (below >= 1) {
      const size_t cc = moe_ws_layout(L, below).total;
      if (cc > need) need = cc;
    }
  }
  return need;
}

inline bool valid_fmt(int f) { return f == BQG_Q8_0 || f == BQG_Q4_0 || f == BQG_I4_ROW || f == BQG_I2_ROW; }

inline int check_layer(const bqg_moe_layer* L) {
  if (L == nullptr) return BQG_ERR_ARG;
  if (L->n_experts < 1 || L->top_k < 1 || L->hidden < 1 || L->inter < 1) return BQG_ERR_ARG;
  if (L->n_experts > BQG_MAX_EXPERTS || L->top_k > BQG_MAX_TOPK) return BQG_ERR_LIMIT;
  if (L->top_k > L->n_experts) return BQG_ERR_SHAPE;
  if (!valid_fmt(L->expert_fmt)) return BQG_ERR_FMT;
  if (L->act != BQG_ACT_GELU_TANH && L->act != BQG_ACT_SILU) return BQG_ERR_ARG;
  if (L->path != BQG_MOE_PATH_AUTO && L->path != BQG_MOE_PATH_CUDA_CORES && L->path != BQG_MOE_PATH_TENSOR_CORES)
    return BQG_ERR_ARG;
  if (L->hidden % 32 || L->inter % 32) return BQG_ERR_SHAPE;
  if (L->expert_fmt == BQG_I2_ROW && (L->hidden % 64 || L->inter % 64)) return BQG_ERR_SHAPE;
  if (L->hidden > kMoeMaxCols || L->inter > kMoeMaxCols) return BQG_ERR_LIMIT;
  if (L->gate == nullptr || L->up == nullptr || L->down == nullptr) return BQG_ERR_ARG;
  if (!aligned(L->gate, 16) || !aligned(L->up, 16) || !aligned(L->down, 16)) return BQG_ERR_ALIGN;
  if (L->gate_stride % 16 || L->up_stride % 16 || L->down_stride % 16) return BQG_ERR_ALIGN;
  if (L->n_experts > 1) {
    if (L->gate_stride < weight_bytes(L->expert_fmt, L->inter, L->hidden) ||
        L->up_stride < weight_bytes(L->expert_fmt, L->inter, L->hidden) ||
        L->down_stride < weight_bytes(L->expert_fmt, L->hidden, L->inter))
      return BQG_ERR_SHAPE;
  }
  if (L->s_gate != nullptr) {
    if (L->s_up == nullptr || L->s_down == nullptr) return BQG_ERR_ARG;
    if (!valid_fmt(L->shared_fmt)) return BQG_ERR_FMT;
    if (L->shared_inter < 1 || L->shared_inter % 32) return BQG_ERR_SHAPE;
    if (L->shared_fmt == BQG_I2_ROW && (L->hidden % 64 || L->shared_inter % 64)) return BQG_ERR_SHAPE;
    if (L->shared_inter > kMoeMaxCols) return BQG_ERR_LIMIT;
    if (!aligned(L->s_gate, 16) || !aligned(L->s_up, 16) || !aligned(L->s_down, 16)) return BQG_ERR_ALIGN;
  }
  return BQG_OK;
}

// one attribute cache per kernel instance (5 x 5)
inline SmemAttrOnce g_moe_attr[25];
inline int moe_kind_index(int kind) {
  return kind == kQ4One ? 0 : kind == kQ8One ? 1 : kind == kI4x64 ? 2 : kind == kI2x64 ? 4 : 3;
}

inline int quant_grid(long long threads, int cap) {
  long long g = (threads + 255) / 256;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return int(g);
}

// One grouped-GEMM launch (phase 0 gate/up, 1 down) of the tensor-core path.
// kind::i8 extras of one launch: per activation row scales and digit sums, fp32 h outputs.
struct TcI8Args {
  const float* bscale[2];
  const int32_t* bsum[2];
  float* h32[2];
};

inline int launch_moe_tc(const bqg_moe_layer* L, const TcLayer& TL, int phase, int tokens, const RouteWs& route,
                         const void* b_routed, const void* b_shared, __half* h_routed, __half* h_shared,
                         float* part, float* sout, const TcI8Args* i8, int dev, const DeviceInfo* info,
                         cudaStream_t s) {
  const bool sh = L->s_gate != nullptr;
  const int pairs = tokens * L->top_k;
  TcParams P{};
  int st;
  if (phase == 0) {
    P.fam[0] = TL.gate;
    P.fam[1] = TL.up;
    P.fam[2] = sh ? TL.s_gate : TL.gate;
    P.fam[3] = sh ? TL.s_up : TL.up;
  } else {
    P.fam[0] = TL.down0;
    P.fam[1] = TL.down1;
    P.fam[2] = sh ? TL.s_down0 : TL.down0;
    P.fam[3] = sh ? TL.s_down1 : TL.down1;
  }
  for (int i = 0; i < 4; ++i) {
    const int ne = i < 2 ? L->n_experts : (sh ? 1 : L->n_experts);
    if ((st = tc_encode_amap(&P.amap[i], P.fam[i], ne)) != BQG_OK) return st;
  }
  const int kb = phase == 0 ? L->hidden : L->inter;
  const int kbs = phase == 0 ? L->hidden : L->shared_inter;
  if (i8 != nullptr) {
    if ((st = tc_encode_bmap_i8(&P.bmap[0], static_cast<const int8_t*>(b_routed), 2 * pairs, kb)) != BQG_OK) return st;
    if (sh && (st = tc_encode_bmap_i8(&P.bmap[1], static_cast<const int8_t*>(b_shared), 2 * tokens, kbs)) != BQG_OK)
      return st;
    for (int i = 0; i < 2; ++i) {
      P.bscale[i] = i8->bscale[i];
      P.bsum[i] = i8->bsum[i];
      P.h32[i] = i8->h32[i];
    }
    P.nmax = kTcNMax / 2;
  } else {
    if ((st = tc_encode_bmap(&P.bmap[0], static_cast<const __half*>(b_routed), pairs, kb)) != BQG_OK) return st;
    if (sh && (st = tc_encode_bmap(&P.bmap[1], static_cast<const __half*>(b_shared), tokens, kbs)) != BQG_OK)
      return st;
    P.nmax = kTcNMax;
  }
  if (!sh) P.bmap[1] = P.bmap[0];
  P.phase = phase;
  P.act = L->act;
  P.tokens = tokens;
  P.has_shared = sh ? 1 : 0;
  P.tiles_r = phase == 0 ? (L->inter + 127) / 128 : (L->hidden + 255) / 256;
  P.tiles_s = phase == 0 ? (L->shared_inter + 127) / 128 : (L->hidden + 255) / 256;
  int win = 0;
  for (int i = 0; i < 4; ++i) win = P.fam[i].win > win ? P.fam[i].win : win;
  tc_raw_ring(win, &P.raw_stages, &P.raw_stage_bytes);
  P.act_info = route.act_info;
  P.n_active = route.n_active;
  P.perm = route.perm;
  P.ctr = route.ctr + phase;
  P.hout[0] = h_routed;
  P.hout[1] = h_shared;
  P.hstride[0] = L->inter;
  P.hstride[1] = L->shared_inter;
  P.hperm[0] = L->expert_fmt != BQG_Q8_0;
  P.hperm[1] = sh && L->shared_fmt != BQG_Q8_0;
  P.yout[0] = part;
  P.yout[1] = sout;
  P.ystride = L->hidden;
  const size_t smem = tc_smem_bytes(P.raw_stages, P.raw_stage_bytes);
  if (i8 != nullptr) {
    if ((st = g_tc_attr_i8.ensure(dev, k_moe_tc<true>, kTcMaxSmem)) != BQG_OK) return st;
    return launch_pdl(k_moe_tc<true>, dim3(info->sm_count), dim3(kTcThreads), smem, s, P);
  }
  if ((st = g_tc_attr.ensure(dev, k_moe_tc<false>, kTcMaxSmem)) != BQG_OK) return st;
  return launch_pdl(k_moe_tc<false>, dim3(info->sm_count), dim3(kTcThreads), smem, s, P);
}

}  // namespace bqg

namespace bqg {
// The layer on the tensor-core path: route grouping (one block), fp16 activation rows, the
// grouped gate/up GEMM with act(g) * u in its epilogue, the grouped down GEMM, the combine.
inline int moe_forward_tc(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w, float* y,
                          int tokens, uint8_t* ws, int dev, const DeviceInfo* info, cudaStream_t s, int skip_negative,
                          int accumulate) {
  const int variant = tc_variant(L);
  TcLayer TL;
  if (variant < 0 || !tc_layer(L, &TL, variant == 1)) return BQG_ERR_SHAPE;
  const MoeTcLayout lay = moe_ws_layout_tc(L, tokens);
  const bool sh = L->s_gate != nullptr;
  const int pairs = tokens * L->top_k;
  RouteWs route;
  route.counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  route.offsets = reinterpret_cast<int32_t*>(ws + lay.offsets);
  route.active = reinterpret_cast<int32_t*>(ws + lay.active);
  route.n_active = reinterpret_cast<int32_t*>(ws + lay.n_active);
  route.perm = reinterpret_cast<int32_t*>(ws + lay.perm);
  route.ctr = reinterpret_cast<uint32_t*>(ws + lay.ctr);
  route.act_info = reinterpret_cast<int4*>(ws + lay.act_info);
  route.skip_negative = skip_negative;
  auto H = [&](size_t o) { return reinterpret_cast<__half*>(ws + o); };
  auto F = [&](size_t o) { return reinterpret_cast<float*>(ws + o); };
  int st;
  // 1. route grouping
  QuantJobs none{};
  none.n = 0;
  if ((st = launch_pdl(k_moe_prep, dim3(1), dim3(kRouteThreads), 0, s, idx, pairs, L->n_experts, route, none)) !=
      BQG_OK)
    return st;
  if (lay.i8) {
    // kind::i8: int8 digit rows of x, gate/up (h in fp32), digit rows of h, down
    auto B = [&](size_t o) { return reinterpret_cast<int8_t*>(ws + o); };
    auto I = [&](size_t o) { return reinterpret_cast<int32_t*>(ws + o); };
    const int rows_grid = quant_grid((long long)pairs * 32, 4 * info->sm_count);
    const int rows_grid_s = quant_grid((long long)tokens * 32, 4 * info->sm_count);
    const int32_t* routed_rows = route.offsets + L->n_experts;
    if ((st = launch_pdl(k_moe_digits, dim3(rows_grid), dim3(256), 0, s, x, (const int32_t*)route.perm, L->top_k,
                         routed_rows, 0, L->hidden, L->expert_fmt, B(lay.xg), F(lay.xg_sc), I(lay.xg_sum))) != BQG_OK)
      return st;
    if (sh && (st = launch_pdl(k_moe_digits, dim3(rows_grid_s), dim3(256), 0, s, x, (const int32_t*)nullptr, 1,
                               (const int32_t*)nullptr, tokens, L->hidden, L->shared_fmt, B(lay.xs), F(lay.xs_sc),
                               I(lay.xs_sum))) != BQG_OK)
      return st;
    TcI8Args a0{};
    a0.bscale[0] = F(lay.xg_sc);
    a0.bsum[0] = I(lay.xg_sum);
    a0.bscale[1] = sh ? F(lay.xs_sc) : nullptr;
    a0.bsum[1] = sh ? I(lay.xs_sum) : nullptr;
    a0.h32[0] = F(lay.h32g);
    a0.h32[1] = sh ? F(lay.h32s) : nullptr;
    if ((st = launch_moe_tc(L, TL, 0, tokens, route, B(lay.xg), sh ? B(lay.xs) : nullptr, nullptr, nullptr, nullptr,
                            nullptr, &a0, dev, info, s)) != BQG_OK)
      return st;
    if ((st = launch_pdl(k_moe_digits, dim3(rows_grid), dim3(256), 0, s, (const float*)F(lay.h32g),
                         (const int32_t*)nullptr, 1, routed_rows, 0, L->inter, L->expert_fmt, B(lay.hg),
                         F(lay.hg_sc), I(lay.hg_sum))) != BQG_OK)
      return st;
    if (sh && (st = launch_pdl(k_moe_digits, dim3(rows_grid_s), dim3(256), 0, s, (const float*)F(lay.h32s),
                               (const int32_t*)nullptr, 1, (const int32_t*)nullptr, tokens, L->shared_inter,
                               L->shared_fmt, B(lay.hs), F(lay.hs_sc), I(lay.hs_sum))) != BQG_OK)
      return st;
    TcI8Args a1{};
    a1.bscale[0] = F(lay.hg_sc);
    a1.bsum[0] = I(lay.hg_sum);
    a1.bscale[1] = sh ? F(lay.hs_sc) : nullptr;
    a1.bsum[1] = sh ? I(lay.hs_sum) : nullptr;
    if ((st = launch_moe_tc(L, TL, 1, tokens, route, B(lay.hg), sh ? B(lay.hs) : nullptr, nullptr, nullptr,
                            F(lay.part), sh ? F(lay.sout) : nullptr, &a1, dev, info, s)) != BQG_OK)
      return st;
  } else {
    // 2. activation rows in fp16 (grouped order for the routed experts, token order for the shared one)
    const long long chunks = (long long)(pairs + (sh ? tokens : 0)) * (L->hidden / 8);
    if ((st = launch_pdl(k_moe_xprep, dim3(quant_grid(chunks, 4 * info->sm_count)), dim3(256), 0, s, x,
                         (const int32_t*)route.perm, (const int32_t*)route.offsets, L->n_experts, L->top_k, tokens,
                         L->hidden, H(lay.xg), int(L->expert_fmt != BQG_Q8_0), sh ? H(lay.xs) : (__half*)nullptr,
                         int(sh && L->shared_fmt != BQG_Q8_0))) != BQG_OK)
      return st;
    // 3. gate/up with h = act(g) * u in the epilogue
    if ((st = launch_moe_tc(L, TL, 0, tokens, route, H(lay.xg), sh ? H(lay.xs) : nullptr, H(lay.hg),
                            sh ? H(lay.hs) : nullptr, nullptr, nullptr, nullptr, dev, info, s)) != BQG_OK)
      return st;
    // 4. down
    if ((st = launch_moe_tc(L, TL, 1, tokens, route, H(lay.hg), sh ? H(lay.hs) : nullptr, nullptr, nullptr,
                            F(lay.part), sh ? F(lay.sout) : nullptr, nullptr, dev, info, s)) != BQG_OK)
      return st;
  }
  // 5. combine
  const long long n = (long long)tokens * L->hidden;
  return launch_pdl(k_moe_combine, dim3(unsigned((n + 255) / 256)), dim3(256), 0, s, (const float*)F(lay.part), idx, w,
                    sh ? (const float*)F(lay.sout) : (const float*)nullptr, y, tokens, L->top_k, L->hidden,
                    L->n_experts, accumulate);
}
}  // namespace bqg

extern "C" size_t moe_workspace_size(const bqg_moe_layer* L, int tokens) {
  if (bqg::check_layer(L) != BQG_OK || tokens < 1) return 0;
  return bqg::moe_ws_total(L, tokens);
}

namespace bqg {
// moe_forward with two internal options: skip_negative (negative ids mark pairs that belong to
// another call: skipped without an error) and accumulate (y += this call's sum instead of y =).
inline int moe_forward_impl(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w, float* y,
                            int tokens, void* workspace, size_t ws_bytes, void* stream, int skip_negative,
                            int accumulate) {
  int st = check_layer(L);
  if (st != BQG_OK) return st;
  if (x == nullptr || idx == nullptr || w == nullptr || y == nullptr || tokens < 1) return BQG_ERR_ARG;
  if ((long long)tokens * L->top_k > (1 << 24)) return BQG_ERR_LIMIT;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(idx, 4) || !aligned(w, 4)) return BQG_ERR_ALIGN;
  const int path = moe_path(L, tokens);
  if (path < 0) return path;
  if (workspace == nullptr || ws_bytes < moe_ws_total(L, tokens)) return BQG_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BQG_ERR_ALIGN;
  int dev;
  DeviceInfo* info;
  st = current_device(&dev, &info);
  if (st != BQG_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (path == BQG_MOE_PATH_TENSOR_CORES)
    return moe_forward_tc(L, x, idx, w, y, tokens, ws, dev, info, s, skip_negative, accumulate);
  const MoeWsLayout lay = moe_ws_layout(L, tokens);
  auto F = [&](size_t o) { return reinterpret_cast<float*>(ws + o); };
  auto R = [&](size_t o) { return reinterpret_cast<uint4*>(ws + o); };
  const bool sh = L->s_gate != nullptr;
  const int pairs = tokens * L->top_k;

  RouteWs route;
  route.counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  route.offsets = reinterpret_cast<int32_t*>(ws + lay.offsets);
  route.active = reinterpret_cast<int32_t*>(ws + lay.active);
  route.n_active = reinterpret_cast<int32_t*>(ws + lay.n_active);
  route.perm = reinterpret_cast<int32_t*>(ws + lay.perm);
  route.ctr = reinterpret_cast<uint32_t*>(ws + lay.ctr);
  route.act_info = reinterpret_cast<int4*>(ws + lay.act_info);
  route.skip_negative = skip_negative;

  // routed and shared matrix families
  const MgMat gate = mg_mat(L->expert_fmt, L->gate, L->gate_stride, L->inter, L->hidden);
  const MgMat up = mg_mat(L->expert_fmt, L->up, L->up_stride, L->inter, L->hidden);
  const MgMat down = mg_mat(L->expert_fmt, L->down, L->down_stride, L->hidden, L->inter);
  MgMat s_gate{}, s_up{}, s_down{};
  if (sh) {
    s_gate = mg_mat(L->shared_fmt, L->s_gate, 0, L->shared_inter, L->hidden);
    s_up = mg_mat(L->shared_fmt, L->s_up, 0, L->shared_inter, L->hidden);
    s_down = mg_mat(L->shared_fmt, L->s_down, 0, L->hidden, L->shared_inter);
  }

  // 1. route grouping + x in integer form
  QuantJobs qx{};
  qx.j[0] = QuantJob{x, nullptr, R(lay.xq), tokens, L->hidden, gate.kind, L->act};
  qx.n = 1;
  if (sh) qx.j[qx.n++] = QuantJob{x, nullptr, R(lay.s_xq), tokens, L->hidden, s_gate.kind, L->act};
  // one thread per 8 values
  const long long xsegs = (long long)tokens * L->hidden / 8 * (sh ? 2 : 1);
  const int prep_grid = 1 + int((xsegs + kRouteThreads - 1) / kRouteThreads < info->sm_count
                                    ? (xsegs + kRouteThreads - 1) / kRouteThreads
                                    : info->sm_count);
  if ((st = launch_pdl(k_moe_prep, dim3(prep_grid), dim3(kRouteThreads), 0, s, idx, pairs, L->n_experts, route, qx)) !=
      BQG_OK)
    return st;

  MgPhase P{};
  P.top_k = L->top_k;
  P.tokens = tokens;
  P.counts = route.counts;
  P.offsets = route.offsets;
  P.active = route.active;
  P.n_active = route.n_active;
  P.perm = route.perm;
  P.act_info = route.act_info;

  // 2. gate/up of the touched experts (and of the shared expert)
  P.m[0] = gate;
  P.m[1] = up;
  P.nmat = 2;
  P.xq = R(lay.xq);
  P.out[0] = F(lay.g);
  P.out[1] = F(lay.u);
  P.x_by_token = 1;
  if (sh) {
    P.m[2] = s_gate;
    P.m[3] = s_up;
    P.s_nmat = 2;
    P.s_xq = R(lay.s_xq);
    P.out[2] = F(lay.gs);
    P.out[3] = F(lay.us);
  }
  P.ctr = route.ctr;
  {
    const int kr = gate.kind, ks = sh ? s_gate.kind : gate.kind;
    const MgKernel k = mg_kernel(kr, ks);
    if ((st = g_moe_attr[moe_kind_index(kr) * 5 + moe_kind_index(ks)].ensure(dev, k, kMgSmemBytes)) != BQG_OK)
      return st;
    if ((st = launch_pdl(k, dim3(info->sm_count), dim3(kGemvThreads), kMgSmemBytes, s, P)) != BQG_OK) return st;
  }

  // 3. h = act(g) * u in integer form
  QuantJobs qh{};
  qh.j[0] = QuantJob{F(lay.g), F(lay.u), R(lay.hq), pairs, L->inter, down.kind, L->act};
  qh.n = 1;
  if (sh) qh.j[qh.n++] = QuantJob{F(lay.gs), F(lay.us), R(lay.hsq), tokens, L->shared_inter, s_down.kind, L->act};
  const long long hsegs = ((long long)pairs * L->inter + (sh ? (long long)tokens * L->shared_inter : 0)) / 8;
  if ((st = launch_pdl(k_moe_quant, dim3(quant_grid(hsegs, 4 * info->sm_count)), dim3(256), 0, s, qh)) != BQG_OK)
    return st;

  // 4. down of the touched experts (and of the shared expert)
  MgPhase D = P;
  D.m[0] = down;
  D.nmat = 1;
  D.xq = R(lay.hq);
  D.out[0] = F(lay.part);
  D.out[1] = nullptr;
  D.x_by_token = 0;
  D.s_nmat = 0;
  if (sh) {
    D.m[2] = s_down;
    D.s_nmat = 1;
    D.s_xq = R(lay.hsq);
    D.out[2] = F(lay.sout);
    D.out[3] = nullptr;
  }
  D.ctr = route.ctr + 1;
  {
    const int kr = down.kind, ks = sh ? s_down.kind : down.kind;
    const MgKernel k = mg_kernel(kr, ks);
    if ((st = g_moe_attr[moe_kind_index(kr) * 5 + moe_kind_index(ks)].ensure(dev, k, kMgSmemBytes)) != BQG_OK)
      return st;
    if ((st = launch_pdl(k, dim3(info->sm_count), dim3(kGemvThreads), kMgSmemBytes, s, D)) != BQG_OK) return st;
  }

  // 5. combine
  const long long n = (long long)tokens * L->hidden;
  return launch_pdl(k_moe_combine, dim3(unsigned((n + 255) / 256)), dim3(256), 0, s, F(lay.part), idx, w,
                    sh ? F(lay.sout) : nullptr, y, tokens, L->top_k, L->hidden, L->n_experts, accumulate);
}
}  // namespace bqg

extern "C" int moe_forward(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w, float* y,
                           int tokens, void* workspace, size_t ws_bytes, void* stream) {
  return bqg::moe_forward_impl(L, x, idx, w, y, tokens, workspace, ws_bytes, stream, 0, 0);
}
