// Host side of the MoE layer: workspace layout, argument checks, tile planning, launches.
#pragma once

#include "host_common.h"
#include "moe.cuh"
#include "qgemv_api.cuh"

namespace bqg {

constexpr int kMoeMaxCols = 8192;  // hidden / inter / shared_inter limit of moe_forward

inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct MoeWsLayout {
  size_t counts, offsets, active, n_active, perm, h, part, hs, sout, total;
};

inline MoeWsLayout moe_ws_layout(const bqg_moe_layer* L, int tokens) {
  MoeWsLayout o{};
  const size_t E = size_t(L->n_experts), pairs = size_t(tokens) * L->top_k;
  size_t off = 0;
  o.counts = off; off += 4 * E;
  o.offsets = off; off += 4 * (E + 1);
  o.active = off; off += 4 * E;
  o.n_active = off; off += 4;
  o.perm = off; off += 4 * pairs;
  off = align256(off);
  o.h = off; off = align256(off + 4 * pairs * L->inter);
  o.part = off; off = align256(off + 4 * pairs * L->hidden);
  if (L->s_gate != nullptr) {
    o.hs = off; off = align256(off + 4 * size_t(tokens) * L->shared_inter);
    o.sout = off; off = align256(off + 4 * size_t(tokens) * L->hidden);
  }
  o.total = off;
  return o;
}

inline bool valid_fmt(int f) { return f == BQG_Q8_0 || f == BQG_Q4_0 || f == BQG_I4_ROW; }

inline int check_layer(const bqg_moe_layer* L) {
  if (L == nullptr) return BQG_ERR_ARG;
  if (L->n_experts < 1 || L->top_k < 1 || L->hidden < 1 || L->inter < 1) return BQG_ERR_ARG;
  if (L->n_experts > BQG_MAX_EXPERTS || L->top_k > BQG_MAX_TOPK) return BQG_ERR_LIMIT;
  if (L->top_k > L->n_experts) return BQG_ERR_SHAPE;
  if (!valid_fmt(L->expert_fmt)) return BQG_ERR_FMT;
  if (L->act != BQG_ACT_GELU_TANH && L->act != BQG_ACT_SILU) return BQG_ERR_ARG;
  if (L->hidden % 32 || L->inter % 32) return BQG_ERR_SHAPE;
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
    if (L->shared_inter > kMoeMaxCols) return BQG_ERR_LIMIT;
    if (!aligned(L->s_gate, 16) || !aligned(L->s_up, 16) || !aligned(L->s_down, 16)) return BQG_ERR_ALIGN;
  }
  return BQG_OK;
}

// Matrix family description for the grouped kernel.
inline int moe_mat(int fmt, const void* base, size_t stride, int rows, int cols, MoeMat* out) {
  MoeMat M{};
  GemvProb P{};
  // reuse the GEMV unit selection (kind, row bytes, units, scale offset)
  const int st = make_gemv_prob(fmt, base, reinterpret_cast<const float*>(base),
                                reinterpret_cast<float*>(const_cast<void*>(base)), rows, cols, &P);
  if (st != BQG_OK) return st;
  M.base = static_cast<const uint8_t*>(base);
  M.stride = (long long)stride;
  M.rows = rows;
  M.cols = cols;
  M.kind = P.kind;
  M.row_bytes = P.row_bytes;
  M.units = P.units;
  M.scale_off = P.scale_off;
  *out = M;
  return BQG_OK;
}

// Lanes per row, rows per tile and tokens per token tile for one matrix family.
inline void moe_plan(const MoeMat& M, int nmat, int& lpr, int& tile_rows, int& tiles, int& tb) {
  lpr = M.units <= 64 ? 8 : (M.units <= 128 ? 16 : 32);
  const int rows_per_pass = kMoeThreads / lpr;
  int tr = kMoeMaxVRows / nmat;
  if (tr > rows_per_pass) tr = rows_per_pass;
  while (tr > 1 && nmat * (((tr * M.row_bytes + 47) / 16) * 16) > kMoeSlotBytes) --tr;
  if (tr > M.rows) tr = M.rows;
  tile_rows = tr;
  tiles = (M.rows + tr - 1) / tr;
  const int uw = unit_weights(M.kind);
  const int per_tok = M.units * (uw + 4) * 4;
  tb = kMoeXBytes / per_tok;
  if (tb > kMoeMaxTok) tb = kMoeMaxTok;
}

inline SmemAttrOnce g_moe_attr;

}  // namespace bqg

extern "C" size_t moe_workspace_size(const bqg_moe_layer* L, int tokens) {
  if (bqg::check_layer(L) != BQG_OK || tokens < 1) return 0;
  return bqg::moe_ws_layout(L, tokens).total;
}

extern "C" int moe_forward(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w, float* y,
                           int tokens, void* workspace, size_t ws_bytes, void* stream) {
  int st = bqg::check_layer(L);
  if (st != BQG_OK) return st;
  if (x == nullptr || idx == nullptr || w == nullptr || y == nullptr || tokens < 1) return BQG_ERR_ARG;
  if ((long long)tokens * L->top_k > (1 << 24)) return BQG_ERR_LIMIT;
  if (!bqg::aligned(x, 16) || !bqg::aligned(y, 16) || !bqg::aligned(idx, 4) || !bqg::aligned(w, 4))
    return BQG_ERR_ALIGN;
  const bqg::MoeWsLayout lay = bqg::moe_ws_layout(L, tokens);
  if (workspace == nullptr || ws_bytes < lay.total) return BQG_ERR_WORKSPACE;
  if (!bqg::aligned(workspace, 256)) return BQG_ERR_ALIGN;
  int dev;
  bqg::DeviceInfo* info;
  st = bqg::current_device(&dev, &info);
  if (st != BQG_OK) return st;
  st = bqg::g_moe_attr.ensure(dev, bqg::k_moe_grouped, bqg::kMoeSmemBytes);
  if (st != BQG_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  bqg::RouteWs route;
  route.counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  route.offsets = reinterpret_cast<int32_t*>(ws + lay.offsets);
  route.active = reinterpret_cast<int32_t*>(ws + lay.active);
  route.n_active = reinterpret_cast<int32_t*>(ws + lay.n_active);
  route.perm = reinterpret_cast<int32_t*>(ws + lay.perm);
  float* h = reinterpret_cast<float*>(ws + lay.h);
  float* part = reinterpret_cast<float*>(ws + lay.part);
  const bool has_shared = L->s_gate != nullptr;
  float* hs = has_shared ? reinterpret_cast<float*>(ws + lay.hs) : nullptr;
  float* sout = has_shared ? reinterpret_cast<float*>(ws + lay.sout) : nullptr;
  const int pairs = tokens * L->top_k;

  // 1. route grouping
  bqg::k_moe_route<<<1, bqg::kRouteThreads, 0, s>>>(idx, pairs, L->n_experts, route);
  if ((st = bqg::launch_status()) != BQG_OK) return st;

  // 2. gate/up + activation, 3. down
  for (int phase = 0; phase < 2; ++phase) {
    bqg::MoePhase P{};
    P.route = route;
    P.tokens = tokens;
    P.top_k = L->top_k;
    P.act = L->act;
    P.gateup = phase == 0;
    if (phase == 0) {
      if ((st = bqg::moe_mat(L->expert_fmt, L->gate, L->gate_stride, L->inter, L->hidden, &P.m0)) != BQG_OK) return st;
      if ((st = bqg::moe_mat(L->expert_fmt, L->up, L->up_stride, L->inter, L->hidden, &P.m1)) != BQG_OK) return st;
      P.nmat = 2;
      P.xin = x;
      P.xin_stride = L->hidden;
      P.out = h;
      P.out_stride = L->inter;
    } else {
      if ((st = bqg::moe_mat(L->expert_fmt, L->down, L->down_stride, L->hidden, L->inter, &P.m0)) != BQG_OK) return st;
      P.m1 = P.m0;
      P.nmat = 1;
      P.xin = h;
      P.xin_stride = L->inter;
      P.out = part;
      P.out_stride = L->hidden;
    }
    bqg::moe_plan(P.m0, P.nmat, P.lpr, P.tile_rows, P.tiles, P.tb);
    if (P.tb < 1) return BQG_ERR_LIMIT;
    if (has_shared) {
      P.s_present = 1;
      if (phase == 0) {
        if ((st = bqg::moe_mat(L->shared_fmt, L->s_gate, 0, L->shared_inter, L->hidden, &P.s0)) != BQG_OK) return st;
        if ((st = bqg::moe_mat(L->shared_fmt, L->s_up, 0, L->shared_inter, L->hidden, &P.s1)) != BQG_OK) return st;
        P.s_xin = x;
        P.s_xin_stride = L->hidden;
        P.s_out = hs;
        P.s_out_stride = L->shared_inter;
      } else {
        if ((st = bqg::moe_mat(L->shared_fmt, L->s_down, 0, L->hidden, L->shared_inter, &P.s0)) != BQG_OK) return st;
        P.s1 = P.s0;
        P.s_xin = hs;
        P.s_xin_stride = L->shared_inter;
        P.s_out = sout;
        P.s_out_stride = L->hidden;
      }
      bqg::moe_plan(P.s0, P.nmat, P.s_lpr, P.s_tile_rows, P.s_tiles, P.s_tb);
      if (P.s_tb < 1) return BQG_ERR_LIMIT;
    }
    const int grid = info->sm_count;
    bqg::k_moe_grouped<<<grid, bqg::kMoeThreads, bqg::kMoeSmemBytes, s>>>(P);
    if ((st = bqg::launch_status()) != BQG_OK) return st;
  }

  // 4. combine in slot order, plus the shared output
  const long long n = (long long)tokens * L->hidden;
  bqg::k_moe_combine<<<int((n + 255) / 256), 256, 0, s>>>(part, idx, w, sout, y, tokens, L->top_k, L->hidden,
                                                            L->n_experts);
  return bqg::launch_status();
}
