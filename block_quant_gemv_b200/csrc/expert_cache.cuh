// Host-resident routed experts with a per-layer cache of device slots.
//
// Sources: TurboFieldfare wiki, "메모리·전문가 스트리밍" (experts streamed from storage into 16
// per-layer slots with LFU replacement and a recency tie-break; hits and misses split so that
// loads overlap computation); Camelid README, "Supported models" (the SSER lane: experts stay in
// host RAM with an adaptive VRAM expert cache); colibri wiki summary, "구현 범위" (per-layer
// cache of routed experts).
//
// The routed experts of one layer stay in (pinned) host memory; `n_slots` device slots hold the
// ones in use.  For each call the host reads the routing (the caller hands over the top-k ids on
// the host, as an engine that streams experts must), splits the experts into hits (resident) and
// misses, picks a victim slot for every miss (an empty slot, else the least frequently used slot
// not needed by this call, the least recently used among equals), and copies the miss's gate, up
// and down matrices into it with cudaMemcpyAsync on the copy stream.  The layer then runs as two
// MoE passes over the slots on the compute stream: the hit experts (and the shared expert) at
// once, overlapping the copies, and the missed experts once their copies have landed, added to
// the same y.  Each expert's bytes cross PCIe once per miss and are read from HBM once per pass.
#pragma once

#include <cuda_runtime.h>

#include <new>

#include "host_common.h"
#include "moe_api.cuh"

// Plain arrays owned by the object (no standard-library templates: the library exports only its
// C ABI).  Sized at creation: n_experts or n_slots entries; idx_a / idx_b grow with the tokens.
struct bqg_expert_cache {
  bqg_expert_cache_desc d;
  size_t gate_bytes, up_bytes, down_bytes;  // bytes of one expert's matrices
  int* slot_of = nullptr;                   // [E] expert -> slot, or -1
  int* expert_in = nullptr;                 // [S] slot -> expert, or -1
  long long* freq = nullptr;                // [S] uses since the slot's expert was loaded (LFU)
  long long* last = nullptr;                // [S] call number of the slot's last use (recency tie-break)
  int* need = nullptr;                      // [S] stamp of the call that needs the slot
  int* order = nullptr;                     // [E] this call's distinct experts, first appearance first
  char* seen = nullptr;                     // [E] scratch flags
  char* is_miss = nullptr;                  // [E] scratch flags
  int* miss_slot = nullptr;                 // [S] slots loaded by this call
  int32_t* idx_a = nullptr;                 // [cap] remapped routing of the two passes
  int32_t* idx_b = nullptr;
  long long idx_cap = 0;
  long long calls = 0;
  bqg_expert_cache_stats stats{};
  cudaEvent_t copies_done = nullptr;        // after this call's slot copies (copy stream)
  cudaEvent_t prev_done = nullptr;          // after the previous call's work (compute stream)
  ~bqg_expert_cache() {
    delete[] slot_of;
    delete[] expert_in;
    delete[] freq;
    delete[] last;
    delete[] need;
    delete[] order;
    delete[] seen;
    delete[] is_miss;
    delete[] miss_slot;
    delete[] idx_a;
    delete[] idx_b;
  }
};

namespace bqg {

// The slot layer: the same experts, n_experts = n_slots, matrices in the device slots.
inline bqg_moe_layer cache_slot_layer(const bqg_expert_cache* c, bool with_shared) {
  bqg_moe_layer L = c->d.layer;
  L.n_experts = c->d.n_slots;
  L.gate = c->d.slot_gate;
  L.up = c->d.slot_up;
  L.down = c->d.slot_down;
  if (!with_shared) {
    L.s_gate = L.s_up = L.s_down = nullptr;
    L.shared_inter = 0;
  }
  return L;
}

inline size_t cache_idx_bytes(int tokens, int top_k) { return align256(size_t(tokens) * top_k * 4); }

}  // namespace bqg

extern "C" int bqg_expert_cache_create(const bqg_expert_cache_desc* d, bqg_expert_cache** out) {
  using namespace bqg;
  if (d == nullptr || out == nullptr) return BQG_ERR_ARG;
  *out = nullptr;
  if (d->n_slots < 1) return BQG_ERR_ARG;
  if (d->n_slots > BQG_MAX_EXPERTS || d->n_slots > d->layer.n_experts) return BQG_ERR_LIMIT;
  if (d->slot_gate == nullptr || d->slot_up == nullptr || d->slot_down == nullptr) return BQG_ERR_ARG;
  // the slot layer must be a valid MoE layer (strides, formats, shapes, alignment)
  bqg_moe_layer S = d->layer;
  S.n_experts = d->n_slots;
  S.gate = d->slot_gate;
  S.up = d->slot_up;
  S.down = d->slot_down;
  if (S.top_k > S.n_experts) S.top_k = S.n_experts;
  int st = check_layer(&S);
  if (st != BQG_OK) return st;
  if (d->layer.gate == nullptr || d->layer.up == nullptr || d->layer.down == nullptr) return BQG_ERR_ARG;
  bqg_expert_cache* c = new (std::nothrow) bqg_expert_cache();
  if (c == nullptr) return BQG_ERR_LIMIT;
  c->d = *d;
  c->gate_bytes = weight_bytes(d->layer.expert_fmt, d->layer.inter, d->layer.hidden);
  c->up_bytes = c->gate_bytes;
  c->down_bytes = weight_bytes(d->layer.expert_fmt, d->layer.hidden, d->layer.inter);
  const int E = d->layer.n_experts, NS = d->n_slots;
  c->slot_of = new (std::nothrow) int[E];
  c->expert_in = new (std::nothrow) int[NS];
  c->freq = new (std::nothrow) long long[NS];
  c->last = new (std::nothrow) long long[NS];
  c->need = new (std::nothrow) int[NS];
  c->order = new (std::nothrow) int[E];
  c->seen = new (std::nothrow) char[E];
  c->is_miss = new (std::nothrow) char[E];
  c->miss_slot = new (std::nothrow) int[NS];
  if (!c->slot_of || !c->expert_in || !c->freq || !c->last || !c->need || !c->order || !c->seen || !c->is_miss ||
      !c->miss_slot) {
    delete c;
    return BQG_ERR_LIMIT;
  }
  for (int e = 0; e < E; ++e) c->slot_of[e] = -1;
  for (int sl = 0; sl < NS; ++sl) {
    c->expert_in[sl] = -1;
    c->freq[sl] = 0;
    c->last[sl] = -1;
    c->need[sl] = -1;
  }
  if (cudaEventCreateWithFlags(&c->copies_done, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->prev_done, cudaEventDisableTiming) != cudaSuccess) {
    if (c->copies_done) cudaEventDestroy(c->copies_done);
    if (c->prev_done) cudaEventDestroy(c->prev_done);
    delete c;
    return BQG_ERR_CUDA;
  }
  *out = c;
  return BQG_OK;
}

extern "C" void bqg_expert_cache_destroy(bqg_expert_cache* c) {
  if (c == nullptr) return;
  cudaEventDestroy(c->copies_done);
  cudaEventDestroy(c->prev_done);
  delete c;
}

extern "C" size_t bqg_expert_cache_workspace_size(const bqg_expert_cache* c, int tokens) {
  using namespace bqg;
  if (c == nullptr || tokens < 1) return 0;
  const bqg_moe_layer L = cache_slot_layer(c, true);
  const size_t ws = moe_workspace_size(&L, tokens);
  if (ws == 0) return 0;
  return 2 * cache_idx_bytes(tokens, L.top_k) + ws;
}

extern "C" int bqg_expert_cache_get_stats(const bqg_expert_cache* c, bqg_expert_cache_stats* s) {
  if (c == nullptr || s == nullptr) return BQG_ERR_ARG;
  *s = c->stats;
  return BQG_OK;
}

extern "C" int bqg_expert_cache_forward(bqg_expert_cache* c, const float* x, const int32_t* idx_host, const float* w,
                                        float* y, int tokens, void* workspace, size_t ws_bytes, void* stream,
                                        void* copy_stream) {
  using namespace bqg;
  if (c == nullptr || x == nullptr || idx_host == nullptr || w == nullptr || y == nullptr || tokens < 1)
    return BQG_ERR_ARG;
  const int k = c->d.layer.top_k, E = c->d.layer.n_experts, pairs = tokens * k;
  if ((long long)tokens * k > (1 << 24)) return BQG_ERR_LIMIT;
  const size_t need_ws = bqg_expert_cache_workspace_size(c, tokens);
  if (workspace == nullptr || need_ws == 0 || ws_bytes < need_ws) return BQG_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BQG_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream), cs = static_cast<cudaStream_t>(copy_stream);
  const long long call = c->calls;

  // 1. the experts this call needs; more than n_slots distinct experts do not fit the slots
  if ((long long)pairs > c->idx_cap) {
    int32_t* a = new (std::nothrow) int32_t[pairs];
    int32_t* b = new (std::nothrow) int32_t[pairs];
    if (a == nullptr || b == nullptr) {
      delete[] a;
      delete[] b;
      return BQG_ERR_LIMIT;
    }
    delete[] c->idx_a;
    delete[] c->idx_b;
    c->idx_a = a;
    c->idx_b = b;
    c->idx_cap = pairs;
  }
  int distinct = 0;
  for (int e = 0; e < E; ++e) c->seen[e] = c->is_miss[e] = 0;
  for (int p = 0; p < pairs; ++p) {
    const int e = idx_host[p];
    if (e < 0 || e >= E || c->seen[e]) continue;
    c->seen[e] = 1;
    if (distinct >= c->d.n_slots) return BQG_ERR_LIMIT;
    c->order[distinct++] = e;
  }

  // 2. hits keep their slots; every miss takes a victim slot
  const int stamp = int(call & 0x7fffffff);
  for (int i = 0; i < distinct; ++i)
    if (c->slot_of[c->order[i]] >= 0) c->need[c->slot_of[c->order[i]]] = stamp;
  int n_miss = 0;
  for (int i = 0; i < distinct; ++i) {
    const int e = c->order[i];
    if (c->slot_of[e] >= 0) continue;
    int victim = -1;
    for (int sl = 0; sl < c->d.n_slots; ++sl) {
      if (c->need[sl] == stamp) continue;
      if (c->expert_in[sl] < 0) {  // an empty slot first
        victim = sl;
        break;
      }
      if (victim < 0 || c->freq[sl] < c->freq[victim] || (c->freq[sl] == c->freq[victim] && c->last[sl] < c->last[victim]))
        victim = sl;
    }
    if (victim < 0) return BQG_ERR_LIMIT;  // cannot happen: distinct <= n_slots
    if (c->expert_in[victim] >= 0) {
      c->slot_of[c->expert_in[victim]] = -1;
      ++c->stats.evictions;
    }
    c->expert_in[victim] = e;
    c->slot_of[e] = victim;
    c->freq[victim] = 0;
    c->need[victim] = stamp;
    c->is_miss[e] = 1;
    c->miss_slot[n_miss++] = victim;
  }

  // 3. copies of the misses into their slots, after the previous call's work on the compute stream
  //    (which may still read the slots being replaced)
  const bool any_miss = n_miss > 0;
  if (any_miss) {
    if (cudaEventRecord(c->prev_done, s) != cudaSuccess || cudaStreamWaitEvent(cs, c->prev_done, 0) != cudaSuccess)
      return BQG_ERR_CUDA;
    const bqg_moe_layer& H = c->d.layer;
    for (int i = 0; i < n_miss; ++i) {
      const int sl = c->miss_slot[i];
      const int e = c->expert_in[sl];
      const uint8_t* hg = static_cast<const uint8_t*>(H.gate) + size_t(e) * H.gate_stride;
      const uint8_t* hu = static_cast<const uint8_t*>(H.up) + size_t(e) * H.up_stride;
      const uint8_t* hd = static_cast<const uint8_t*>(H.down) + size_t(e) * H.down_stride;
      uint8_t* dg = static_cast<uint8_t*>(c->d.slot_gate) + size_t(sl) * H.gate_stride;
      uint8_t* du = static_cast<uint8_t*>(c->d.slot_up) + size_t(sl) * H.up_stride;
      uint8_t* dd = static_cast<uint8_t*>(c->d.slot_down) + size_t(sl) * H.down_stride;
      if (cudaMemcpyAsync(dg, hg, c->gate_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
          cudaMemcpyAsync(du, hu, c->up_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
          cudaMemcpyAsync(dd, hd, c->down_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return BQG_ERR_CUDA;
      c->stats.bytes_copied += (long long)(c->gate_bytes + c->up_bytes + c->down_bytes);
    }
    if (cudaEventRecord(c->copies_done, cs) != cudaSuccess) return BQG_ERR_CUDA;
  }

  // 4. the two passes' routing over the slots (-1: the pair belongs to the other pass); ids
  //    outside [0, n_experts) stay invalid in the first pass, which skips and flags them
  for (int p = 0; p < pairs; ++p) {
    const int e = idx_host[p];
    if (e < 0 || e >= E) {
      c->idx_a[p] = c->d.n_slots;  // outside the slot layer: skipped and flagged
      c->idx_b[p] = -1;
      continue;
    }
    const int sl = c->slot_of[e];
    c->idx_a[p] = c->is_miss[e] ? -1 : sl;
    c->idx_b[p] = c->is_miss[e] ? sl : -1;
  }
  for (int i = 0; i < distinct; ++i) {
    const int sl = c->slot_of[c->order[i]];
    ++c->freq[sl];
    c->last[sl] = call;
    if (c->is_miss[c->order[i]]) ++c->stats.misses;
    else ++c->stats.hits;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* dev_a = reinterpret_cast<int32_t*>(ws);
  int32_t* dev_b = reinterpret_cast<int32_t*>(ws + cache_idx_bytes(tokens, k));
  uint8_t* moe_ws = ws + 2 * cache_idx_bytes(tokens, k);
  const size_t moe_ws_bytes = ws_bytes - 2 * cache_idx_bytes(tokens, k);
  // pageable source: the copy is staged before the call returns, so the arrays may change later
  if (cudaMemcpyAsync(dev_a, c->idx_a, size_t(pairs) * 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      (any_miss && cudaMemcpyAsync(dev_b, c->idx_b, size_t(pairs) * 4, cudaMemcpyHostToDevice, s) != cudaSuccess))
    return BQG_ERR_CUDA;

  // 5. the hit experts and the shared expert, then (after the copies) the missed experts
  const bqg_moe_layer LA = cache_slot_layer(c, true);
  int st = moe_forward_impl(&LA, x, dev_a, w, y, tokens, moe_ws, moe_ws_bytes, stream, 1, 0);
  if (st != BQG_OK) return st;
  if (any_miss) {
    if (cudaStreamWaitEvent(s, c->copies_done, 0) != cudaSuccess) return BQG_ERR_CUDA;
    const bqg_moe_layer LB = cache_slot_layer(c, false);
    st = moe_forward_impl(&LB, x, dev_b, w, y, tokens, moe_ws, moe_ws_bytes, stream, 1, 1);
    if (st != BQG_OK) return st;
  }
  ++c->calls;
  ++c->stats.calls;
  return BQG_OK;
}
