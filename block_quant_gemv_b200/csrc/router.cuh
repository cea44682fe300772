// MoE router: logits l = R x (fp32), then per token softmax over all experts, the top-k by
// logit (an exact tie goes to the lower expert index) and weights renormalised over the
// selected experts.
//
// Sources: TurboFieldfare wiki, "메모리·전문가 스트리밍" (router choosing top-8 of 128 routed
// experts per token); colibri wiki summary, "핵심 아이디어" (256 routed experts); Camelid
// README, "Windows bring-up, perf & GPU" (exact expert-probability ties go to the lower index).
#pragma once

#include "common.cuh"
#include "host_common.h"

namespace bqg {

// ---------------------------------------------------------------- router logits
// One CTA per (expert row e, tile of up to TT tokens), 256 threads striding over the row in
// 16-byte loads (unrolled so that several loads are in flight per thread).  Each thread keeps
// one accumulator per token; lanes are reduced with a fixed butterfly and the 8 warps in a
// fixed order through shared memory, so results are deterministic.
constexpr int kRouterThreads = 256;
constexpr int kRouterTok = 8;

template <int TT>
__global__ void __launch_bounds__(kRouterThreads) k_router_logits(const float* __restrict__ R,
                                                                  const float* __restrict__ x,
                                                                  float* __restrict__ logits, int tokens,
                                                                  int n_experts, int hidden) {
  __shared__ float part[kRouterThreads / 32][TT];
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x;
  const int t0 = blockIdx.y * TT;
  const int nt = min(TT, tokens - t0);
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  const float4* r4 = reinterpret_cast<const float4*>(R + size_t(e) * hidden);
  const int h4 = hidden / 4;
#pragma unroll 4
  for (int k = threadIdx.x; k < h4; k += kRouterThreads) {
    const float4 r = __ldg(r4 + k);
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (t < nt) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + size_t(t0 + t) * hidden) + k);
        acc[t] = fmaf(r.x, v.x, acc[t]);
        acc[t] = fmaf(r.y, v.y, acc[t]);
        acc[t] = fmaf(r.z, v.z, acc[t]);
        acc[t] = fmaf(r.w, v.w, acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const float s = warp_sum(acc[t]);
    if (lane == 0) part[warp][t] = s;
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kRouterThreads / 32; ++w) s += part[w][threadIdx.x];
    logits[size_t(t0 + threadIdx.x) * n_experts + e] = s;
  }
}

// ---------------------------------------------------------------- softmax + top-k + renormalise
// One warp per token.  Lane l holds logits of experts l, l+32, ... (at most 8 per lane).
// Each of the k rounds picks the largest unselected logit, ties to the lower index,
// by a warp butterfly over (value, index) pairs.  Then p = softmax over all experts
// (max-subtracted, expf) and w_j = p_j / sum of the selected p.
constexpr int kTopkWarps = 4;
constexpr int kTopkPerLane = BQG_MAX_EXPERTS / 32;

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__global__ void __launch_bounds__(kTopkWarps * 32) k_router_topk(const float* __restrict__ logits, int tokens,
                                                                 int n_experts, int k, int32_t* __restrict__ idx,
                                                                 float* __restrict__ weights) {
  griddep_launch_dependents();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= tokens) return;
  const float* lrow = logits + size_t(t) * n_experts;
  float v[kTopkPerLane];
  uint32_t taken = 0;  // bit i: expert lane + 32 i already selected (or absent)
#pragma unroll
  for (int i = 0; i < kTopkPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < n_experts) {
      v[i] = lrow[e];
    } else {
      v[i] = 0.f;
      taken |= 1u << i;
    }
  }
  // softmax over all experts: max and sum of exp(l - max), fixed reduction order
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kTopkPerLane; ++i)
    if (!(taken >> i & 1u)) m = fmaxf(m, v[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < kTopkPerLane; ++i)
    if (!(taken >> i & 1u)) z += expf(v[i] - m);
  z = warp_sum(z);

  int sel_e[BQG_MAX_TOPK];
  float sel_p[BQG_MAX_TOPK];
  float psum = 0.f;
#pragma unroll
  for (int j = 0; j < BQG_MAX_TOPK; ++j) {
    if (j >= k) break;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kTopkPerLane; ++i) {
      const int e = lane + 32 * i;
      if (!(taken >> i & 1u) && better(v[i], e, bv, bi)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    const float p = expf(bv - m) / z;  // softmax probability of the selected expert
    sel_e[j] = bi;
    sel_p[j] = p;
    psum += p;
  }
  if (lane < k) {
    // lane j writes slot j (registers indexed by a runtime j are avoided with a select loop)
    int e_out = 0;
    float p_out = 0.f;
#pragma unroll
    for (int j = 0; j < BQG_MAX_TOPK; ++j)
      if (j == lane) {
        e_out = sel_e[j];
        p_out = sel_p[j];
      }
    idx[size_t(t) * k + lane] = e_out;
    weights[size_t(t) * k + lane] = p_out / psum;
  }
}

}  // namespace bqg

extern "C" int moe_router_logits(const float* R, const float* x, float* logits, int tokens, int n_experts, int hidden,
                                 void* stream) {
  if (R == nullptr || x == nullptr || logits == nullptr || tokens < 1 || n_experts < 1 || hidden < 1)
    return BQG_ERR_ARG;
  if (n_experts > BQG_MAX_EXPERTS) return BQG_ERR_LIMIT;
  if (hidden % 4 != 0 || hidden > BQG_MAX_COLS) return BQG_ERR_SHAPE;
  if (!bqg::aligned(R, 16) || !bqg::aligned(x, 16) || !bqg::aligned(logits, 4)) return BQG_ERR_ALIGN;
  int dev;
  bqg::DeviceInfo* info;
  const int st = bqg::current_device(&dev, &info);
  if (st != BQG_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int gx = n_experts;
  const int threads = bqg::kRouterThreads;
  if (tokens == 1) {
    return bqg::launch_pdl(bqg::k_router_logits<1>, dim3(gx, 1), dim3(threads), 0, s, R, x, logits, tokens, n_experts, hidden);
  } else if (tokens <= 2) {
    return bqg::launch_pdl(bqg::k_router_logits<2>, dim3(gx, 1), dim3(threads), 0, s, R, x, logits, tokens, n_experts, hidden);
  } else if (tokens <= 4) {
    return bqg::launch_pdl(bqg::k_router_logits<4>, dim3(gx, 1), dim3(threads), 0, s, R, x, logits, tokens, n_experts, hidden);
  } else {
    const int gy = (tokens + bqg::kRouterTok - 1) / bqg::kRouterTok;
    if (gy > 65535) return BQG_ERR_LIMIT;
    return bqg::launch_pdl(bqg::k_router_logits<bqg::kRouterTok>, dim3(gx, gy), dim3(threads), 0, s, R, x, logits, tokens,
                           n_experts, hidden);
  }
  return bqg::launch_status();
}

extern "C" int moe_router_topk(const float* logits, int tokens, int n_experts, int k, int32_t* idx, float* weights,
                               void* stream) {
  if (logits == nullptr || idx == nullptr || weights == nullptr || tokens < 1 || n_experts < 1 || k < 1)
    return BQG_ERR_ARG;
  if (n_experts > BQG_MAX_EXPERTS || k > BQG_MAX_TOPK) return BQG_ERR_LIMIT;
  if (k > n_experts) return BQG_ERR_SHAPE;
  if (!bqg::aligned(logits, 4) || !bqg::aligned(idx, 4) || !bqg::aligned(weights, 4)) return BQG_ERR_ALIGN;
  int dev;
  bqg::DeviceInfo* info;
  const int st = bqg::current_device(&dev, &info);
  if (st != BQG_OK) return st;
  const int grid = (tokens + bqg::kTopkWarps - 1) / bqg::kTopkWarps;
  return bqg::launch_pdl(bqg::k_router_topk, dim3(grid), dim3(bqg::kTopkWarps * 32), 0,
                         static_cast<cudaStream_t>(stream), logits, tokens, n_experts, k, idx, weights);
}
