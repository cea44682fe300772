// Host side of qgemv / qgemv_batched: argument checks, problem descriptors, launch.
#pragma once

#include "host_common.h"
#include "qgemv.cuh"

namespace bqg {

inline size_t weight_bytes(int fmt, int rows, int cols) {
  if (rows < 1 || cols < 32 || cols % 32 != 0) return 0;
  const size_t nb = size_t(cols) / 32;
  switch (fmt) {
    case BQG_Q8_0: return size_t(rows) * nb * 34;
    case BQG_Q4_0: return size_t(rows) * nb * 18;
    case BQG_I4_ROW: {
      const size_t packed = size_t(rows) * size_t(cols / 2);
      return (packed + 15) / 16 * 16 + 4 * size_t(rows);
    }
    case BQG_I2_ROW: {
      if (cols % 64 != 0) return 0;
      const size_t packed = size_t(rows) * size_t(cols / 4);
      return (packed + 15) / 16 * 16 + 4 * size_t(rows);
    }
    default: return 0;
  }
}

// Fills a GemvProb from one (fmt, W, x, y, rows, cols) after checking it.
inline int make_gemv_prob(int fmt, const void* W, const float* x, float* y, int rows, int cols, GemvProb* out) {
  if (W == nullptr || x == nullptr || y == nullptr || rows < 1 || cols < 1) return BQG_ERR_ARG;
  if (fmt != BQG_Q8_0 && fmt != BQG_Q4_0 && fmt != BQG_I4_ROW && fmt != BQG_I2_ROW) return BQG_ERR_FMT;
  if (cols % 32 != 0 || cols > BQG_MAX_COLS) return BQG_ERR_SHAPE;
  if (fmt == BQG_I2_ROW && cols % 64 != 0) return BQG_ERR_SHAPE;
  if (!aligned(W, 16) || !aligned(x, 16) || !aligned(y, 4)) return BQG_ERR_ALIGN;
  GemvProb P{};
  P.W = static_cast<const uint8_t*>(W);
  P.x = x;
  P.y = y;
  P.rows = rows;
  P.cols = cols;
  const int nb = cols / 32;
  if (fmt == BQG_Q8_0) {
    P.kind = (nb % 2 == 0) ? kQ8Pair : kQ8One;
    P.row_bytes = nb * 34;
  } else if (fmt == BQG_Q4_0) {
    P.kind = (nb % 2 == 0) ? kQ4Pair : kQ4One;
    P.row_bytes = nb * 18;
  } else if (fmt == BQG_I2_ROW) {
    P.kind = kI2x64;
    P.row_bytes = cols / 4;
    const long long packed = (long long)rows * P.row_bytes;
    if ((packed + 15) / 16 * 16 > 0x7fffffffLL) return BQG_ERR_LIMIT;
    P.scale_off = int((packed + 15) / 16 * 16);
  } else {
    P.kind = (cols % 64 == 0) ? kI4x64 : kI4x32;
    P.row_bytes = cols / 2;
    const long long packed = (long long)rows * P.row_bytes;
    if ((packed + 15) / 16 * 16 > 0x7fffffffLL) return BQG_ERR_LIMIT;
    P.scale_off = int((packed + 15) / 16 * 16);
  }
  P.units = P.row_bytes / unit_bytes(P.kind);
  if (P.units > kGemvCompute) return BQG_ERR_SHAPE;
  *out = P;
  return BQG_OK;
}

// Cost of a Q4_0 / int4 byte relative to a Q8_0 byte, in sixteenths (1.5 measured best on the
// decode step: 115.0 us against 117.2 us for a pure byte split; 2.0 gives 134 us).
#ifndef BQG_GEMV_NIBBLE_COST16
#define BQG_GEMV_NIBBLE_COST16 24
#endif

inline SmemAttrOnce g_gemv_attr1, g_gemv_attrN;

template <int MAXP>
inline int launch_gemv(GemvParams<MAXP>& prm, long long total_rows, cudaStream_t stream) {
  int dev;
  DeviceInfo* info;
  int st = current_device(&dev, &info);
  if (st != BQG_OK) return st;
  SmemAttrOnce& attr = (MAXP == 1) ? g_gemv_attr1 : g_gemv_attrN;
  st = attr.ensure(dev, k_qgemv<MAXP>, kGemvSmemBytes);
  if (st != BQG_OK) return st;
  // Cost-balanced split: a row costs its bytes times a per-format weight in sixteenths (the
  // nibble formats carry about twice the weights per byte of Q8_0, so more integer dot work per
  // byte).  CTA c owns the rows whose first cost unit lies in [c*T/G, (c+1)*T/G).
  long long total = 0;
  long long row_cost[MAXP];
  for (int i = 0; i < prm.n; ++i) {
    const int w16 = is_q8(prm.p[i].kind) ? 16 : BQG_GEMV_NIBBLE_COST16;
    row_cost[i] = (long long)prm.p[i].row_bytes * w16;
    prm.p[i].byte_start = total;  // here: the matrix's first cost unit
    total += (long long)prm.p[i].rows * row_cost[i];
  }
  prm.total_bytes = total;
  long long g = total_rows < info->sm_count ? total_rows : info->sm_count;
  if (g > kGemvMaxGrid) g = kGemvMaxGrid;
  const int grid = int(g);
  // first_row(b) = the first (problem, row) whose start cost is >= b; b grows with c, so one
  // forward sweep over the problems serves all CTAs.
  int sweep = 0;
  auto first_row = [&](long long b, int& p, int& r) {
    for (p = sweep; p < prm.n; ++p) {
      const GemvProb& P = prm.p[p];
      const long long end = P.byte_start + (long long)P.rows * row_cost[p];
      if (b < end) {
        const long long off = b - P.byte_start;
        r = off <= 0 ? 0 : int((off + row_cost[p] - 1) / row_cost[p]);
        if (r < P.rows) {
          sweep = p;
          return;
        }
      }
    }
    sweep = p = prm.n;  // past the end
    r = 0;
  };
  CtaRange prev{};
  for (int c = 0; c <= grid; ++c) {
    CtaRange cur{};
    first_row(total * c / grid, cur.p0, cur.r0);
    if (c > 0) {
      prm.cta[c - 1].p0 = prev.p0;
      prm.cta[c - 1].r0 = prev.r0;
      prm.cta[c - 1].p1 = cur.p0;
      prm.cta[c - 1].r1 = cur.r0;
    }
    prev = cur;
  }
  if (prm.am_p >= 0) {  // the CTAs whose row range includes rows of the argmax output
    prm.am_ctas = 0;
    for (int c = 0; c < grid; ++c) {
      const CtaRange& r = prm.cta[c];
      const int q = prm.am_p;
      const int ra = q == r.p0 ? r.r0 : 0;
      const int rb = q < r.p1 ? prm.p[q].rows : (q == r.p1 ? r.r1 : 0);
      if (q >= r.p0 && q <= r.p1 && q < prm.n && ra < rb) ++prm.am_ctas;
    }
    if (prm.am_ctas == 0) return BQG_ERR_ARG;
  }
  k_qgemv<MAXP><<<grid, kGemvThreads, kGemvSmemBytes, stream>>>(prm);
  return launch_status();
}

}  // namespace bqg

extern "C" size_t bqg_weight_bytes(int fmt, int rows, int cols) { return bqg::weight_bytes(fmt, rows, cols); }

namespace bqg {
// The greedy-argmax outputs of a GEMV launch (none when token is null).
template <int MAXP>
inline int set_argmax(GemvParams<MAXP>& prm, int index, int32_t* token, float* value, unsigned long long* state) {
  prm.am_p = -1;
  if (token == nullptr && state == nullptr && value == nullptr) return BQG_OK;
  if (token == nullptr || state == nullptr || index < 0 || index >= prm.n) return BQG_ERR_ARG;
  if (!aligned(token, 4) || !aligned(state, 8) || (value != nullptr && !aligned(value, 4))) return BQG_ERR_ALIGN;
  prm.am_p = index;
  prm.am_token = token;
  prm.am_value = value;
  prm.am_state = state;
  return BQG_OK;
}

inline int qgemv_impl(int fmt, const void* W, const float* x, float* y, int rows, int cols, int32_t* token,
                      float* value, unsigned long long* state, void* stream) {
  GemvParams<1> prm{};
  int st = make_gemv_prob(fmt, W, x, y, rows, cols, &prm.p[0]);
  if (st != BQG_OK) return st;
  prm.n = 1;
  if ((st = set_argmax(prm, 0, token, value, state)) != BQG_OK) return st;
  return launch_gemv<1>(prm, rows, static_cast<cudaStream_t>(stream));
}

inline int qgemv_batched_impl(const bqg_gemv_desc* descs, int n, int am_index, int32_t* token, float* value,
                              unsigned long long* state, void* stream) {
  if (descs == nullptr || n < 1) return BQG_ERR_ARG;
  if (n > BQG_MAX_BATCH) return BQG_ERR_LIMIT;
  static_assert(sizeof(GemvParams<BQG_MAX_BATCH>) < 32000, "kernel parameter block too large");
  GemvParams<BQG_MAX_BATCH> prm{};
  long long total_rows = 0;
  for (int i = 0; i < n; ++i) {
    const bqg_gemv_desc& d = descs[i];
    if (d.reserved != 0) return BQG_ERR_ARG;
    int st = make_gemv_prob(d.fmt, d.W, d.x, d.y, d.rows, d.cols, &prm.p[i]);
    if (st != BQG_OK) return st;
    total_rows += d.rows;
  }
  prm.n = n;
  const int st = set_argmax(prm, am_index, token, value, state);
  if (st != BQG_OK) return st;
  return launch_gemv<BQG_MAX_BATCH>(prm, total_rows, static_cast<cudaStream_t>(stream));
}
}  // namespace bqg

extern "C" int qgemv(int fmt, const void* W, const float* x, float* y, int rows, int cols, void* stream) {
  return bqg::qgemv_impl(fmt, W, x, y, rows, cols, nullptr, nullptr, nullptr, stream);
}

extern "C" int qgemv_batched(const bqg_gemv_desc* descs, int n, void* stream) {
  return bqg::qgemv_batched_impl(descs, n, -1, nullptr, nullptr, nullptr, stream);
}

extern "C" int qgemv_argmax(int fmt, const void* W, const float* x, float* y, int rows, int cols, int32_t* token,
                            float* max_value, unsigned long long* state, void* stream) {
  if (token == nullptr || state == nullptr) return BQG_ERR_ARG;
  return bqg::qgemv_impl(fmt, W, x, y, rows, cols, token, max_value, state, stream);
}

extern "C" int qgemv_batched_argmax(const bqg_gemv_desc* descs, int n, int argmax_index, int32_t* token,
                                    float* max_value, unsigned long long* state, void* stream) {
  if (token == nullptr || state == nullptr) return BQG_ERR_ARG;
  return bqg::qgemv_batched_impl(descs, n, argmax_index, token, max_value, state, stream);
}
