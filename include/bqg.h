/*
 * bqg.h — C ABI of libbqg.so: block-quantized GEMV, routed MoE layer and prefill-chunk GEMM
 * for NVIDIA B200 (sm_100a).
 *
 * What the calls compute comes from the descriptions of local LLM inference engines that
 * stream quantized weights during decode:
 *   - Camelid README, "Engine status" (Q8_0 inference) and "Gemma 4" (Q4_0 projections decoded
 *     on the GPU by GEMVs; dense shared expert + sparse top-8 branch of a 128-expert MoE);
 *   - colibri wiki summary, "핵심 아이디어" (256 routed experts, ~19 MB int4 experts) and
 *     "구현 범위" (packed int4 with a per-row scale);
 *   - TurboFieldfare wiki, "메모리·전문가 스트리밍" (top-8 of 128 routed experts, dense shared
 *     branch, prefill in chunks of at most 128 tokens reusing each expert read);
 *   - llama-modchip review, "개요" (decode speed is set by the weight bytes read per token).
 *
 * Conventions for every call
 *   - Pointers named W, x, y, X, Y, R, logits, idx, weights, workspace and the pointers inside
 *     bqg_moe_layer are DEVICE pointers owned by the caller.  Descriptor arrays
 *     (bqg_gemv_desc*, bqg_moe_layer*) are HOST pointers read during the call only.
 *   - The library allocates no device memory, keeps no per-call state and never synchronises
 *     the device, except where a call says so.  All work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL means the legacy default stream).
 *   - Arguments are validated on the host before any launch.  A failed check returns a
 *     negative bqg_status and launches nothing.  A failed launch returns BQG_ERR_CUDA.
 *   - Sizes are element counts unless named *_bytes.  Matrices are row-major.
 *   - Float outputs are fp32 (fp16 for the prefill GEMM).  Accumulation is fp32.
 *
 * Weight formats (the byte layout of one matrix with `rows` rows of `cols` weights; rows are
 * stored one after another, row r holding its cols/32 blocks in order):
 *   BQG_Q8_0   block of 32 weights = 34 bytes: little-endian fp16 scale d, then int8 q[32];
 *              weight = d * q.
 *   BQG_Q4_0   block of 32 weights = 18 bytes: fp16 d, then qs[16]; weight 2j of the block is
 *              the LOW nibble of qs[j] and weight 2j+1 the HIGH nibble; weight = (q - 8) * d.
 *   BQG_I4_ROW row r = cols/2 bytes of two's-complement nibbles (weight 2j in the low nibble
 *              of byte j); after all rows, zero padding to a 16-byte boundary, then one
 *              little-endian fp32 scale per row; y_r = s_r * sum_i q_ri * x_i.
 */
#ifndef BQG_H
#define BQG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status, enums, limits */
enum bqg_status {
  BQG_OK = 0,
  BQG_ERR_ARG = -1,       /* null pointer, non-positive size or unknown enum value        */
  BQG_ERR_FMT = -2,       /* weight format not accepted by this call                       */
  BQG_ERR_SHAPE = -3,     /* shape precondition violated (cols % 32, k > n_experts, ...)   */
  BQG_ERR_ALIGN = -4,     /* pointer alignment precondition violated                       */
  BQG_ERR_WORKSPACE = -5, /* workspace NULL or smaller than moe_workspace_size()           */
  BQG_ERR_CUDA = -6,      /* a CUDA runtime call or kernel launch failed                   */
  BQG_ERR_DEVICE = -7,    /* current device is not a compute capability 10.0 GPU           */
  BQG_ERR_LIMIT = -8      /* a documented maximum is exceeded (descriptor count, sizes)    */
};

enum bqg_fmt { BQG_Q8_0 = 1, BQG_Q4_0 = 2, BQG_I4_ROW = 3 };
enum bqg_act { BQG_ACT_GELU_TANH = 1, BQG_ACT_SILU = 2 };

#define BQG_MAX_COLS 15360       /* largest cols (K) accepted by the GEMV and MoE calls     */
#define BQG_MAX_BATCH 256        /* largest descriptor count of one qgemv_batched call     */
#define BQG_MAX_EXPERTS 256      /* largest n_experts of the router / MoE calls            */
#define BQG_MAX_TOPK 8           /* largest k of the router / MoE calls                    */

/* Device-side error bits, reported by bqg_device_errors(). */
#define BQG_DEVERR_TIMEOUT 0x1   /* a bounded in-kernel wait gave up (the kernel returned early) */
#define BQG_DEVERR_EXPERT_ID 0x2 /* moe_forward met an expert id outside [0, n_experts); skipped */

/* Human-readable name of a bqg_status value (static string, never NULL). */
const char* bqg_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int bqg_version(void);

/* Byte size of a rows x cols matrix in the canonical layout of `fmt` (see above), or 0 when
 * the format is unknown or the shape is invalid (rows < 1, cols < 32 or cols % 32 != 0). */
size_t bqg_weight_bytes(int fmt, int rows, int cols);

/* Reads and clears the device-side error bits (BQG_DEVERR_*) of the current device.
 * Synchronises the device.  Returns BQG_OK or BQG_ERR_CUDA; *bits receives the bits. */
int bqg_device_errors(int* bits);

/* ---------------------------------------------------------------- a1, a2, a3: one GEMV
 * qgemv: y = W x for one quantized matrix.
 *   Source: Camelid README, "Engine status" (Q8_0) and "Gemma 4" (Q4_0 projection GEMVs);
 *   colibri wiki summary, "구현 범위" (packed int4 with per-row scale).
 *   fmt   BQG_Q8_0, BQG_Q4_0 or BQG_I4_ROW.
 *   W     device, bqg_weight_bytes(fmt, rows, cols) bytes, 16-byte aligned.
 *   x     device fp32 [cols], 16-byte aligned.   y  device fp32 [rows], 4-byte aligned.
 *   rows  >= 1.   cols  multiple of 32, 32 <= cols <= BQG_MAX_COLS.
 *   y must not overlap W or x.  Results are deterministic (fixed summation order). */
int qgemv(int fmt, const void* W, const float* x, float* y, int rows, int cols, void* stream);

/* ---------------------------------------------------------------- a4: a decode step's GEMVs
 * qgemv_batched: every descriptor's y = W x, in ONE persistent launch that streams all the
 * matrices back to back (the weight stream of one decode step).  The descriptors are
 * independent: no descriptor's y may be another descriptor's x (or overlap any W or x).
 *   Source: llama-modchip review, "개요" (decode time is the weight bytes per token);
 *   Camelid README, "Gemma 4" (captured decode graph of projection GEMVs).
 *   descs  HOST array of n descriptors, each obeying the qgemv preconditions.
 *   n      1 <= n <= BQG_MAX_BATCH. */
typedef struct {
  int fmt;
  int rows;
  int cols;
  int reserved; /* must be 0 */
  const void* W;
  const float* x;
  float* y;
} bqg_gemv_desc;

int qgemv_batched(const bqg_gemv_desc* descs, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BQG_H */
