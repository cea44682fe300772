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
 *   - Float outputs are fp32 (fp16 for the prefill GEMM).  The GEMV and MoE kernels hold each
 *     32 or 64 activation values as 16-bit fixed point with their own scale
 *     (|x - s X| <= max|x| / 65534), sum each block's products exactly in int32 and the blocks
 *     in fp32; the prefill GEMM multiplies fp16 operands with fp32 accumulation.
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
 *   BQG_I2_ROW row r = cols/4 bytes of two's-complement 2-bit values (weight 4j+k in bits
 *              2k..2k+1 of byte j: 0b00 = 0, 0b01 = 1, 0b10 = -2, 0b11 = -1); after all rows, zero
 *              padding to a 16-byte boundary, then one fp32 scale per row; cols % 64 == 0.
 *              Source: colibri wiki summary, "구현 범위" (packed int2 with a per-row scale).
 */
#ifndef BQG_H
#define BQG_H

#include <stddef.h>
#include <stdint.h>

/* Only the functions below are exported; everything else in the library has hidden visibility. */
#if defined(__GNUC__)
#define BQG_API __attribute__((visibility("default")))
#else
#define BQG_API
#endif

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

enum bqg_fmt { BQG_Q8_0 = 1, BQG_Q4_0 = 2, BQG_I4_ROW = 3, BQG_I2_ROW = 4 };
enum bqg_act { BQG_ACT_GELU_TANH = 1, BQG_ACT_SILU = 2 };

/* How moe_forward runs the experts (bqg_moe_layer.path).  Both compute the same layer.
 *   BQG_MOE_PATH_AUTO          the tensor cores (when the shapes allow it) from
 *                              BQG_MOE_TC_MIN_TOKENS tokens on; the CUDA cores otherwise.
 *   BQG_MOE_PATH_CUDA_CORES    grouped GEMV with integer dot products: every expert item is applied
 *                              to its tokens one at a time (best for 1..7 tokens).
 *   BQG_MOE_PATH_TENSOR_CORES  grouped expert GEMM on tcgen05: weights dequantized once into tensor
 *                              memory and multiplied by all the expert's tokens at once (prefill
 *                              chunks, decode batches).  Two variants:
 *                              - kind::i8 when every family (routed, and shared if present) is
 *                                BQG_I4_ROW or BQG_I2_ROW with hidden, inter and shared_inter
 *                                multiples of 128: weights as exact bytes, x and the gated hidden
 *                                values as 16-bit fixed point per row (two int8 digits), int32 sums;
 *                              - kind::f16 otherwise (Q8_0, Q4_0, int4; no int2): hidden, inter and
 *                                shared_inter multiples of 64, activations within the fp16 range.
 *                              Returns BQG_ERR_SHAPE when neither variant takes the layer. */
enum bqg_moe_path { BQG_MOE_PATH_AUTO = 0, BQG_MOE_PATH_CUDA_CORES = 1, BQG_MOE_PATH_TENSOR_CORES = 2 };
#define BQG_MOE_TC_MIN_TOKENS 8

#define BQG_MAX_COLS 15360       /* largest cols (K) of the GEMV, router and prefill calls  */
#define BQG_MAX_BATCH 256        /* largest descriptor count of one qgemv_batched call     */
#define BQG_MAX_EXPERTS 256      /* largest n_experts of the router / MoE calls            */
#define BQG_MAX_TOPK 8           /* largest k of the router / MoE calls                    */
#define BQG_MAX_MOE_COLS 7168    /* largest hidden / inter / shared_inter of moe_forward   */

/* Device-side error bits, reported by bqg_device_errors(). */
#define BQG_DEVERR_TIMEOUT 0x1   /* a bounded in-kernel wait gave up (the kernel returned early) */
#define BQG_DEVERR_EXPERT_ID 0x2 /* moe_forward met an expert id outside [0, n_experts); skipped */

/* Human-readable name of a bqg_status value (static string, never NULL).
 *   Source: Camelid README, "Why" and "At a glance" (the engine fails closed with typed errors
 *   instead of guessing); every call here returns one of the bqg_status values above. */
BQG_API const char* bqg_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
BQG_API int bqg_version(void);

/* Byte size of a rows x cols matrix in the canonical layout of `fmt` (see above), or 0 when
 * the format is unknown or the shape is invalid (rows < 1, cols < 32 or cols % 32 != 0). */
BQG_API size_t bqg_weight_bytes(int fmt, int rows, int cols);

/* Reads and clears the device-side error bits (BQG_DEVERR_*) of the current device.
 * Synchronises the device.  Returns BQG_OK or BQG_ERR_CUDA; *bits receives the bits. */
BQG_API int bqg_device_errors(int* bits);

/* ---------------------------------------------------------------- a1, a2, a3: one GEMV
 * qgemv: y = W x for one quantized matrix.
 *   Source: Camelid README, "Engine status" (Q8_0) and "Gemma 4" (Q4_0 projection GEMVs);
 *   colibri wiki summary, "구현 범위" (packed int4 with per-row scale).
 *   fmt   BQG_Q8_0, BQG_Q4_0, BQG_I4_ROW or BQG_I2_ROW (cols % 64 == 0).
 *   W     device, bqg_weight_bytes(fmt, rows, cols) bytes, 16-byte aligned.
 *   x     device fp32 [cols], 16-byte aligned.   y  device fp32 [rows], 4-byte aligned.
 *   rows  >= 1.   cols  multiple of 32, 32 <= cols <= BQG_MAX_COLS.
 *   y must not overlap W or x.  Results are deterministic (fixed summation order). */
BQG_API int qgemv(int fmt, const void* W, const float* x, float* y, int rows, int cols, void* stream);

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

BQG_API int qgemv_batched(const bqg_gemv_desc* descs, int n, void* stream);

/* ---------------------------------------------------------------- LM head with the greedy token
 * qgemv_argmax, qgemv_batched_argmax: the same GEMVs as qgemv / qgemv_batched, and in the same
 * launch the greedy token of one output vector: *token = the index of the largest value of y
 * (of descriptor argmax_index), values compared as IEEE floats (-0.0 == +0.0), an exact tie
 * going to the lower index; *max_value (optional) = that value.  The token is the argmax of the
 * fp32 y the call writes, bit for bit.
 *   Source: Camelid README, "At a glance" (the Apple Silicon path: GPU decode with on-GPU greedy
 *   sampling) and "Supported models" (the first token is the argmax of the head's logits).
 *   token      device int32 [1].   max_value  device fp32 [1], or NULL.
 *   state      device, 2 x uint64 (16 bytes, 8-byte aligned) of working state: zero it once
 *              before the first call (cudaMemset); every call that completes leaves it zero again.
 *              Calls sharing a state must be ordered (one stream); after a device error
 *              (bqg_device_errors) zero it again.
 *   Each CTA reduces the rows it wrote, then one 64-bit atomicMax per CTA merges them and the
 *   last CTA to finish writes the token: no extra launch, no extra pass over y.
 *   Finite y values are a precondition. */
BQG_API int qgemv_argmax(int fmt, const void* W, const float* x, float* y, int rows, int cols, int32_t* token,
                         float* max_value, unsigned long long* state, void* stream);
BQG_API int qgemv_batched_argmax(const bqg_gemv_desc* descs, int n, int argmax_index, int32_t* token,
                                 float* max_value, unsigned long long* state, void* stream);

/* ---------------------------------------------------------------- a11: prefill-chunk GEMM
 * qgemm_prefill: Y = X W^T with fp16 activations and Q4_0 weights on the tcgen05 tensor
 * cores (fp16 operands, fp32 accumulation in tensor memory, fp16 output, round to nearest).
 *   Source: TurboFieldfare wiki, "메모리·전문가 스트리밍" (prefill in chunks of at most 128
 *   tokens, each weight read reused by every prompt row of the chunk).
 *   fmt     BQG_Q4_0.
 *   W       device, bqg_weight_bytes(BQG_Q4_0, n, k) bytes, 16-byte aligned.
 *   X       device fp16 [tokens x k] row-major, 16-byte aligned.
 *   Y       device fp16 [tokens x n] row-major, 16-byte aligned.
 *   tokens  1..128.   n  >= 16, multiple of 16.   k  multiple of 256, 256 <= k <= BQG_MAX_COLS.
 *   Small n is split along k over a thread-block cluster (up to 8 CTAs) whose partial tiles are
 *   summed in a fixed order, so results are deterministic. */
BQG_API int qgemm_prefill(int fmt, const void* W, const void* X, void* Y, int tokens, int n, int k,
                  void* stream);

/* ---------------------------------------------------------------- a5: router logits
 * moe_router_logits: logits[t, e] = sum_h R[e, h] x[t, h] in fp32.
 *   Source: TurboFieldfare wiki, "메모리·전문가 스트리밍" (router choosing experts per token).
 *   R       device fp32 [n_experts x hidden], 16-byte aligned.
 *   x       device fp32 [tokens x hidden], 16-byte aligned.   logits  device fp32 [tokens x n_experts].
 *   tokens >= 1, 1 <= n_experts <= BQG_MAX_EXPERTS, hidden multiple of 4, 4 <= hidden <= BQG_MAX_COLS. */
BQG_API int moe_router_logits(const float* R, const float* x, float* logits, int tokens, int n_experts,
                      int hidden, void* stream);

/* ---------------------------------------------------------------- a6: softmax, top-k, renormalise
 * moe_router_topk: per token, idx[t, 0..k-1] = the k experts with the largest logits in
 * descending order, an exact tie going to the lower expert index; weights[t, j] =
 * p[idx[t, j]] / sum_j' p[idx[t, j']] with p = softmax(logits[t, :]) over all n_experts.
 *   Source: TurboFieldfare wiki, "메모리·전문가 스트리밍" (top-8 of 128); colibri wiki summary,
 *   "핵심 아이디어" (256 routed experts); Camelid README, "Windows bring-up, perf & GPU"
 *   (an exact expert-probability tie goes to the lower index).
 *   logits  device fp32 [tokens x n_experts] (finite values).
 *   idx     device int32 [tokens x k].   weights  device fp32 [tokens x k].
 *   tokens >= 1, 1 <= k <= BQG_MAX_TOPK, k <= n_experts <= BQG_MAX_EXPERTS. */
BQG_API int moe_router_topk(const float* logits, int tokens, int n_experts, int k, int32_t* idx,
                    float* weights, void* stream);

/* ---------------------------------------------------------------- a7-a10: the MoE layer
 * One routed-expert layer.  Expert e's gate matrix starts at gate + e * gate_stride bytes
 * (likewise up and down).  gate and up are [inter x hidden]; down is [hidden x inter]; all
 * three in expert_fmt.  The optional shared expert (s_gate == NULL means none) has
 * s_gate, s_up [shared_inter x hidden] and s_down [hidden x shared_inter] in shared_fmt.
 * act selects the gated activation for both: GeGLU with the tanh form of GELU, or SwiGLU. */
typedef struct {
  int n_experts;     /* 1..BQG_MAX_EXPERTS                          */
  int top_k;         /* 1..BQG_MAX_TOPK, <= n_experts               */
  int hidden;        /* multiple of 32, <= BQG_MAX_MOE_COLS         */
  int inter;         /* multiple of 32, <= BQG_MAX_MOE_COLS         */
  int expert_fmt;    /* BQG_Q8_0, BQG_Q4_0, BQG_I4_ROW or BQG_I2_ROW  */
  int act;           /* BQG_ACT_GELU_TANH or BQG_ACT_SILU           */
  const void* gate;  /* device, 16-byte aligned                      */
  const void* up;
  const void* down;
  size_t gate_stride; /* bytes between consecutive experts, multiple of 16 */
  size_t up_stride;
  size_t down_stride;
  int shared_inter;  /* multiple of 32, <= BQG_MAX_MOE_COLS (ignored without a shared expert) */
  int shared_fmt;
  const void* s_gate; /* NULL: no shared expert */
  const void* s_up;
  const void* s_down;
  int path;          /* BQG_MOE_PATH_*: which kernels run the experts (0 = choose by token count) */
} bqg_moe_layer;

/* Bytes of device workspace moe_forward needs for `tokens` tokens (0 on invalid arguments).
 *   Source: TurboFieldfare wiki, "메모리·전문가 스트리밍" (tokens are grouped by expert so that
 *   each expert read serves every row routed to it): the workspace holds that grouping (counts,
 *   offsets, the permutation of the (token, slot) pairs) and the per-pair intermediate rows.
 *   The caller allocates it once (PyTorch allocator or cudaMalloc) and may reuse it for every
 *   call with at most `tokens` tokens; its contents are scratch. */
BQG_API size_t moe_workspace_size(const bqg_moe_layer* L, int tokens);

/* moe_forward: y[t] = sum_{j<k} w[t, j] * FFN_{idx[t, j]}(x[t]) (+ shared FFN(x[t])), where
 * FFN(v) = down (act(gate v) * (up v)).  Tokens are grouped by expert on the device so that
 * each touched expert's weights are streamed once per call and applied to all its tokens.
 * The per-(token, slot) outputs are summed in slot order j = 0..k-1, then the shared output
 * is added, so results are deterministic.
 *   Source: Camelid README, "Gemma 4" (dense shared-expert + sparse top-8 branch); TurboFieldfare
 *   wiki, "메모리·전문가 스트리밍" (routed experts split from the shared branch, each expert read
 *   reused by every row routed to it).
 *   L          HOST pointer to the layer description.
 *   x          device fp32 [tokens x hidden], 16-byte aligned.
 *   idx, w     device int32 / fp32 [tokens x top_k] (as written by moe_router_topk).
 *   y          device fp32 [tokens x hidden], must not overlap x.
 *   workspace  device, >= moe_workspace_size(L, tokens) bytes, 256-byte aligned; contents
 *              are scratch, overwritten by the call.
 *   An expert id outside [0, n_experts) is skipped and sets BQG_DEVERR_EXPERT_ID. */
BQG_API int moe_forward(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w,
                float* y, int tokens, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- host-resident experts, device slot cache
 * An expert cache keeps a layer's routed experts in HOST memory (pinned, for asynchronous copies)
 * and the ones in use in n_slots device slots.  bqg_expert_cache_forward computes exactly
 * moe_forward's y for routing ids given on the host: it loads the missing experts into slots
 * (replacing the least frequently used slot that this call does not need, the least recently
 * used among equals) with cudaMemcpyAsync on copy_stream, runs the hit experts and the shared
 * expert on stream while those copies are in flight, then the missed experts once they have
 * landed, summed into the same y.
 *   Source: TurboFieldfare wiki, "메모리·전문가 스트리밍" (16 expert slots per layer, LFU with a
 *   recency tie-break, hits and misses split, loads overlapped with compute); Camelid README,
 *   "Supported models" (SSER: host-resident experts with an adaptive VRAM expert cache); colibri
 *   wiki summary, "구현 범위" (per-layer expert cache).
 * bqg_expert_cache_desc.layer describes the routed experts as in moe_forward, except that gate,
 * up and down are HOST pointers to the stacked experts (expert e at base + e * stride); the
 * optional shared expert's pointers are DEVICE pointers.  slot_gate / slot_up / slot_down are
 * DEVICE buffers of n_slots * {gate, up, down}_stride bytes (16-byte aligned), owned by the
 * caller.  The cache object itself is host memory allocated by bqg_expert_cache_create.
 *   - At most n_slots distinct experts per call (else BQG_ERR_LIMIT, nothing done).
 *   - idx_host: HOST int32 [tokens x top_k] routing ids (as written by moe_router_topk and copied
 *     to the host); w, x, y: device, as for moe_forward.
 *   - workspace: device, >= bqg_expert_cache_workspace_size(cache, tokens) bytes, 256-aligned.
 *   - Calls on one cache must be made from one host thread, in order, on the same two streams;
 *     the cache's bookkeeping is updated before the work is enqueued, so after an error destroy
 *     and re-create it. */
typedef struct {
  bqg_moe_layer layer;  /* routed experts on the HOST (gate, up, down), shared expert on the device */
  int n_slots;          /* device slots, 1 .. min(n_experts, BQG_MAX_EXPERTS) */
  void* slot_gate;      /* DEVICE n_slots * layer.gate_stride bytes */
  void* slot_up;        /* DEVICE n_slots * layer.up_stride bytes */
  void* slot_down;      /* DEVICE n_slots * layer.down_stride bytes */
} bqg_expert_cache_desc;

typedef struct {
  long long calls;        /* completed forward calls */
  long long hits;         /* distinct experts found in a slot, summed over calls */
  long long misses;       /* distinct experts loaded, summed over calls */
  long long evictions;    /* slots whose expert was replaced */
  long long bytes_copied; /* host-to-device bytes of the loads */
} bqg_expert_cache_stats;

typedef struct bqg_expert_cache bqg_expert_cache;

BQG_API int bqg_expert_cache_create(const bqg_expert_cache_desc* desc, bqg_expert_cache** cache);
BQG_API void bqg_expert_cache_destroy(bqg_expert_cache* cache);
BQG_API size_t bqg_expert_cache_workspace_size(const bqg_expert_cache* cache, int tokens);
BQG_API int bqg_expert_cache_forward(bqg_expert_cache* cache, const float* x, const int32_t* idx_host,
                                     const float* w, float* y, int tokens, void* workspace, size_t ws_bytes,
                                     void* stream, void* copy_stream);
BQG_API int bqg_expert_cache_get_stats(const bqg_expert_cache* cache, bqg_expert_cache_stats* stats);

/* ---------------------------------------------------------------- moe_forward without allocation
 * moe_forward_noalloc: the same computation as moe_forward, for callers that cannot allocate
 * device memory around the call (a CUDA graph captured by another component, a runtime that
 * forbids cudaMalloc after start-up, a plugin that only receives input and output buffers).
 * The pages describe no such call; it has no counterpart there.
 * Its scratch lives in a fixed array of BQG_NOALLOC_SCRATCH_BYTES inside the library image,
 * held by every GPU that loads the library until the process exits; the call allocates and
 * frees nothing.  Arguments are those of moe_forward without the workspace.
 *   - Returns BQG_ERR_LIMIT when moe_workspace_size(L, tokens) exceeds BQG_NOALLOC_SCRATCH_BYTES.
 *     32 MiB covers the Gemma-4-26B-A4B-like layer (hidden 2816, 128 experts, shared expert) up
 *     to 128 tokens (21.5 MB; 25.2 MB on the CUDA cores) and the GLM-like layer (hidden 6144, 256
 *     int4 experts of 2048) up to 64 tokens (25.2 MB); a GLM-like 128-token chunk (50 MB) does not
 *     fit.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current, and again after the device's context was destroyed and re-created
 *     (cudaDeviceReset); make that first call before any stream capture that includes it.
 *   - All calls on a device share the one array: calls that may overlap on the GPU (different
 *     streams without ordering between them) race and must not be issued.  Calls ordered on one
 *     stream are fine; the array keeps the last call's contents, and every region the kernels read
 *     is written first by the same call, so nothing needs clearing. */
#define BQG_NOALLOC_SCRATCH_BYTES (32u << 20)
BQG_API int moe_forward_noalloc(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w,
                                float* y, int tokens, void* stream);

/* ---------------------------------------------------------------- failure-detection self-test
 * bqg_selftest_wait_timeout: launches one kernel (one CTA) whose single mbarrier wait nothing
 * completes.  The wait is the bounded wait every kernel of the library uses: after 2 s it gives
 * up, sets BQG_DEVERR_TIMEOUT in the device error word and the kernel returns, so the context
 * stays usable.  Read (and clear) the bit with bqg_device_errors.  The pages describe no such
 * call; it shows that a stuck pipeline ends with a status instead of a hang.
 *   stream  CUDA stream (NULL: the default stream).  Returns BQG_OK once launched. */
BQG_API int bqg_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BQG_H */

