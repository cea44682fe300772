// libbqg.so — the single translation unit of the library (kernels + C ABI).
//
// Layout of the sources:
//   common.cuh       device helpers (mbarrier, bulk copies, bounded waits, error word)
//   host_common.h    host helpers (device checks, cached attributes)
//   qgemv.cuh        dequantize-fused GEMV kernel (single matrix and decode-step list)
//   qgemv_api.cuh    qgemv / qgemv_batched entry points
//   router.cuh       router logits and softmax/top-k/renormalise kernels + entry points
//   moe.cuh          grouped MoE layer kernels + moe_forward
//   prefill.cuh      tcgen05 prefill-chunk GEMM + qgemm_prefill
//   selftest.cuh     failure-detection self-test (a bounded wait that runs out)
#include "common.cuh"
#include "host_common.h"
#include "qgemv_api.cuh"
#include "router.cuh"
#include "moe_api.cuh"
#include "prefill.cuh"
#include "selftest.cuh"

extern "C" const char* bqg_status_string(int status) {
  switch (status) {
    case BQG_OK: return "BQG_OK";
    case BQG_ERR_ARG: return "BQG_ERR_ARG: null pointer, non-positive size or unknown enum value";
    case BQG_ERR_FMT: return "BQG_ERR_FMT: weight format not accepted by this call";
    case BQG_ERR_SHAPE: return "BQG_ERR_SHAPE: shape precondition violated";
    case BQG_ERR_ALIGN: return "BQG_ERR_ALIGN: pointer alignment precondition violated";
    case BQG_ERR_WORKSPACE: return "BQG_ERR_WORKSPACE: workspace missing or too small";
    case BQG_ERR_CUDA: return "BQG_ERR_CUDA: CUDA runtime call or kernel launch failed";
    case BQG_ERR_DEVICE: return "BQG_ERR_DEVICE: current device is not compute capability 10.0";
    case BQG_ERR_LIMIT: return "BQG_ERR_LIMIT: a documented maximum is exceeded";
    default: return "BQG: unknown status";
  }
}

extern "C" int bqg_version(void) { return 100; }

extern "C" int bqg_device_errors(int* bits) {
  if (bits == nullptr) return BQG_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return BQG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, bqg::g_dev_errors, sizeof(int)) != cudaSuccess) return BQG_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(bqg::g_dev_errors, &zero, sizeof(int)) != cudaSuccess) return BQG_ERR_CUDA;
  *bits = v;
  return BQG_OK;
}

// ---------------------------------------------------------------- moe_forward without allocation
// Some callers cannot allocate device memory around a call: code running inside a CUDA graph
// being captured by someone else, real-time or embedded runtimes that forbid cudaMalloc after
// start-up, and plugins handed only input and output buffers by a host framework that owns
// all allocations.  For them moe_forward_noalloc runs the same MoE kernels with their scratch
// (routing tables and per-pair intermediate rows) in the fixed array below, which is part of
// the library image: every GPU that loads the library holds these bytes until the process
// exits, and no call allocates or frees anything.
static __device__ __align__(256) uint8_t g_moe_noalloc_scratch[BQG_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_moe_noalloc_scratch per device.  In host code the array's name is only a
// host-side stand-in, so the address must be asked from the runtime (once per device).
std::atomic<void*> g_noalloc_scratch_ptr[bqg::kMaxDevices];
}  // namespace

extern "C" int moe_forward_noalloc(const bqg_moe_layer* L, const float* x, const int32_t* idx, const float* w,
                                   float* y, int tokens, void* stream) {
  const size_t need = moe_workspace_size(L, tokens);
  if (need == 0) {
    const int st = bqg::check_layer(L);
    return st != BQG_OK ? st : BQG_ERR_ARG;
  }
  if (need > size_t(BQG_NOALLOC_SCRATCH_BYTES)) return BQG_ERR_LIMIT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= bqg::kMaxDevices) return BQG_ERR_CUDA;
  void* scratch = g_noalloc_scratch_ptr[dev].load(std::memory_order_acquire);
  if (scratch == nullptr) {
    // first call on this device: look the array up with this device current
    if (cudaGetSymbolAddress(&scratch, g_moe_noalloc_scratch) != cudaSuccess || scratch == nullptr)
      return BQG_ERR_CUDA;
    g_noalloc_scratch_ptr[dev].store(scratch, std::memory_order_release);
  }
  // Every region of the scratch is written by the kernels before it is read, so nothing has to
  // be cleared between calls.
  return moe_forward(L, x, idx, w, y, tokens, scratch, size_t(BQG_NOALLOC_SCRATCH_BYTES), stream);
}
