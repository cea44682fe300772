// libbqg.so — the single translation unit of the library (kernels + C ABI).
//
// Layout of the sources:
//   common.cuh       device helpers (mbarrier, bulk copies, bounded waits, error word)
//   host_common.h    host helpers (device checks, cached attributes)
//   qgemv.cuh        dequantize-fused GEMV kernel (single matrix and decode-step list)
//   qgemv_api.cuh    qgemv / qgemv_batched entry points
//   router.cuh       router logits and softmax/top-k/renormalise kernels + entry points
//   moe.cuh          grouped MoE layer kernels (CUDA cores)
//   moe_tc.cuh       grouped expert GEMM on tcgen05 (many tokens)
//   moe_api.cuh      moe_forward: workspace, path choice, launches
//   expert_cache.cuh host-resident experts with a device slot cache
//   prefill.cuh      tcgen05 prefill-chunk GEMM + qgemm_prefill
//   selftest.cuh     failure-detection self-test (a bounded wait that runs out)
#include "common.cuh"
#include "host_common.h"
#include "qgemv_api.cuh"
#include "router.cuh"
#include "moe_api.cuh"
#include "expert_cache.cuh"
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
// Device address of g_moe_noalloc_scratch per device, with the id of the CUDA context it was
// looked up in.  In host code the array's name is only a host-side stand-in, so the address is
// asked from the runtime with that device current: once per device (the first call), and again
// only if the device's context has been destroyed and re-created since (the module, and with it
// the array, may then sit at another address).
struct NoallocScratch {
  std::atomic<void*> ptr{nullptr};
  std::atomic<unsigned long long> ctx{0};
};
NoallocScratch g_noalloc_scratch[bqg::kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (false if the driver cannot tell).
bool current_context_id(unsigned long long* id) {
  static std::atomic<CtxGetCurrentFn> get_current{nullptr};
  static std::atomic<CtxGetIdFn> get_id{nullptr};
  CtxGetCurrentFn fc = get_current.load(std::memory_order_acquire);
  CtxGetIdFn fi = get_id.load(std::memory_order_acquire);
  if (fc == nullptr || fi == nullptr) {
    void* p1 = nullptr;
    void* p2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || p1 == nullptr || p2 == nullptr)
      return false;
    fc = reinterpret_cast<CtxGetCurrentFn>(p1);
    fi = reinterpret_cast<CtxGetIdFn>(p2);
    get_current.store(fc, std::memory_order_release);
    get_id.store(fi, std::memory_order_release);
  }
  CUcontext c = nullptr;
  return fc(&c) == CUDA_SUCCESS && c != nullptr && fi(c, id) == CUDA_SUCCESS;
}
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
  NoallocScratch& slot = g_noalloc_scratch[dev];
  // The first call on a device (and the first after its context was re-created) does the
  // set-up: make it before any stream capture that includes the call.
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  void* scratch = slot.ptr.load(std::memory_order_acquire);
  if (scratch == nullptr || (have_ctx && slot.ctx.load(std::memory_order_acquire) != ctx)) {
    if (cudaGetSymbolAddress(&scratch, g_moe_noalloc_scratch) != cudaSuccess || scratch == nullptr)
      return BQG_ERR_CUDA;
    slot.ctx.store(ctx, std::memory_order_release);
    slot.ptr.store(scratch, std::memory_order_release);
  }
  // Every region of the scratch is written by the kernels before it is read, so nothing has to
  // be cleared between calls.
  return moe_forward(L, x, idx, w, y, tokens, scratch, size_t(BQG_NOALLOC_SCRATCH_BYTES), stream);
}
