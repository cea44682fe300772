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
#include "common.cuh"
#include "host_common.h"
#include "qgemv_api.cuh"
#include "router.cuh"
#include "moe_api.cuh"

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
