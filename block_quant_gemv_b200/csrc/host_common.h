// Host-side helpers shared by the C-ABI entry points: device capability checks, cached
// device attributes, argument checks.  Part of the single translation unit bqg.cu.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "bqg.h"

namespace bqg {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sm_count = 0;
  int cc_major = 0;
  int cc_minor = 0;
  std::atomic<bool> ready{false};  // the fields above are set (written once, under g_device_mutex)
};

inline DeviceInfo g_devices[kMaxDevices];
inline std::mutex g_device_mutex;

// Attributes of the current device (queried once per device; calls from several host threads
// are safe, and a failed query is retried by the next call).  Returns BQG_OK, BQG_ERR_CUDA or
// BQG_ERR_DEVICE (not compute capability 10.0).
inline int current_device(int* dev_out, DeviceInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BQG_ERR_CUDA;
  DeviceInfo& d = g_devices[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_device_mutex);
    if (!d.ready.load(std::memory_order_relaxed)) {
      int sm = 0, major = 0, minor = 0;
      if (cudaDeviceGetAttribute(&sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return BQG_ERR_CUDA;
      d.sm_count = sm;
      d.cc_major = major;
      d.cc_minor = minor;
      d.ready.store(true, std::memory_order_release);
    }
  }
  if (d.cc_major != 10 || d.cc_minor != 0) return BQG_ERR_DEVICE;
  *dev_out = dev;
  *info = &d;
  return BQG_OK;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BQG_OK : BQG_ERR_CUDA;
}

// Launch with programmatic stream serialization (dependent launch): the kernel may be
// scheduled before the previous kernel on the stream has finished, and waits for it with
// griddep_wait() before reading anything that kernel wrote.  Launch processing and the
// kernel's prologue then overlap the previous kernel's tail.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    (void)cudaGetLastError();
    return BQG_ERR_CUDA;
  }
  return launch_status();
}

// Per-device "dynamic shared memory attribute already set" flags for one kernel.
struct SmemAttrOnce {
  std::atomic<bool> done[kMaxDevices] = {};
  template <typename K>
  int ensure(int dev, K kernel, size_t bytes) {
    if (done[dev].load(std::memory_order_acquire)) return BQG_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) != cudaSuccess)
      return BQG_ERR_CUDA;
    done[dev].store(true, std::memory_order_release);
    return BQG_OK;
  }
};

}  // namespace bqg
