// Status strings, version and the device check of the Uno C ABI.
#include <atomic>

#include <cuda_runtime.h>

#include "uno.h"
#include "uno_host.h"

namespace uno_host {

int check_device() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];  // 0 unknown, 1 ok, 2 not sm_100
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return UNO_ERR_CUDA;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c == 1) return UNO_OK;
    if (c == 2) return UNO_ERR_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return UNO_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < kMaxDevices) cache[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok ? UNO_OK : UNO_ERR_DEVICE;
}

}  // namespace uno_host

extern "C" const char* uno_status_string(int status) {
  switch (status) {
    case UNO_OK: return "UNO_OK";
    case UNO_ERR_NULL: return "UNO_ERR_NULL: a required pointer is NULL";
    case UNO_ERR_SIZE: return "UNO_ERR_SIZE: a size is out of the supported range";
    case UNO_ERR_ALIGN: return "UNO_ERR_ALIGN: a pointer or row stride is not 16-byte aligned";
    case UNO_ERR_DTYPE: return "UNO_ERR_DTYPE: unknown dtype";
    case UNO_ERR_WORKSPACE: return "UNO_ERR_WORKSPACE: workspace missing or too small";
    case UNO_ERR_CUDA: return "UNO_ERR_CUDA: a CUDA call or kernel launch failed";
    case UNO_ERR_DEVICE: return "UNO_ERR_DEVICE: the current device is not an sm_100 GPU";
    default: return "UNO_ERR_UNKNOWN";
  }
}

extern "C" int uno_version(void) { return 100; }  // 0.1.0
