// Host-side helpers shared by the Uno entry points.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "uno.h"

namespace uno_host {

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// UNO_OK when the current device is an sm_100 part (compute capability 10.0),
// UNO_ERR_DEVICE otherwise, UNO_ERR_CUDA when the runtime cannot say. The
// answer is cached per device ordinal.
int check_device();

}  // namespace uno_host
