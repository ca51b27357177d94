// Device-side status word shared by every kernel of the library.
//
// The library is built as one translation unit, so this single __device__
// word is visible to all kernels.  A kernel that gives up (a bounded wait ran
// out, or a device-side input check failed) stores the first error code here
// with atomicCAS and returns normally; the host reads and clears it through
// hstu_get_device_status().
#pragma once

#include <cstdint>

#include "../../include/hstu.h"

namespace hstu {

__device__ unsigned int g_device_status = 0;

__device__ __forceinline__ void record_status(hstu_status_t code) {
  atomicCAS(&g_device_status, 0u, static_cast<unsigned int>(code));
}

}  // namespace hstu
