// status.cuh — the per-device status word the kernels report into.
//
// The whole library is one translation unit (mfp8.cu includes every kernel
// header), so this definition exists once; each device that loads the
// library holds its own copy.
#pragma once

#include "../../include/mfp8.h"

namespace mfp8 {

__device__ int g_device_status = 0;

// Keep the first error: later ones are usually consequences of it.
__device__ __forceinline__ void record_device_status(int code) {
    atomicCAS(&g_device_status, 0, code);
}

}  // namespace mfp8
