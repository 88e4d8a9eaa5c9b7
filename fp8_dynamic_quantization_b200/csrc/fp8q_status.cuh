// Device-side error word of the fp8q library (one per device, zero at load).
// Kernels record the first error they meet (e.g. a bounded wait that gave
// up) instead of trapping; the host reads it with fp8q_device_status().
#pragma once

namespace fp8q {

__device__ int g_device_status;

__device__ __forceinline__ void record_error(int code) {
    atomicCAS(&g_device_status, 0, code);
}

}  // namespace fp8q
