// Device-side error words of the fp8q library: one per stream slot, zero at
// load.  A kernel records the first error it meets (e.g. a bounded wait
// that gave up) in the slot of the stream it was launched on, instead of
// trapping.  The host assigns slots 1..kStatusSlots-1 to streams in the
// order they first launch a GEMM; streams beyond that share slot 0.  The host
// reads one stream's word with fp8q_get_last_device_status and all of them
// with fp8q_device_status.
#pragma once

namespace fp8q {

constexpr int kStatusSlots = 256;

__device__ int g_stream_status[kStatusSlots];

__device__ __forceinline__ void record_error(int slot, int code) {
    atomicCAS(&g_stream_status[slot], 0, code);
}

}  // namespace fp8q
