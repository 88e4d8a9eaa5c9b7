// Device helpers shared by the fp8q kernels (sm_100a).
//
// Numerics follow the method as the pages state it ("Size the per-tensor
// FP8 dynamic-quant amax grid to the input", Test Coverage: amax is an exact
// reduction and scale = amax / 448; "How to Profile DeepSeek-V3 Inference
// Kernels Using Triton Autotuning": block-wise quantisation to FP8 with
// per-block scales):
//   amax   = max |x| as an unsigned max over the 15-bit magnitude field of
//            the bf16 bit patterns.  For IEEE formats the magnitude order of
//            non-NaN values equals the unsigned order of these bits, and
//            every NaN sorts above +Inf, so the max is exact and NaN
//            propagates -- independent of the reduction order.
//   scale  = __fdiv_rn(amax, 448.f)           (one IEEE fp32 division)
//   code   = cvt.rn.satfinite.e4m3x2.f32(__fdiv_rn(x, scale))
//            (round to nearest even, saturate to +-448, NaN -> 0x7F)
//   scale == 0 (all-zero tensor or group): code = sign bit of x.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8q {

constexpr float kE4M3Max = 448.0f;

// bf16 bit patterns packed two per 32-bit word: element 2i in the low half.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Largest 15-bit magnitude field among the 8 bf16 values of a 16-byte vector.
__device__ __forceinline__ uint32_t absmax8(const uint4& v) {
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(v.x & m, v.y & m);
    uint32_t b = __vmaxu2(v.z & m, v.w & m);
    uint32_t c = __vmaxu2(a, b);
    return max(c & 0xFFFFu, c >> 16);
}

// fp32 value of a bf16 magnitude field produced by absmax8.
__device__ __forceinline__ float amax_bits_to_f32(uint32_t bits) {
    return __uint_as_float(bits << 16);
}

__device__ __forceinline__ float scale_from_amax(float amax) {
    return __fdiv_rn(amax, kE4M3Max);
}

// Two fp32 values -> two E4M3 codes; `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Codes of one bf16 pair under scale s (s != 0).
__device__ __forceinline__ uint32_t quant_pair(uint32_t w, float s) {
    return cvt_e4m3x2(__fdiv_rn(bf16_lo(w), s), __fdiv_rn(bf16_hi(w), s));
}

// Signed-zero codes of one bf16 pair (the zero-scale convention).
__device__ __forceinline__ uint32_t zero_pair(uint32_t w) {
    return ((w >> 8) & 0x80u) | ((w >> 16) & 0x8000u);
}

// Codes of 8 bf16 values (one 16-byte vector) -> 8 bytes.
__device__ __forceinline__ uint2 quant8(const uint4& v, float s) {
    uint2 r;
    if (s != 0.0f) {
        r.x = quant_pair(v.x, s) | (quant_pair(v.y, s) << 16);
        r.y = quant_pair(v.z, s) | (quant_pair(v.w, s) << 16);
    } else {
        r.x = zero_pair(v.x) | (zero_pair(v.y) << 16);
        r.y = zero_pair(v.z) | (zero_pair(v.w) << 16);
    }
    return r;
}

// Streaming global accesses: read-only, no L1 allocation; stores evict-first.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream8(void* p, const uint2& v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ uint32_t warp_max(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Max over a block of NT threads; every thread gets the result.
template <int NT>
__device__ __forceinline__ uint32_t block_max(uint32_t v, uint32_t* smem /* NT/32 words */) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) smem[w] = v;
    __syncthreads();
    uint32_t r = (l < NT / 32) ? smem[l] : 0u;
    return warp_max(r);
}

}  // namespace fp8q
