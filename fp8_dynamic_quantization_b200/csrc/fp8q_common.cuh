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
//   code   = cvt.rn.satfinite.e4m3x2.f32(RN(x / scale))
//            (round to nearest even, saturate to +-448, NaN -> 0x7F)
//   scale == 0 (all-zero tensor or group): code = sign bit of x.
//
// RN(x / scale) without a division per element: with r = RN(1/scale)
// (__frcp_rn, once per scale), q0 = RN(x*r), rem = x - q0*scale (one fma),
// q = fma(rem, r, q0), two values per f32x2 instruction (quant8_x2), the
// sign of each code then taken from x -- Markstein's correction step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).  Here x is a bf16 value and
// scale = RN(amax/448) with amax a bf16 value, so only 128 x 128 pairs of
// significands can occur; the quotient is scale-invariant in the normal
// range, and every pair was checked to give exactly RN(x/scale) (the test
// suite also compares every (x, amax) pair of bf16 bit patterns with the
// oracle's IEEE division on the GPU).  The scale must lie in [2^-90, 2^126]:
// then any quotient that can give a nonzero code (>= 2^-10) has |x| >=
// 2^-100, so the remainder is a normal number and exact, and smaller
// quotients stay below 2^-10 (a signed-zero code) even where a subnormal x
// makes the remainder inexact.  Other scales (tiny, infinite, NaN) and
// inputs above the amax (possible only when the caller supplies the amax)
// take __fdiv_rn instead.
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

// RN(1/448) in fp32.
constexpr float kInvE4M3Max = 0x1.24924ap-9f;

// scale = RN(amax / 448) from the amax's 15-bit bf16 magnitude field.  For
// finite amax the same reciprocal-corrected step as for the codes (with the
// constant r = RN(1/448)) gives RN(amax/448) exactly -- checked for all
// 32640 finite bf16 magnitudes, subnormals included; Inf and NaN take the
// IEEE division.
__device__ __forceinline__ float scale_from_amax_bits(uint32_t bits) {
    const float a = __uint_as_float(bits << 16);
    if (bits >= 0x7F80u) return __fdiv_rn(a, kE4M3Max);
    const float q0 = __fmul_rn(a, kInvE4M3Max);
    const float nrem = __fmaf_rn(q0, kE4M3Max, -a);
    return __fmaf_rn(-nrem, kInvE4M3Max, q0);
}


// Two fp32 values -> two E4M3 codes; `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Packed fp32 pairs: two fp32 values in one 64-bit register, for the
// sm_100 f32x2 arithmetic (one instruction for both lanes of the pair).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// A scale and what dividing by it needs.
struct Scale {
    float s;      // the scale
    float r;      // RN(1/s)
    int mode;     // 0: s == 0; 1: reciprocal-corrected division; 2: IEEE division
    uint64_t r2;  // (r, r) packed
    uint64_t ns2; // (-s, -s) packed
};

__device__ __forceinline__ Scale make_scale(float s) {
    Scale d;
    d.s = s;
    d.r = __frcp_rn(s);
    d.mode = (s == 0.0f) ? 0 : (s >= 0x1p-90f && s <= 0x1p126f) ? 1 : 2;
    d.r2 = f32x2(d.r, d.r);
    d.ns2 = f32x2(-s, -s);
    return d;
}

// Signed-zero codes of one bf16 pair (the zero-scale convention).
__device__ __forceinline__ uint32_t zero_pair(uint32_t w) {
    return ((w >> 8) & 0x80u) | ((w >> 16) & 0x8000u);
}

// Codes of 8 bf16 values for a scale in the reciprocal-corrected range
// (Scale::mode == 1) and values no larger than the amax, two values per
// instruction: q0 = RN(x*r) (an fma with -0 added, which is the product
// itself, signed zeros included), rem = RN(x - q0*s) (exact), q =
// RN(q0 + rem*r).  This is the step above with the remainder's sign
// flipped, which gives the same quotient for every x except x = -0, where
// it gives +0; so the sign bit of every code is then set from x itself (the
// sign of x / s is the sign of x for every x, zeros and underflows
// included).  Checked on the CPU for every bf16 x with |x| <= amax against
// RN(x / s) for every finite bf16 amax with s in the range above
// (1,031,103,648 pairs, codes equal), and on the GPU by the exhaustive
// (x, amax) test.
__device__ __forceinline__ uint2 quant8_x2(const uint4& v, uint64_t r2, uint64_t ns2) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint64_t nz2 = f32x2(-0.0f, -0.0f);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t x2 = f32x2(bf16_lo(w[i]), bf16_hi(w[i]));
        const uint64_t q0 = fma_f32x2(x2, r2, nz2);
        const uint64_t rem = fma_f32x2(q0, ns2, x2);
        float lo, hi;
        f32x2_split(fma_f32x2(rem, r2, q0), lo, hi);
        c[i] = cvt_e4m3x2(lo, hi);
    }
    uint2 r;
    r.x = (c[0] | (c[1] << 16)) | (__byte_perm(v.x, v.y, 0x7531) & 0x80808080u);
    r.y = (c[2] | (c[3] << 16)) | (__byte_perm(v.z, v.w, 0x7531) & 0x80808080u);
    return r;
}

// Codes of 8 bf16 values (one 16-byte vector) -> 8 bytes.  `exact` forces
// the IEEE division (for values that may exceed the amax).
__device__ __forceinline__ uint2 quant8(const uint4& v, const Scale& d, bool exact = false) {
    uint2 r;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
    if (d.mode == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) c[i] = zero_pair(w[i]);
    } else if (d.mode == 1 && !exact) {
        return quant8_x2(v, d.r2, d.ns2);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            c[i] = cvt_e4m3x2(__fdiv_rn(bf16_lo(w[i]), d.s), __fdiv_rn(bf16_hi(w[i]), d.s));
    }
    r.x = c[0] | (c[1] << 16);
    r.y = c[2] | (c[3] << 16);
    return r;
}

// ---------------------------------------------------------------------------
// ue8m0 scales: the scale is the smallest power of two 2^e >= amax/448 with
// e clamped to [-127, 127], stored as the E8M0 byte e + 127 (255 = NaN).
// For a normal bf16 amax = 1.f x 2^E, amax/448 = (1.f / 1.75) x 2^(E-8) and
// 1.f / 1.75 lies in [4/7, 1] when the 7-bit fraction field is at most 0x60
// (1.75) and in (1, 8/7) above it, so e = E - 8, plus 1 above 0x60.  Zero,
// subnormal and small amax clamp to e = -127; Inf and NaN give 255.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e8m0_from_amax_bits(uint32_t m) {
    if (m >= 0x7F80u) return 255u;
    const int E = int(m >> 7) - 127;
    const int e = max(E - 8 + ((m & 0x7Fu) > 0x60u ? 1 : 0), -127);
    return uint32_t(e + 127);
}

// 2^-(b-127) as fp32 (b <= 247 for any finite bf16 amax, so 254 - b >= 7:
// a normal number), NaN for b = 255.
__device__ __forceinline__ float e8m0_inverse(uint32_t b) {
    return b == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float((254u - b) << 23);
}

// Codes of 8 bf16 values for a power-of-two scale: e4m3_rne(x * 2^-e).  The
// product is exact unless it falls below 2^-126, where every candidate
// rounds to a signed-zero code anyway; |x| <= amax keeps it within +-448.
__device__ __forceinline__ uint2 quant8_pow2(const uint4& v, float inv) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = cvt_e4m3x2(__fmul_rn(bf16_lo(w[i]), inv), __fmul_rn(bf16_hi(w[i]), inv));
    uint2 r;
    r.x = c[0] | (c[1] << 16);
    r.y = c[2] | (c[3] << 16);
    return r;
}

// Streaming global accesses: read-only, no L1 allocation; stores evict-first.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
// L2 eviction priorities for the two passes of the per-tensor path over a
// tensor that fits in L2 several times over: the amax pass marks the lines
// it reads evict-last, so the apply pass finds them in L2, and the apply
// pass marks them evict-first as it reads them, so they do not crowd the
// next kernel's working set.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint4 ld_stream16_hint(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p), "l"(pol));
    return v;
}
// 32-byte read (16 bf16 values); the address must be 32-byte aligned.
__device__ __forceinline__ void ld_stream32(const void* p, uint4& a, uint4& b) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}
__device__ __forceinline__ void st_stream16(void* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_stream8(void* p, const uint2& v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// Programmatic dependent launch.  The library launches its kernels as
// programmatic dependents of the work before them on the stream: a kernel
// first lets its successor begin launching (its CTAs are placed as this
// kernel's CTAs retire), then waits until its predecessor has completed and
// that grid's writes are visible, before it touches global memory.  So the
// launch of each kernel overlaps the tail of the one before it, and stream
// order is kept.  Launched without the attribute, both are no-ops.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
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
