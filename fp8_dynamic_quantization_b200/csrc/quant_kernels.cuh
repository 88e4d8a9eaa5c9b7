// Quantisation kernels: bf16 -> E4M3 codes + fp32 scales (sm_100a).
//
// All of them are HBM-bound streaming kernels: 16-byte vector loads of 8
// bf16 values, several loads in flight per thread, grids sized to the input
// (never a fixed grid with idle blocks; compare "Size the per-tensor FP8
// dynamic-quant amax grid to the input", Description: a fixed 1024-block
// grid with a 1024-way atomic sets a data-independent floor).
//
//  group128_quant_kernel     one pass: amax of each 1x128 group, its scale,
//                            codes ("How to Profile DeepSeek-V3 Inference
//                            Kernels Using Triton Autotuning", Benchmarking
//                            the Activation Quantization Kernel).
//  amax_partial_kernel       per-tensor amax, one partial max per CTA.
//  apply_kernel              per-tensor apply pass: reduces the partials
//                            (or reads one amax word), computes the scale,
//                            writes codes.  Walks the tensor backwards, so
//                            the part of x the amax pass read last is still
//                            in L2 when it is read again.
//  per_tensor_fused_kernel   small tensors: one launch; values stay in
//                            registers across a bounded grid barrier.
//  block128_quant_kernel     128x128 weight blocks (offline step).
#pragma once

#include "fp8q_common.cuh"
#include "fp8q_status.cuh"

namespace fp8q {

constexpr int kQuantThreads = 256;

// Address of 16-byte vector `i` of a row-major [rows, vec_per_row*8] bf16
// matrix with row stride ld (elements).  CONTIG: ld == row length.
template <bool CONTIG>
__device__ __forceinline__ int64_t vec_offset(int64_t i, int64_t vec_per_row, int64_t ld) {
    if (CONTIG) return i * 8;
    const int64_t r = i / vec_per_row;
    return r * ld + (i - r * vec_per_row) * 8;
}

// ---------------------------------------------------------------------------
// Per-1x128-group quantisation.  8 threads own one group: thread `sub`
// holds its 16-byte chunks sub and sub+8 (16 values), so one load
// instruction of a warp covers four 128-byte runs, fully coalesced, and the
// per-group work (3 shuffles, the scale and its reciprocal) is shared by 16
// values per thread.  Each thread carries U groups per iteration (2U loads
// in flight).
// ---------------------------------------------------------------------------
template <int U, bool CONTIG>
__global__ void __launch_bounds__(kQuantThreads)
group128_quant_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                      uint8_t* __restrict__ q, int64_t ldq,
                      float* __restrict__ scales, int64_t groups, int64_t G) {
    const int sub = threadIdx.x & 7;
    const int64_t g_first = (int64_t(blockIdx.x) * kQuantThreads + threadIdx.x) >> 3;
    const int64_t g_stride = (int64_t(gridDim.x) * kQuantThreads) >> 3;
    // A warp owns groups 4w..4w+3 (g_stride is a multiple of 4), so testing
    // the first of them keeps the loop warp-uniform for the shuffles.
    for (int64_t g0 = g_first; (g0 & ~int64_t(3)) < groups; g0 += U * g_stride) {
        uint4 a[U], b[U];
        int64_t xo[U], qo[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = g0 + u * g_stride;
            if (CONTIG) {
                xo[u] = g * 128 + sub * 8;
                qo[u] = xo[u];
            } else {
                const int64_t r = g / G, c = g - r * G;
                xo[u] = r * ldx + c * 128 + sub * 8;
                qo[u] = r * ldq + c * 128 + sub * 8;
            }
            const bool ok = g < groups;
            a[u] = ok ? ld_stream16(x + xo[u]) : make_uint4(0, 0, 0, 0);
            b[u] = ok ? ld_stream16(x + xo[u] + 64) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = g0 + u * g_stride;
            uint32_t m = max(absmax8(a[u]), absmax8(b[u]));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            const Scale d = make_scale(scale_from_amax_bits(m));
            if (g < groups) {
                st_stream8(q + qo[u], quant8(a[u], d));
                st_stream8(q + qo[u] + 64, quant8(b[u], d));
                if (sub == 0) scales[g] = d.s;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Per-tensor amax: partial max per CTA into partials[blockIdx.x].
// ---------------------------------------------------------------------------
template <int U, bool CONTIG>
__global__ void __launch_bounds__(kQuantThreads)
amax_partial_kernel(const uint16_t* __restrict__ x, int64_t nvec, int64_t vec_per_row,
                    int64_t ldx, uint32_t* __restrict__ partials) {
    __shared__ uint32_t red[kQuantThreads / 32];
    const int64_t stride = int64_t(gridDim.x) * kQuantThreads;
    uint32_t m = 0;
    for (int64_t i0 = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x; i0 < nvec; i0 += U * stride) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            v[u] = (i < nvec) ? ld_stream16(x + vec_offset<CONTIG>(i, vec_per_row, ldx))
                              : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) m = max(m, absmax8(v[u]));
    }
    m = block_max<kQuantThreads>(m, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// ---------------------------------------------------------------------------
// Per-tensor apply: amax = max(partials[0:nparts]); scale; codes.
// ---------------------------------------------------------------------------
// CHECK: the amax comes from the caller, so a vector may hold values above
// it (or Inf); such vectors take the IEEE division.
template <int U, bool CONTIG, bool CHECK>
__global__ void __launch_bounds__(kQuantThreads)
apply_kernel(const uint16_t* __restrict__ x, int64_t nvec, int64_t vec_per_row, int64_t ldx,
             const uint32_t* __restrict__ partials, int nparts,
             uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ scale_out) {
    __shared__ uint32_t red[kQuantThreads / 32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < nparts; i += kQuantThreads)
        m = max(m, __ldcg(partials + i) & 0x7FFFu);
    m = block_max<kQuantThreads>(m, red);
    const Scale d = make_scale(scale_from_amax_bits(m));
    if (blockIdx.x == 0 && threadIdx.x == 0 && scale_out) *scale_out = d.s;

    const int64_t stride = int64_t(gridDim.x) * kQuantThreads;
    const int64_t span = U * stride;
    const int64_t first = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x;
    const int64_t iters = (nvec + span - 1) / span;
    for (int64_t it = iters - 1; it >= 0; --it) {       // backwards: L2 hits first
        const int64_t i0 = it * span + first;
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            v[u] = (i < nvec) ? ld_stream16(x + vec_offset<CONTIG>(i, vec_per_row, ldx))
                              : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < nvec) {
                const int64_t qo = CONTIG ? i * 8 : vec_offset<false>(i, vec_per_row, ldq);
                st_stream8(q + qo, quant8(v[u], d, CHECK && absmax8(v[u]) > m));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Per-tensor, single launch, for tensors that fit in the registers of a grid
// of at most one CTA per SM (all CTAs resident together).  Barrier state
// lives in the caller's workspace: ws[0] arrival count, ws[1] = generation
// (high 16 bits) | amax (low 16 bits), ws[2..] one partial max per CTA.
// Every CTA publishes its partial and arrives (acq_rel atomic); the last one
// reduces the partials, resets the count and publishes generation+1 with
// the amax (release); the others poll ws[1] (acquire) for at most
// `spin_cycles` SM clock cycles, after which they record FP8Q_ERR_TIMEOUT and
// return without writing outputs.  A one-CTA grid needs no barrier at all.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <int U, bool CONTIG>
__global__ void __launch_bounds__(kQuantThreads)
per_tensor_fused_kernel(const uint16_t* __restrict__ x, int64_t nvec, int64_t vec_per_row,
                        int64_t ldx, uint8_t* __restrict__ q, int64_t ldq,
                        float* __restrict__ scale_out, uint32_t* ws, int64_t spin_cycles) {
    __shared__ uint32_t red[kQuantThreads / 32];
    __shared__ uint32_t s_word;     // bit 31: timed out; bit 30: this CTA is last; low 16: amax
    const int64_t stride = int64_t(gridDim.x) * kQuantThreads;
    const int64_t first = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x;
    uint32_t gen0 = 0;
    if (gridDim.x > 1 && threadIdx.x == 0) gen0 = ld_relaxed_gpu(ws + 1) >> 16;

    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = first + u * stride;
        v[u] = (i < nvec) ? ld_stream16(x + vec_offset<CONTIG>(i, vec_per_row, ldx))
                          : make_uint4(0, 0, 0, 0);
    }
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) m = max(m, absmax8(v[u]));
    m = block_max<kQuantThreads>(m, red);

    uint32_t amax = m;
    if (gridDim.x > 1) {
        if (threadIdx.x == 0) {
            ws[2 + blockIdx.x] = m;
            const uint32_t arrived = atom_add_acq_rel_gpu(ws, 1u);
            uint32_t word = 0;
            if (arrived == gridDim.x - 1) {
                word = 1u << 30;
            } else {
                const long long t0 = clock64();
                uint32_t w1;
                while (((w1 = ld_acquire_gpu(ws + 1)) >> 16) == gen0) {
                    if (clock64() - t0 > spin_cycles) break;
                    __nanosleep(20);
                }
                word = ((w1 >> 16) == gen0) ? (1u << 31) : (w1 & 0xFFFFu);
                if (word >> 31) record_error(6 /* FP8Q_ERR_TIMEOUT */);
            }
            s_word = word;
        }
        __syncthreads();
        const uint32_t word = s_word;
        if (word >> 31) return;
        if (word & (1u << 30)) {
            // last CTA: reduce the partials, reset the count, publish
            uint32_t mm = 0;
            for (int i = threadIdx.x; i < int(gridDim.x); i += kQuantThreads)
                mm = max(mm, ld_relaxed_gpu(ws + 2 + i));
            mm = block_max<kQuantThreads>(mm, red);
            if (threadIdx.x == 0) {
                ws[0] = 0;
                st_release_gpu(ws + 1, (((gen0 + 1) & 0xFFFFu) << 16) | mm);
            }
            amax = mm;
        } else {
            amax = word & 0xFFFFu;
        }
    }
    const Scale d = make_scale(scale_from_amax_bits(amax));
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = d.s;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = first + u * stride;
        if (i < nvec) {
            const int64_t qo = CONTIG ? i * 8 : vec_offset<false>(i, vec_per_row, ldq);
            st_stream8(q + qo, quant8(v[u], d));
        }
    }
}

// out = max(partials[0:n]); one CTA.
__global__ void __launch_bounds__(kQuantThreads)
reduce_partials_kernel(const uint32_t* __restrict__ partials, int n, uint32_t* __restrict__ out) {
    __shared__ uint32_t red[kQuantThreads / 32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < n; i += kQuantThreads) m = max(m, __ldcg(partials + i));
    m = block_max<kQuantThreads>(m, red);
    if (threadIdx.x == 0) *out = m;
}

// scale = amax / 448 from an amax word, for an empty apply.
__global__ void scale_only_kernel(const uint32_t* __restrict__ amax_bits, float* __restrict__ scale) {
    if (threadIdx.x == 0) *scale = scale_from_amax_bits(*amax_bits & 0x7FFFu);
}

// ---------------------------------------------------------------------------
// 128x128 block quantisation of a weight W[N,K]: one CTA per block; each
// thread keeps its 8 vectors in registers between the amax and the apply.
// grid = (K/128, ceil(N/128)).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQuantThreads)
block128_quant_kernel(const uint16_t* __restrict__ w, int64_t N, int64_t ldw,
                      uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sb, int64_t G) {
    __shared__ uint32_t red[kQuantThreads / 32];
    const int64_t kb = blockIdx.x, nb = blockIdx.y;
    uint4 v[8];
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int j = threadIdx.x + u * kQuantThreads;       // 0..2047
        const int64_t r = nb * 128 + (j >> 4);
        const int c = (j & 15) * 8;
        v[u] = (r < N) ? ld_stream16(w + r * ldw + kb * 128 + c) : make_uint4(0, 0, 0, 0);
        m = max(m, absmax8(v[u]));
    }
    m = block_max<kQuantThreads>(m, red);
    const Scale d = make_scale(scale_from_amax_bits(m));
    if (threadIdx.x == 0) sb[nb * G + kb] = d.s;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int j = threadIdx.x + u * kQuantThreads;
        const int64_t r = nb * 128 + (j >> 4);
        const int c = (j & 15) * 8;
        if (r < N) st_stream8(q + r * ldq + kb * 128 + c, quant8(v[u], d));
    }
}

}  // namespace fp8q
