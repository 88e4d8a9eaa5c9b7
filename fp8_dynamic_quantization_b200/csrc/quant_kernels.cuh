// Quantisation kernels: bf16 -> E4M3 codes + fp32 scales (sm_100a).
//
// All of them are HBM-bound streaming kernels: 16-byte vector loads of 8
// bf16 values (32-byte loads in group128_contig4_kernel), several loads in
// flight per thread, grids sized to the input
// (never a fixed grid with idle blocks; compare "Size the per-tensor FP8
// dynamic-quant amax grid to the input", Description: a fixed 1024-block
// grid with a 1024-way atomic sets a data-independent floor).
//
//  group128_contig4_kernel / one pass: amax of each 1x128 group, its scale,
//  group128_contig_kernel /  codes ("How to Profile DeepSeek-V3 Inference
//  group128_quant_kernel     Kernels Using Triton Autotuning", Benchmarking
//                            the Activation Quantization Kernel); the first
//                            for contiguous tensors with 32-byte aligned
//                            input and 16-byte aligned codes, the second for
//                            other contiguous tensors, the third for strided.
//  amax_contig_kernel /      per-tensor amax, one partial max per CTA
//  amax_partial_kernel       (contiguous / strided).
//  apply_contig_kernel /     per-tensor apply pass (contiguous / strided):
//  apply_kernel              reduces the partials
//                            (or reads one amax word), computes the scale,
//                            writes codes.  Walks the tensor backwards, so
//                            the part of x the amax pass read last is still
//                            in L2 when it is read again; a tensor of at most
//                            half the L2 is held there whole (evict-last
//                            reads in the amax pass, evict-first here).
//  per_tensor_cluster_kernel small tensors: one launch of one thread-block
//                            cluster; values stay in registers while the
//                            CTAs exchange partial maxima on chip.
//  per_channel_quant_kernel  one scale per row (a token, or an output
//                            channel of a weight).
//  block128_quant_kernel     128x128 weight blocks (offline step).
//  Both group and block kernels also have a ue8m0 form (E8 = true): the
//  scale is the smallest power of two >= amax/448, written as an E8M0 byte.
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
// E8: ue8m0 scales (E8M0 bytes in `scales`) instead of fp32 amax/448.
template <int U, bool CONTIG, bool E8 = false>
__global__ void __launch_bounds__(kQuantThreads)
group128_quant_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                      uint8_t* __restrict__ q, int64_t ldq,
                      void* __restrict__ scales, int64_t groups, int64_t G) {
    pdl_begin();   // a GEMM launched after this one may start its weight loads now
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
            if (E8) {
                const uint32_t sb = e8m0_from_amax_bits(m);
                const float inv = e8m0_inverse(sb);
                if (g < groups) {
                    st_stream8(q + qo[u], quant8_pow2(a[u], inv));
                    st_stream8(q + qo[u] + 64, quant8_pow2(b[u], inv));
                    if (sub == 0) static_cast<uint8_t*>(scales)[g] = uint8_t(sb);
                }
            } else {
                const Scale d = make_scale(scale_from_amax_bits(m));
                if (g < groups) {
                    st_stream8(q + qo[u], quant8(a[u], d));
                    st_stream8(q + qo[u] + 64, quant8(b[u], d));
                    if (sub == 0) static_cast<float*>(scales)[g] = d.s;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Per-tensor amax: partial max per CTA into partials[blockIdx.x].
// KEEP: the tensor fits in L2 with room to spare; its lines are read
// evict-last for the apply pass that follows.
// ---------------------------------------------------------------------------
template <int U, bool CONTIG, bool KEEP = false>
__global__ void __launch_bounds__(kQuantThreads)
amax_partial_kernel(const uint16_t* __restrict__ x, int64_t nvec, int64_t vec_per_row,
                    int64_t ldx, uint32_t* __restrict__ partials) {
    pdl_begin();
    __shared__ uint32_t red[kQuantThreads / 32];
    const int64_t stride = int64_t(gridDim.x) * kQuantThreads;
    const uint64_t pol = KEEP ? l2_policy_evict_last() : 0ull;
    uint32_t m = 0;
    for (int64_t i0 = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x; i0 < nvec; i0 += U * stride) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            const uint16_t* src = x + vec_offset<CONTIG>(i, vec_per_row, ldx);
            v[u] = (i < nvec) ? (KEEP ? ld_stream16_hint(src, pol) : ld_stream16(src)) : make_uint4(0, 0, 0, 0);
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
// it (or Inf); such vectors take the IEEE division.  KEEP: the amax pass
// kept the tensor in L2; read it evict-first (its last use).
template <int U, bool CONTIG, bool CHECK, bool KEEP = false>
__global__ void __launch_bounds__(kQuantThreads)
apply_kernel(const uint16_t* __restrict__ x, int64_t nvec, int64_t vec_per_row, int64_t ldx,
             const uint32_t* __restrict__ partials, int nparts,
             uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ scale_out) {
    pdl_begin();
    __shared__ uint32_t red[kQuantThreads / 32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < nparts; i += kQuantThreads)
        m = max(m, __ldcg(partials + i) & 0x7FFFu);
    m = block_max<kQuantThreads>(m, red);
    const Scale d = make_scale(scale_from_amax_bits(m));
    if (blockIdx.x == 0 && threadIdx.x == 0 && scale_out) *scale_out = d.s;

    const int64_t stride = int64_t(gridDim.x) * kQuantThreads;
    const uint64_t pol = KEEP ? l2_policy_evict_first() : 0ull;
    const int64_t span = U * stride;
    const int64_t first = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x;
    const int64_t iters = (nvec + span - 1) / span;
    for (int64_t it = iters - 1; it >= 0; --it) {       // backwards: L2 hits first
        const int64_t i0 = it * span + first;
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            const uint16_t* src = x + vec_offset<CONTIG>(i, vec_per_row, ldx);
            v[u] = (i < nvec) ? (KEEP ? ld_stream16_hint(src, pol) : ld_stream16(src)) : make_uint4(0, 0, 0, 0);
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
// Contiguous tensors (row stride == row length): the same passes over
// chunks of kQuantThreads x U consecutive 16-byte vectors.  Thread t of a
// CTA handles vectors t, t + 256, ... of its chunk, so every load and store
// of the chunk is one base pointer plus a constant offset, and only the
// last, partial chunk checks bounds; the grid strides over chunks.  This
// keeps the index arithmetic out of the per-vector work, which (with the
// per-element division) is what bounds these kernels when x is in L2.
// ---------------------------------------------------------------------------
template <int U, bool KEEP = false>
__global__ void __launch_bounds__(kQuantThreads)
amax_contig_kernel(const uint4* __restrict__ x, int64_t nvec, uint32_t* __restrict__ partials) {
    pdl_begin();
    __shared__ uint32_t red[kQuantThreads / 32];
    constexpr int kChunk = kQuantThreads * U;
    const uint64_t pol = KEEP ? l2_policy_evict_last() : 0ull;
    const int64_t nchunks = (nvec + kChunk - 1) / kChunk;
    uint32_t m = 0;
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
        const int64_t base = c * kChunk + threadIdx.x;
        const uint4* xp = x + base;
        uint4 v[U];
        if (c * kChunk + kChunk <= nvec) {
#pragma unroll
            for (int u = 0; u < U; ++u)
                v[u] = KEEP ? ld_stream16_hint(xp + u * kQuantThreads, pol) : ld_stream16(xp + u * kQuantThreads);
        } else {
#pragma unroll
            for (int u = 0; u < U; ++u)
                v[u] = base + u * kQuantThreads < nvec ? ld_stream16(xp + u * kQuantThreads) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) m = max(m, absmax8(v[u]));
    }
    m = block_max<kQuantThreads>(m, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// Apply pass over chunks, last chunk first (the amax pass read the end of
// the tensor last, so that part is the likeliest to be in L2).  CHECK and
// KEEP as in apply_kernel.
template <int U, bool CHECK, bool KEEP = false>
__global__ void __launch_bounds__(kQuantThreads)
apply_contig_kernel(const uint4* __restrict__ x, int64_t nvec, const uint32_t* __restrict__ partials,
                    int nparts, uint2* __restrict__ q, float* __restrict__ scale_out) {
    pdl_begin();
    __shared__ uint32_t red[kQuantThreads / 32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < nparts; i += kQuantThreads)
        m = max(m, __ldcg(partials + i) & 0x7FFFu);
    m = block_max<kQuantThreads>(m, red);
    const Scale d = make_scale(scale_from_amax_bits(m));
    if (blockIdx.x == 0 && threadIdx.x == 0 && scale_out) *scale_out = d.s;

    constexpr int kChunk = kQuantThreads * U;
    const uint64_t pol = KEEP ? l2_policy_evict_first() : 0ull;
    const int64_t nchunks = (nvec + kChunk - 1) / kChunk;
    const bool fast = d.mode == 1 && !CHECK;
    for (int64_t c = nchunks - 1 - blockIdx.x; c >= 0; c -= gridDim.x) {
        const int64_t base = c * kChunk + threadIdx.x;
        const uint4* xp = x + base;
        uint2* qp = q + base;
        if (c * kChunk + kChunk <= nvec) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                v[u] = KEEP ? ld_stream16_hint(xp + u * kQuantThreads, pol) : ld_stream16(xp + u * kQuantThreads);
            if (fast) {
#pragma unroll
                for (int u = 0; u < U; ++u) st_stream8(qp + u * kQuantThreads, quant8_x2(v[u], d.r2, d.ns2));
            } else {
#pragma unroll
                for (int u = 0; u < U; ++u)
                    st_stream8(qp + u * kQuantThreads, quant8(v[u], d, CHECK && absmax8(v[u]) > m));
            }
        } else {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (base + u * kQuantThreads < nvec) {
                    const uint4 v = ld_stream16(xp + u * kQuantThreads);
                    st_stream8(qp + u * kQuantThreads, quant8(v, d, CHECK && absmax8(v) > m));
                }
            }
        }
    }
}

// Per-1x128-group quantisation of a contiguous [M, K] tensor: chunks of
// U x 32 consecutive groups (8 threads per group as in
// group128_quant_kernel; lanes 8j..8j+7 of a warp own group 4w+j of each
// 32-group slice, so a warp's four groups are in or out of range together
// except in the last chunk).
template <int U, bool E8 = false>
__global__ void __launch_bounds__(kQuantThreads)
group128_contig_kernel(const uint4* __restrict__ x, uint2* __restrict__ q, void* __restrict__ scales,
                       int64_t groups) {
    pdl_begin();
    constexpr int kSlice = kQuantThreads / 8;               // groups per slice (32)
    constexpr int kChunk = kSlice * U;                      // groups per chunk
    const int sub = threadIdx.x & 7;
    const int gl = threadIdx.x >> 3;                        // group within a slice
    const int64_t nchunks = (groups + kChunk - 1) / kChunk;
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
        const int64_t g0 = c * kChunk + gl;                 // this thread's group in slice 0
        const uint4* xp = x + g0 * 16 + sub;                // a group is 16 vectors
        uint2* qp = q + g0 * 16 + sub;
        const bool full = c * kChunk + kChunk <= groups;
        uint4 a[U], b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool ok = full || g0 + u * kSlice < groups;
            a[u] = ok ? ld_stream16(xp + u * kSlice * 16) : make_uint4(0, 0, 0, 0);
            b[u] = ok ? ld_stream16(xp + u * kSlice * 16 + 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = g0 + u * kSlice;
            // a warp's four groups: test the first, so the shuffles stay warp-uniform
            if (!full && ((g - (gl & 3)) >= groups)) break;
            uint32_t m = max(absmax8(a[u]), absmax8(b[u]));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            if (!full && g >= groups) continue;
            if (E8) {
                const uint32_t sb = e8m0_from_amax_bits(m);
                const float inv = e8m0_inverse(sb);
                st_stream8(qp + u * kSlice * 16, quant8_pow2(a[u], inv));
                st_stream8(qp + u * kSlice * 16 + 8, quant8_pow2(b[u], inv));
                if (sub == 0) static_cast<uint8_t*>(scales)[g] = uint8_t(sb);
            } else {
                const Scale d = make_scale(scale_from_amax_bits(m));
                st_stream8(qp + u * kSlice * 16, quant8(a[u], d));
                st_stream8(qp + u * kSlice * 16 + 8, quant8(b[u], d));
                if (sub == 0) static_cast<float*>(scales)[g] = d.s;
            }
        }
    }
}

// Per-1x128-group quantisation of a contiguous [M, K] tensor with 4 threads
// per group and 32-byte loads: thread `sub` of a group reads its vectors
// 2sub, 2sub+1 and 8+2sub, 9+2sub (a warp's load covers 8 whole groups in
// 128-byte runs) and stores its codes 16 bytes at a time.  A CTA takes 64
// consecutive groups per iteration; a warp's 8 groups are in or out of range
// together except in the last chunk.  x must be 32-byte aligned, q 16-byte.
template <bool E8 = false>
__global__ void __launch_bounds__(kQuantThreads)
group128_contig4_kernel(const uint4* __restrict__ x, uint4* __restrict__ q, void* __restrict__ scales,
                        int64_t groups) {
    pdl_begin();
    constexpr int kChunk = kQuantThreads / 4;               // groups per chunk (64)
    const int sub = threadIdx.x & 3;
    const int gl = threadIdx.x >> 2;                        // group within a chunk
    const int64_t nchunks = (groups + kChunk - 1) / kChunk;
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
        const int64_t g = c * kChunk + gl;
        const bool full = c * kChunk + kChunk <= groups;
        // a warp's eight groups: test the first, so the shuffles stay warp-uniform
        if (!full && (g - (gl & 7)) >= groups) continue;
        const bool ok = full || g < groups;
        uint4 v[4];
        if (ok) {
            ld_stream32(x + g * 16 + 2 * sub, v[0], v[1]);  // a group is 16 vectors of 8 values
            ld_stream32(x + g * 16 + 8 + 2 * sub, v[2], v[3]);
        } else {
            v[0] = v[1] = v[2] = v[3] = make_uint4(0, 0, 0, 0);
        }
        uint32_t m = max(max(absmax8(v[0]), absmax8(v[1])), max(absmax8(v[2]), absmax8(v[3])));
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        if (!ok) continue;
        uint2 c0, c1, c2, c3;
        if (E8) {
            const uint32_t sb = e8m0_from_amax_bits(m);
            const float inv = e8m0_inverse(sb);
            c0 = quant8_pow2(v[0], inv); c1 = quant8_pow2(v[1], inv);
            c2 = quant8_pow2(v[2], inv); c3 = quant8_pow2(v[3], inv);
            if (sub == 0) static_cast<uint8_t*>(scales)[g] = uint8_t(sb);
        } else {
            const Scale d = make_scale(scale_from_amax_bits(m));
            c0 = quant8(v[0], d); c1 = quant8(v[1], d); c2 = quant8(v[2], d); c3 = quant8(v[3], d);
            if (sub == 0) static_cast<float*>(scales)[g] = d.s;
        }
        st_stream16(q + g * 8 + sub, make_uint4(c0.x, c0.y, c1.x, c1.y));      // codes: 8 vectors of 16
        st_stream16(q + g * 8 + 4 + sub, make_uint4(c2.x, c2.y, c3.x, c3.y));
    }
}

// ---------------------------------------------------------------------------
// Per-tensor, single launch, for tensors that fit in the registers of one
// thread-block cluster (up to 8 CTAs of NT threads, U vectors per thread;
// a single CTA is launched without a cluster and needs no exchange).  Each CTA reduces its values to one partial max in shared
// memory; after a cluster barrier every CTA reads all partials through
// distributed shared memory (mapa + ld.shared::cluster), so the whole amax
// exchange stays on chip.  A second barrier phase keeps each CTA's shared
// memory alive until every peer has read it.
// ---------------------------------------------------------------------------
constexpr int kClusterMax = 8;

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t ld_shared_cluster(const uint32_t* local, uint32_t rank) {
    uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local)), remote, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
    return v;
}

template <int U, bool CONTIG, int NT>
__global__ void __launch_bounds__(NT)
per_tensor_cluster_kernel(const uint16_t* __restrict__ x, int64_t nvec, int64_t vec_per_row,
                          int64_t ldx, uint8_t* __restrict__ q, int64_t ldq,
                          float* __restrict__ scale_out) {
    pdl_begin();
    constexpr int kClusterThreads = NT;
    __shared__ uint32_t red[kClusterThreads / 32];
    __shared__ uint32_t part;                     // this CTA's partial max
    const uint32_t crank = cluster_rank(), csize = cluster_nctarank();
    const int64_t stride = int64_t(csize) * kClusterThreads;
    const int64_t first = int64_t(crank) * kClusterThreads + threadIdx.x;

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
    m = block_max<kClusterThreads>(m, red);
    if (threadIdx.x == 0) part = m;
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
    uint32_t mm = 0;
    if (threadIdx.x < 32) {
        if (threadIdx.x < csize) mm = ld_shared_cluster(&part, threadIdx.x);
        mm = warp_max(mm);
    }
    // done reading the peers' shared memory
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    if (threadIdx.x == 0) red[0] = mm;
    __syncthreads();
    const Scale d = make_scale(scale_from_amax_bits(red[0]));
    if (crank == 0 && threadIdx.x == 0) *scale_out = d.s;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = first + u * stride;
        if (i < nvec) {
            const int64_t qo = CONTIG ? i * 8 : vec_offset<false>(i, vec_per_row, ldq);
            st_stream8(q + qo, quant8(v[u], d));
        }
    }
    // keep this CTA's shared memory until every peer has read it
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// out = max(partials[0:n]); one CTA.
__global__ void __launch_bounds__(kQuantThreads)
reduce_partials_kernel(const uint32_t* __restrict__ partials, int n, uint32_t* __restrict__ out) {
    pdl_begin();
    __shared__ uint32_t red[kQuantThreads / 32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < n; i += kQuantThreads) m = max(m, __ldcg(partials + i));
    m = block_max<kQuantThreads>(m, red);
    if (threadIdx.x == 0) *out = m;
}

// scale = amax / 448 from an amax word, for an empty apply.
__global__ void scale_only_kernel(const uint32_t* __restrict__ amax_bits, float* __restrict__ scale) {
    pdl_begin();
    if (threadIdx.x == 0) *scale = scale_from_amax_bits(*amax_bits & 0x7FFFu);
}

// ---------------------------------------------------------------------------
// Per-channel (per-row) quantisation: one CTA per row at a time.  A row of
// up to U*256*8 values stays in registers (one read of x); the CTA loads its
// next row before reducing the current one, so the loads of one row overlap
// the reduction and stores of the previous.  Longer rows take two passes,
// the second re-reading the row from L2 (at most a few thousand rows are in
// flight).  vpr = 16-byte vectors per row.
// ---------------------------------------------------------------------------
template <int U>
__global__ void __launch_bounds__(kQuantThreads)
per_channel_quant_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t vpr, int64_t ldx,
                         uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ scales) {
    pdl_begin();
    __shared__ uint32_t red[kQuantThreads / 32];
    if (vpr <= int64_t(U) * kQuantThreads) {
        uint4 cur[U], nxt[U];
        auto load = [&](int64_t r, uint4* v) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t j = threadIdx.x + int64_t(u) * kQuantThreads;
                v[u] = (r < M && j < vpr) ? ld_stream16(x + r * ldx + j * 8) : make_uint4(0, 0, 0, 0);
            }
        };
        int64_t r = blockIdx.x;
        load(r, cur);
        for (; r < M; r += gridDim.x) {
            load(r + gridDim.x, nxt);
            uint32_t m = 0;
#pragma unroll
            for (int u = 0; u < U; ++u) m = max(m, absmax8(cur[u]));
            m = block_max<kQuantThreads>(m, red);
            const Scale d = make_scale(scale_from_amax_bits(m));
            if (threadIdx.x == 0) scales[r] = d.s;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t j = threadIdx.x + int64_t(u) * kQuantThreads;
                if (j < vpr) st_stream8(q + r * ldq + j * 8, quant8(cur[u], d));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) cur[u] = nxt[u];
        }
        return;
    }
    for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
        const uint16_t* xr = x + r * ldx;
        uint32_t m = 0;
        for (int64_t i = threadIdx.x; i < vpr; i += 4 * kQuantThreads) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t j = i + u * kQuantThreads;
                v[u] = j < vpr ? ld_stream16(xr + j * 8) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) m = max(m, absmax8(v[u]));
        }
        m = block_max<kQuantThreads>(m, red);
        const Scale d = make_scale(scale_from_amax_bits(m));
        if (threadIdx.x == 0) scales[r] = d.s;
        uint8_t* qr = q + r * ldq;
        for (int64_t i = threadIdx.x; i < vpr; i += kQuantThreads)
            st_stream8(qr + i * 8, quant8(ld_stream16(xr + i * 8), d));
    }
}

// ---------------------------------------------------------------------------
// 128x128 block quantisation of a weight W[N,K]: one CTA per block; each
// thread keeps its 8 vectors in registers between the amax and the apply.
// grid = (K/128, ceil(N/128)).
// ---------------------------------------------------------------------------
template <bool E8 = false>   // E8: E8M0 scale bytes in `sb` (ue8m0 variant)
__global__ void __launch_bounds__(kQuantThreads)
block128_quant_kernel(const uint16_t* __restrict__ w, int64_t N, int64_t ldw,
                      uint8_t* __restrict__ q, int64_t ldq, void* __restrict__ sb, int64_t G) {
    pdl_begin();
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
    if (E8) {
        const uint32_t b = e8m0_from_amax_bits(m);
        const float inv = e8m0_inverse(b);
        if (threadIdx.x == 0) static_cast<uint8_t*>(sb)[nb * G + kb] = uint8_t(b);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = threadIdx.x + u * kQuantThreads;
            const int64_t r = nb * 128 + (j >> 4);
            const int c = (j & 15) * 8;
            if (r < N) st_stream8(q + r * ldq + kb * 128 + c, quant8_pow2(v[u], inv));
        }
        return;
    }
    const Scale d = make_scale(scale_from_amax_bits(m));
    if (threadIdx.x == 0) static_cast<float*>(sb)[nb * G + kb] = d.s;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int j = threadIdx.x + u * kQuantThreads;
        const int64_t r = nb * 128 + (j >> 4);
        const int c = (j & 15) * 8;
        if (r < N) st_stream8(q + r * ldq + kb * 128 + c, quant8(v[u], d));
    }
}

}  // namespace fp8q
