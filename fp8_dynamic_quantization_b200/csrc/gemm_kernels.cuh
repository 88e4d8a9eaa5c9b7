// Block-scaled FP8 GEMM for sm_100a.
//
//   Y[m,n] = bf16( sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in kb} A[m,k] B[n,k] )
//
// ("How to Profile DeepSeek-V3 Inference Kernels Using Triton Autotuning":
// FP8 GEMM with per-block scaling, BLOCK_SIZE_K = 128, activation scales per
// 1x128 group and weight scales per 128x128 block.)
//
// The scales are arbitrary fp32 values, not powers of two, so the tensor
// cores cannot apply them: each 128-wide K block is multiplied into a fresh
// TMEM accumulator, and the promotion warps read that block's partial sum
// (tcgen05.ld), multiply it by sa*sb in fp32 and add it to an fp32 running
// sum held in registers.  Two TMEM buffers ping-pong so the MMA of block
// kb+1 overlaps the promotion of block kb.
//
// Warp roles (one CTA per SM, persistent over work units):
//   warp 0      TMA producer: P and Q tiles of one K block per pipeline stage
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (4 x K=32)
//   warps 2..   promotion / epilogue, 128 threads per 128 accumulator columns
//
// Operand roles.  The MMA computes D[128 rows, BN cols] = P * Q^T with P and
// Q K-major tiles in shared memory.
//   normal  (SWAP = false): P = A rows (m), Q = B rows (n).  Row scale
//           sa[m,kb]; column scale sb[n/128,kb] is uniform per 128 columns.
//   swapped (SWAP = true) : P = B rows (n), Q = A rows (m), for skinny M --
//           the weight fills the 128-row MMA dimension and the few tokens
//           become the MMA's N.  Row scale sb[n/128,kb] is uniform per tile;
//           column scales sa[m,kb] are staged in shared memory per unit.
// Split-K: a unit may cover a sub-range of K blocks; its fp32 partial goes
// to the workspace and splitk_reduce_kernel adds the splits in fixed order.
#pragma once

#include <cuda.h>
#include "ptx_sm100.cuh"
#include "fp8q_status.cuh"

namespace fp8q {

struct GemmParams {
    const float* sa;     // [M, G]
    const float* sb;     // [ceil(N/128), G]
    uint16_t* y;         // bf16 [M, ldy]
    float* ws;           // split-K partials [splits, M, ldw]
    int64_t ldy, ldw;
    int M, N, G;
    int tiles_p, tiles_q, splits, units;
};

template <int BN, bool SWAP, int STAGES>
struct GemmCfg {
    static constexpr int kEpiWG = BN > 128 ? 2 : 1;            // promotion warpgroups
    static constexpr int kCW = BN > 128 ? 128 : BN;            // columns per thread
    static constexpr int kThreads = 64 + 128 * kEpiWG;
    static constexpr int kPBytes = 128 * 128;                  // 128 rows x 128 K bytes
    static constexpr int kQBytes = BN * 128;
    static constexpr int kStageBytes = kPBytes + kQBytes;
    static constexpr int kTmemCols = (2 * BN) < 32 ? 32 : 2 * BN;
    static constexpr int kSlabFloats = SWAP ? (32768 / 4) : 0; // swapped-mode sa slab
    static constexpr size_t kSmemBytes = 1024 + size_t(STAGES) * kStageBytes
                                         + size_t(kSlabFloats) * 4 + 256;
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
    static_assert(!SWAP || BN <= 128, "swapped tiles hold at most 128 tokens");
};

__device__ __forceinline__ void unit_coords(const GemmParams& p, int u, int& tp, int& tq,
                                            int& kb0, int& kb1) {
    const int split = u % p.splits;
    const int tile = u / p.splits;
    tp = tile % p.tiles_p;
    tq = tile / p.tiles_p;
    kb0 = int((int64_t(split) * p.G) / p.splits);
    kb1 = int((int64_t(split + 1) * p.G) / p.splits);
}

template <int BN, bool SWAP, int STAGES>
__global__ void __launch_bounds__(GemmCfg<BN, SWAP, STAGES>::kThreads, 1)
block_gemm_kernel(const __grid_constant__ CUtensorMap tmP,
                  const __grid_constant__ CUtensorMap tmQ, const GemmParams p) {
    using C = GemmCfg<BN, SWAP, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = smem;                                        // STAGES x (P | Q)
    float* slab = reinterpret_cast<float*>(smem + size_t(STAGES) * C::kStageBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(
        smem + size_t(STAGES) * C::kStageBytes + size_t(C::kSlabFloats) * 4);
    uint64_t* full = bars;                   // [STAGES] TMA landed
    uint64_t* empty = bars + STAGES;         // [STAGES] MMA done reading
    uint64_t* tfull = bars + 2 * STAGES;     // [2] block partial ready in TMEM
    uint64_t* tempty = bars + 2 * STAGES + 2;// [2] promotion done reading TMEM
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { ptx::mbar_init(&full[s], 1); ptx::mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) { ptx::mbar_init(&tfull[b], 1); ptx::mbar_init(&tempty[b], 4 * C::kEpiWG); }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) { ptx::prefetch_tmap(&tmP); ptx::prefetch_tmap(&tmQ); }
    if (warp == 1) { ptx::tmem_alloc(tmem_base_smem, C::kTmemCols); ptx::tmem_relinquish(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;

    auto fail = [&]() { *abort_flag = 1; record_error(6 /* FP8Q_ERR_TIMEOUT */); };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int u = blockIdx.x; u < p.units && !*abort_flag; u += gridDim.x) {
                int tp, tq, kb0, kb1;
                unit_coords(p, u, tp, tq, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!ptx::mbar_wait(&empty[s], ph ^ 1)) { fail(); break; }
                    uint8_t* dst = tiles + size_t(s) * C::kStageBytes;
                    ptx::mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                    ptx::tma_load_2d(dst, &tmP, &full[s], kb * 128, tp * 128);
                    ptx::tma_load_2d(dst + C::kPBytes, &tmQ, &full[s], kb * 128, tq * BN);
                }
                if (*abort_flag) break;
            }
            if (*abort_flag) {
                // Let this thread's own copies land before the CTA exits.
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j)
                    ptx::mbar_wait(&full[j % STAGES], (j / STAGES) & 1, 100000000LL);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_e4m3_f32(BN);
            uint32_t it = 0, c = 0;
            for (int u = blockIdx.x; u < p.units && !*abort_flag; u += gridDim.x) {
                int tp, tq, kb0, kb1;
                unit_coords(p, u, tp, tq, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it, ++c) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    const uint32_t buf = c & 1, tph = (c >> 1) & 1;
                    if (!ptx::mbar_wait(&tempty[buf], tph ^ 1)) { fail(); break; }
                    if (!ptx::mbar_wait(&full[s], ph)) { fail(); break; }
                    ptx::tc_fence_after();
                    const uint32_t pa = ptx::smem_u32(tiles + size_t(s) * C::kStageBytes);
                    const uint32_t qa = pa + C::kPBytes;
                    const uint32_t d = tmem_base + buf * BN;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        ptx::mma_f8(d, ptx::sw128_kmajor_desc(pa + 32 * k),
                                    ptx::sw128_kmajor_desc(qa + 32 * k), idesc, k > 0);
                    ptx::mma_commit(&empty[s]);
                    ptx::mma_commit(&tfull[buf]);
                }
                if (*abort_flag) break;
            }
            if (*abort_flag && c > 0)
                ptx::mbar_wait(&tfull[(c - 1) & 1], ((c - 1) >> 1) & 1, 100000000LL);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ promotion
        const int e = warp - 2;                   // 0 .. 4*kEpiWG-1
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int chalf = e >> 2;                 // which 128-column half (BN = 256)
        const int row = quarter * 32 + lane;      // TMEM lane = tile row
        const int nthreads = 128 * C::kEpiWG;
        const int etid = threadIdx.x - 64;
        uint32_t c = 0;
        float acc[C::kCW];
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            int tp, tq, kb0, kb1;
            unit_coords(p, u, tp, tq, kb0, kb1);
            const int nkb = kb1 - kb0;
            // Scale sources for this unit.
            const int m_row = tp * 128 + row;                  // normal: token row
            const int n_row = tp * 128 + row;                  // swapped: weight row
            const int q0 = tq * BN;
            if (SWAP) {
                // slab[kbl * BN + j] = sa[q0 + j, kb0 + kbl]
                ptx::named_bar_sync(1, nthreads);
                for (int i = etid; i < nkb * BN; i += nthreads) {
                    const int kbl = i / BN, j = i - kbl * BN;
                    const int m = q0 + j;
                    slab[i] = (m < p.M) ? __ldg(p.sa + int64_t(m) * p.G + kb0 + kbl) : 0.0f;
                }
                ptx::named_bar_sync(1, nthreads);
            }
#pragma unroll
            for (int j = 0; j < C::kCW; ++j) acc[j] = 0.0f;

            // Scale of K block kb for this thread (normal mode) / tile (swapped).
            auto row_scale = [&](int kb) -> float {
                if (SWAP) return __ldg(p.sb + int64_t(tp) * p.G + kb);
                const int nb = (q0 + chalf * 128) >> 7;
                const float sbv = (nb * 128 < p.N) ? __ldg(p.sb + int64_t(nb) * p.G + kb) : 0.0f;
                const float sav = (m_row < p.M) ? __ldg(p.sa + int64_t(m_row) * p.G + kb) : 0.0f;
                return sav * sbv;
            };
            float s_next = row_scale(kb0);
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb, ++c) {
                const float s_cur = s_next;
                if (kb + 1 < kb1) s_next = row_scale(kb + 1);
                const uint32_t buf = c & 1, tph = (c >> 1) & 1;
                if (!ptx::mbar_wait(&tfull[buf], tph)) { fail(); ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16)
                                       + buf * BN + chalf * 128;
                const float* sl = slab + (kb - kb0) * BN;
                if (C::kCW >= 32) {
#pragma unroll
                    for (int cc = 0; cc < C::kCW / 32; ++cc) {
                        float v[32];
                        ptx::tmem_ld32(taddr + cc * 32, v);
                        ptx::tmem_wait_ld();
                        if (cc == C::kCW / 32 - 1) {
                            ptx::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float sj = SWAP ? s_cur * sl[cc * 32 + j] : s_cur;
                            acc[cc * 32 + j] = fmaf(v[j], sj, acc[cc * 32 + j]);
                        }
                    }
                } else {
                    float v[16];
                    ptx::tmem_ld16(taddr, v);
                    ptx::tmem_wait_ld();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float sj = SWAP ? s_cur * sl[j] : s_cur;
                        acc[j] = fmaf(v[j], sj, acc[j]);
                    }
                }
            }
            if (!ok) break;

            // ---------------------------------------------------- epilogue
            if (p.splits == 1) {
                if (!SWAP) {
                    const int m = m_row;
                    const int n_first = q0 + chalf * 128;
                    if (m < p.M) {
                        uint16_t* yr = p.y + int64_t(m) * p.ldy;
#pragma unroll
                        for (int j = 0; j < C::kCW; j += 8) {
                            const int n = n_first + j;
                            if (n + 8 <= p.N) {
                                uint4 w;
                                w.x = ptx::pack_bf16x2(acc[j + 0], acc[j + 1]);
                                w.y = ptx::pack_bf16x2(acc[j + 2], acc[j + 3]);
                                w.z = ptx::pack_bf16x2(acc[j + 4], acc[j + 5]);
                                w.w = ptx::pack_bf16x2(acc[j + 6], acc[j + 7]);
                                *reinterpret_cast<uint4*>(yr + n) = w;
                            } else {
#pragma unroll
                                for (int t = 0; t < 8; ++t)
                                    if (n + t < p.N)
                                        yr[n + t] = uint16_t(ptx::pack_bf16x2(acc[j + t], 0.0f) & 0xFFFF);
                            }
                        }
                    }
                } else {
                    const int n = n_row;
                    if (n < p.N) {
#pragma unroll
                        for (int j = 0; j < C::kCW; ++j) {
                            const int m = q0 + j;
                            if (m < p.M)
                                p.y[int64_t(m) * p.ldy + n] =
                                    uint16_t(ptx::pack_bf16x2(acc[j], 0.0f) & 0xFFFF);
                        }
                    }
                }
            } else {
                const int split = u % p.splits;
                float* wsp = p.ws + int64_t(split) * p.M * p.ldw;
                if (!SWAP) {
                    const int m = m_row;
                    const int n_first = q0 + chalf * 128;
                    if (m < p.M) {
                        float* wr = wsp + int64_t(m) * p.ldw;
#pragma unroll
                        for (int j = 0; j < C::kCW; j += 4) {
                            const int n = n_first + j;
                            if (n + 4 <= p.N) {
                                *reinterpret_cast<float4*>(wr + n) =
                                    make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
                            } else {
#pragma unroll
                                for (int t = 0; t < 4; ++t)
                                    if (n + t < p.N) wr[n + t] = acc[j + t];
                            }
                        }
                    }
                } else {
                    const int n = n_row;
                    if (n < p.N) {
#pragma unroll
                        for (int j = 0; j < C::kCW; ++j) {
                            const int m = q0 + j;
                            if (m < p.M) wsp[int64_t(m) * p.ldw + n] = acc[j];
                        }
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// Fixed-order sum of the split-K partials and conversion to bf16.
// Each thread handles 4 consecutive columns of one row.
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ ws, int splits, int M, int N, int64_t ldw,
                     uint16_t* __restrict__ y, int64_t ldy) {
    const int64_t cols4 = (N + 3) / 4;
    const int64_t total = int64_t(M) * cols4;
    for (int64_t i = int64_t(blockIdx.x) * 256 + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * 256) {
        const int64_t m = i / cols4;
        const int n = int(i - m * cols4) * 4;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (n + 4 <= N) {
            for (int s = 0; s < splits; ++s) {
                const float4 v = __ldcs(reinterpret_cast<const float4*>(
                    ws + (int64_t(s) * M + m) * ldw + n));
                a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
            }
            uint2 o;
            o.x = ptx::pack_bf16x2(a[0], a[1]);
            o.y = ptx::pack_bf16x2(a[2], a[3]);
            *reinterpret_cast<uint2*>(y + m * ldy + n) = o;
        } else {
            for (int s = 0; s < splits; ++s)
                for (int t = 0; t < 4 && n + t < N; ++t)
                    a[t] += ws[(int64_t(s) * M + m) * ldw + n + t];
            for (int t = 0; t < 4 && n + t < N; ++t)
                y[m * ldy + n + t] = uint16_t(ptx::pack_bf16x2(a[t], 0.0f) & 0xFFFF);
        }
    }
}

}  // namespace fp8q
