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
// TMEM accumulator buffer, and the promotion warps read that block's partial
// sum (tcgen05.ld), multiply it by sa*sb and add it to an fp32 running sum
// held in registers as packed pairs (fma.rn.f32x2 in place).  kNumBuf TMEM buffers rotate so
// the MMAs of the next K blocks overlap the promotion of this one.
//
// CTA pairs (PAIR): a cluster of two CTAs computes a 256 x BN tile with
// cta_group::2 MMAs issued by the leader; each CTA loads its own 128 rows of
// the P tile and half of the Q tile, and holds its 128 rows of every partial
// in its own TMEM.  Both CTAs promote; the peer's promotion warps hand TMEM
// buffers back by arriving on the leader's barriers.  With BN = 256 (TS) the
// epilogue converts the tile to bf16 into shared memory and bulk-stores it
// (cp.async.bulk.tensor), so the promotion warps return to the next tile's
// partials without waiting for the global stores.
//
// Warp roles (one CTA per SM, persistent over work units):
//   warpgroup 0   warp 0: TMA producer (P and Q tiles of one K block per
//                 pipeline stage); warp 1: TMEM allocation and the single
//                 thread that issues tcgen05.mma; warp 2: the ue8m0
//                 scale-slot writer (scale mode 2), otherwise idle; warp 3
//                 idle.  With several
//                 promotion warpgroups warpgroup 0 hands registers to them
//                 (setmaxnreg 40/232 or 56/216 for two, 32/160 for three).
//   warpgroups 1+ promotion / epilogue: thread = one TMEM lane (tile row)
//                 and a slice of kCW accumulator columns (128 for 256-wide
//                 tiles, else at most 64); warpgroup w-1 owns columns
//                 [(w-1)*kCW, w*kCW).  A thread loads its slice in chunks
//                 (48 + 80 columns for 128-column slices, else at most 64)
//                 and releases the TMEM buffer as soon as the last chunk
//                 has landed.
//
// Operand roles.  The MMA computes D[128 rows, BN cols] = P * Q^T with P and
// Q K-major tiles in shared memory (128-byte swizzle).
//   normal  (SWAP = false): P = A rows (m), Q = B rows (n).  Row scale
//           sa[m,kb]; column scale sb[n/128,kb] is uniform per 128 columns.
//           With SS the producer also copies each group of 4 K blocks'
//           scales (a 128 x 4 fp32 box of sa and the tile's sb rows) into
//           a shared-memory ring, so the promotion never waits on a global
//           load.
//   swapped (SWAP = true) : P = B rows (n), Q = A rows (m), for skinny M --
//           the weight fills the 128-row MMA dimension and the few tokens
//           become the MMA's N.  The per-column scale sa[m,kb]*sb[tile,kb]
//           is computed once per work unit into shared memory.
// Split-K: a unit may cover a sub-range of K blocks; its fp32 partial goes
// to the workspace and splitk_reduce_kernel adds the splits in fixed order.
// Split tail (normal and pair tiles): when the tiles leave a last wave that
// would occupy only a few SMs, the first full_tiles tiles run whole and each
// of the remaining tail tiles is split into tail_splits K ranges, so the
// last wave is short and fills the SMs; those partials go to the workspace
// (tile-local [unit][tile rows][BN] fp32) and tail_reduce_kernel adds them
// in fixed order into Y.
// Programmatic dependent launch: every GEMM is launched as a programmatic
// dependent of the previous kernel on the stream; its prologue (barriers,
// TMEM allocation, tensor-map prefetch) overlaps that kernel's tail, and
// every thread waits for it (griddepcontrol.wait) before touching global
// memory.  With p.pdl set (the previous kernel writes only A and sa), the
// producer first issues the weight halves of its first STAGES stages.

// Scale mode SM:
//   0  fp32 block scales, promoted per K block as above.
//   1  per-tensor scales (the GEMM of the per-tensor dynamic path): sa and
//      sb are single fp32 values, so the MMAs accumulate a unit's whole K
//      range into one TMEM buffer and the epilogue multiplies by sa*sb once.
//   2  ue8m0 block scales (E8M0 bytes sa [M, G], sb [ceil(N/128), G]): the
//      tensor cores apply them (tcgen05.mma kind::mxf8f6f4.block_scale), so
//      again one TMEM accumulation per unit and no promotion.  Per group of 4
//      K blocks warp 2 writes the tile's scale bytes into a
//      shared-memory slot laid out as 32 rows x 16 bytes per 128 rows
//      (row j holds rows j, 32+j, 64+j, 96+j, four K blocks each); the MMA
//      warp copies each such block to TMEM with tcgen05.cp 32x128b.warpx4,
//      which replicates it into all four lane quarters -- the layout the
//      block-scaled MMA reads: A row m at lane m, column base + m/32; B row n
//      at column base + n/32 in every lane quarter; the byte picked by the
//      instruction's scale-factor id, here kb % 4.
//   3  per-channel scales (sa [M] per row of A, sb [N] per row of B): one
//      TMEM accumulation per unit; the epilogue multiplies row m by its
//      scale and column n by the one staged for the tile in shared memory.
#pragma once

#include <cuda.h>
#include "fp8q_common.cuh"
#include "ptx_sm100.cuh"
#include "fp8q_status.cuh"

namespace fp8q {

struct GemmParams {
    const float* sa;     // [M, G]
    const float* sb;     // [ceil(N/128), G]
    uint16_t* y;         // bf16 [M, ldy]
    float* ws;           // split-K partials [splits, M, ldw], or the split tail's
    int64_t ldy, ldw;
    int M, N, G;
    int tiles_p, splits, units;
    int full_units;      // units [0, full_units): tiles x splits; the rest are split-tail units
    int full_tiles;      // tiles before the split tail
    int tail_splits;     // K ranges per tail tile; their partials go to ws as [unit - full_units][tile rows][BN]
    // Flags as bytes and no field the kernel does not read: the struct is
    // passed by value to every launch, and growing it from 120 to 136
    // bytes measurably slowed the kernel (2%).
    uint8_t scale_vec4;  // sa/sb rows readable as float4 (G % 4 == 0, 16-byte aligned)
    uint8_t sf_words;    // ue8m0: 4 scale bytes readable as one word (G % 4 == 0, 4-byte aligned)
    uint8_t pdl;         // the weights do not depend on the previous kernel (it produces A and sa)
    uint8_t status_slot; // error word of the launching stream (g_stream_status index)
    uint8_t ystore;      // TS tiles: Y has a tensor map (tmY) for bulk stores from shared memory
    long long wait_budget;  // SM clock cycles a barrier wait may take before giving up
};
static_assert(sizeof(GemmParams) <= 104, "GemmParams size");

template <int BN, bool SWAP, int STAGES, bool PAIR = false, int SM = 0, bool SS = false>
struct GemmCfg {
    static constexpr bool PT = SM == 1;                        // per-tensor scales
    static constexpr bool MX = SM == 2;                        // ue8m0 scales applied by the MMA
    static constexpr bool PC = SM == 3;                        // per-channel scales
    // BN is the MMA's N.  PAIR: a CTA pair computes a 256 x BN tile with
    // cta_group::2 MMAs; each CTA holds 128 rows of A and BN/2 rows of B,
    // and its TMEM receives its 128 rows x BN columns of every product.
    static constexpr int kCW = BN == 256 ? 128 : (BN < 64 ? BN : 64);  // columns per promotion thread
    static constexpr int kEpiWG = BN / kCW;                    // promotion warpgroups (1..3)
    static constexpr int kThreads = 128 + 128 * kEpiWG;
    // Register split (setmaxnreg) between warpgroup 0 and the promotion
    // warpgroups; it must add up to at most threads x launch registers.
    static constexpr int kRegWG0 = kEpiWG == 2 ? (kCW == 128 ? 40 : 56) : 32;
    static constexpr int kRegEpi = kEpiWG == 2 ? (kCW == 128 ? 232 : 216) : 160;
    static constexpr int kLaunchRegs = ((65536 / kThreads) / 8) * 8 > 255 ? 255 : ((65536 / kThreads) / 8) * 8;
    static_assert(kEpiWG == 1 || 128 * kRegWG0 + 128 * kEpiWG * kRegEpi <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    static_assert(kEpiWG <= 3, "at most three promotion warpgroups");
    static constexpr int kTileRows = PAIR ? 256 : 128;         // rows of P per work unit
    // TS: the epilogue of whole tiles converts Y to bf16 into a shared-memory
    // tile (each promotion warp its 32 rows x kCW columns, 128-byte
    // swizzled) and bulk-stores it, so the promotion warps go back to the
    // next tile's partials without waiting for the global stores.
    static constexpr bool TS = PAIR && BN == 256 && (SM == 0 || SM == 1 || SM == 3);
    static constexpr int kYBytes = TS ? 128 * BN * 2 : 0;
    static constexpr int kPBytes = 128 * 128;                  // 128 rows x 128 K bytes
    static constexpr int kQRows = PAIR ? BN / 2 : BN;         // B (or A) rows this CTA loads
    static constexpr int kQBytes = kQRows * 128;
    static constexpr int kStageBytes = kPBytes + kQBytes;
    // MX keeps TMEM columns [448, 512) for four scale-factor slots of 16
    // columns (B scales at +0..7, A scales at +8..11).
    static constexpr int kSfSlots = MX ? 4 : 0;
    static constexpr int kSfCol0 = 448;
    static constexpr int kSfSlotBytes = 3 * 512;               // A block, B rows 0-127, B rows 128-255
    static constexpr int kDataCols = MX ? kSfCol0 : 512;
    static constexpr int kNumBuf = (kDataCols / BN) < 8 ? (kDataCols / BN) : 8;
    static constexpr int kTmemCols = MX ? 512 : kNumBuf * BN <= 32 ? 32 : kNumBuf * BN <= 64 ? 64
                                   : kNumBuf * BN <= 128 ? 128 : kNumBuf * BN <= 256 ? 256 : 512;
    static constexpr int kMaxUnitKb = 64;                      // K blocks per unit (swapped mode)
    // swapped-mode scale slab (block scales); per-channel: the tile's column scales
    static constexpr int kSlabFloats = (SWAP && SM == 0) ? BN * kMaxUnitKb : PC ? BN : 0;
    // SS: block scales staged through shared memory.  The producer copies,
    // per group of 4 K blocks, the tile's 128 x 4 row scales and its
    // BN/128 x 4 column-block scales into a ring of kScaleSlots slots.
    static constexpr int kScaleSlots = SS ? 4 : 0;
    static constexpr int kSbRows = BN / 128;                   // column blocks per tile (SS)
    static constexpr int kScaleSlotBytes = 2048 + 128;         // 128 x 4 fp32, then kSbRows x 4 fp32
    static constexpr uint32_t kScaleTx = 2048 + 16 * kSbRows;  // bytes one slot receives
    static constexpr size_t kSmemBytes = 1024 + size_t(STAGES) * kStageBytes + size_t(kYBytes)
                                         + size_t(kSlabFloats) * 4 + size_t(kScaleSlots) * kScaleSlotBytes
                                         + size_t(kSfSlots) * kSfSlotBytes + 512;
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN");
    static_assert(kCW % 16 == 0, "columns per thread");
    static_assert(!SWAP || BN <= 128, "swapped tiles hold at most 128 tokens");
    // normal mode: each 64-column promotion slice starts at a multiple of 64,
    // so it lies inside one 128-column weight-scale block (uniform scale)
    static_assert(SWAP || kCW == 64 || kCW == 128, "normal-mode slices are 64 or 128 columns");
    static_assert(!PAIR || (!SWAP && (BN == 256 || BN == 128)), "CTA pairs compute 256 x 256 or 256 x 128 tiles");
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert((2 * STAGES + 2 * kNumBuf + 2 * kScaleSlots + 2 * kSfSlots) * 8 + 8 <= 512, "barrier area");
    static_assert(!SS || (!SWAP && !PAIR && SM == 0 && (BN == 128 || BN == 256)), "staged scales: normal 128/256 tiles");
    static_assert(!MX || (!PAIR && kNumBuf >= 1), "ue8m0 tiles: one CTA, at least one TMEM buffer");
};

__device__ __forceinline__ void unit_coords(const GemmParams& p, int u, int& tp, int& tq,
                                            int& kb0, int& kb1) {
    int split, tile, splits;
    if (u < p.full_units) {
        splits = p.splits;
        split = u % splits;
        tile = u / splits;
    } else {                                   // split tail
        splits = p.tail_splits;
        const int v = u - p.full_units;
        split = v % splits;
        tile = p.full_tiles + v / splits;
    }
    tp = tile % p.tiles_p;
    tq = tile / p.tiles_p;
    kb0 = int((int64_t(split) * p.G) / splits);
    kb1 = int((int64_t(split + 1) * p.G) / splits);
}

// Accumulators are kept as packed fp32 pairs: acc2[i] holds columns 2i and
// 2i+1, so the packed fma.rn.f32x2 works on them in place.

// acc2[j/2] += (v[j], v[j+1]) * (s, s) for j in [0, N).
template <int N>
__device__ __forceinline__ void fma_uniform(uint64_t* acc2, const float* v, uint64_t s2) {
#pragma unroll
    for (int j = 0; j < N; j += 2) ptx::fma2p(acc2[j / 2], v[j], v[j + 1], s2);
}

// acc2[j/2] += (v[j], v[j+1]) * (sl[j], sl[j+1]), scales from shared memory.
template <int N>
__device__ __forceinline__ void fma_columns(uint64_t* acc2, const float* v, const float* sl) {
#pragma unroll
    for (int j = 0; j < N; j += 2)
        ptx::fma2p(acc2[j / 2], v[j], v[j + 1], *reinterpret_cast<const uint64_t*>(sl + j));
}

// Scales of 4 consecutive K blocks [4*g4, 4*g4+4) of one scale row
// (zeros past G or for an absent row).
__device__ __forceinline__ float4 load_scale4(const float* row, int g4, int G, bool vec4, bool valid) {
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    const int k0 = 4 * g4;
    if (!valid || k0 >= G) return r;
    if (vec4) return __ldg(reinterpret_cast<const float4*>(row + k0));
    r.x = __ldg(row + k0);
    if (k0 + 1 < G) r.y = __ldg(row + k0 + 1);
    if (k0 + 2 < G) r.z = __ldg(row + k0 + 2);
    if (k0 + 3 < G) r.w = __ldg(row + k0 + 3);
    return r;
}

__device__ __forceinline__ float pick4(const float4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Epilogue stores.  A promotion thread holds one tile row, so storing rows
// directly makes each warp store touch 32 rows in 16-byte pieces.  Within
// each group of 8 lanes (8 rows), an 8 x 8 transpose of 16-byte chunks
// (three butterfly stages of shuffles) turns a[k] = chunk k of this lane's
// row into a[k] = chunk g8 of row (group base + k); store k then writes
// that row's 8 chunks (128 contiguous bytes) from the 8 lanes, and a warp
// store covers 4 whole row segments.  All 32 lanes must call it.
__device__ __forceinline__ void transpose8x8(uint4 (&a)[8], int g8) {
#pragma unroll
    for (int sft = 4; sft >= 1; sft >>= 1) {
        const bool up = (g8 & sft) != 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k & sft) continue;
            const uint4 snd = up ? a[k] : a[k | sft];
            uint4 rcv;
            rcv.x = __shfl_xor_sync(0xFFFFFFFFu, snd.x, sft);
            rcv.y = __shfl_xor_sync(0xFFFFFFFFu, snd.y, sft);
            rcv.z = __shfl_xor_sync(0xFFFFFFFFu, snd.z, sft);
            rcv.w = __shfl_xor_sync(0xFFFFFFFFu, snd.w, sft);
            if (up) a[k] = rcv;
            else a[k | sft] = rcv;
        }
    }
}

// ue8m0 mode: E8M0 bytes of K blocks [4g, 4g+4) for one 128-row block of
// the P operand (is_p) or the Q operand, packed 4 per word (K block 4g+b in
// byte b); rows, blocks and K blocks out of range give 127 (scale 1).
template <int BN, bool SWAP>
__device__ __forceinline__ uint32_t sf_word(const GemmParams& p, bool is_p, int tp, int tq, int row, int g) {
    const uint8_t* sa = reinterpret_cast<const uint8_t*>(p.sa);   // [M, G]
    const uint8_t* sb = reinterpret_cast<const uint8_t*>(p.sb);   // [ceil(N/128), G]
    int64_t base = -1;                                            // byte offset of K block 0
    if (is_p) {
        if (!SWAP) { const int m = tp * 128 + row; if (m < p.M) base = int64_t(m) * p.G; }
        else base = int64_t(tp) * p.G;                            // one weight block per P tile
    } else {
        if (!SWAP) { const int n = tq * BN + row; if (row < BN && n < p.N) base = int64_t(n >> 7) * p.G; }
        else { const int m = tq * BN + row; if (row < BN && m < p.M) base = int64_t(m) * p.G; }
    }
    const uint8_t* src = (is_p != SWAP) ? sa : sb;
    if (p.sf_words) {                       // K blocks 4g..4g+3 are bytes 0..3 of one aligned word
        return base >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(src + base + 4 * g)) : 0x7F7F7F7Fu;
    }
    uint32_t w = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int kb = 4 * g + b;
        const uint32_t v = (base >= 0 && kb < p.G) ? uint32_t(__ldg(src + base + kb)) : 127u;
        w |= v << (8 * b);
    }
    return w;
}

// One scale slot: the A block (P rows) and ceil(BN/128) B blocks, each 32
// rows x 16 bytes; lane j writes row j of every block.
template <int BN, bool SWAP>
__device__ __forceinline__ void build_sf_slot(uint8_t* dst, const GemmParams& p, int lane, int tp, int tq, int g) {
    uint4 a;
    a.x = sf_word<BN, SWAP>(p, true, tp, tq, lane, g);
    a.y = sf_word<BN, SWAP>(p, true, tp, tq, 32 + lane, g);
    a.z = sf_word<BN, SWAP>(p, true, tp, tq, 64 + lane, g);
    a.w = sf_word<BN, SWAP>(p, true, tp, tq, 96 + lane, g);
    *reinterpret_cast<uint4*>(dst + lane * 16) = a;
#pragma unroll
    for (int blk = 0; blk < (BN + 127) / 128; ++blk) {
        uint4 b;
        b.x = sf_word<BN, SWAP>(p, false, tp, tq, 128 * blk + lane, g);
        b.y = sf_word<BN, SWAP>(p, false, tp, tq, 128 * blk + 32 + lane, g);
        b.z = sf_word<BN, SWAP>(p, false, tp, tq, 128 * blk + 64 + lane, g);
        b.w = sf_word<BN, SWAP>(p, false, tp, tq, 128 * blk + 96 + lane, g);
        *reinterpret_cast<uint4*>(dst + 512 * (1 + blk) + lane * 16) = b;
    }
}

template <int BN, bool SWAP, int STAGES, bool PAIR = false, int SM = 0, bool SS = false>
__global__ void __launch_bounds__(GemmCfg<BN, SWAP, STAGES, PAIR, SM, SS>::kThreads, 1)
block_gemm_kernel(const __grid_constant__ CUtensorMap tmP,
                  const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmSA,    // row scales [M, G] fp32 (SS only)
                  const __grid_constant__ CUtensorMap tmSB,    // column-block scales [NB, G] fp32 (SS only)
                  const __grid_constant__ CUtensorMap tmY,     // bf16 Y [M, N], 64 x 32 boxes (TS with p.ystore)
                  const GemmParams p) {
    using C = GemmCfg<BN, SWAP, STAGES, PAIR, SM, SS>;
    constexpr bool PT = C::PT, MX = C::MX, PC = C::PC;
    constexpr bool ONE = PT || MX || PC;  // one TMEM accumulation per unit, no per-K-block promotion
    constexpr int NB = C::kNumBuf;
    // Per-K-block promotion (block scales): the MMA's commit to empty[s]
    // also tells the promotion warps that K block `it`'s partial is in TMEM,
    // and the promotion warps hand a TMEM buffer back by arriving on the
    // full barrier of the K block that will reuse it (it + NB).  So the
    // MMA thread waits once and commits once per K block.
    constexpr bool MERGED = !ONE;
    constexpr uint32_t kRelease = (PAIR ? 2u : 1u) * 4u * C::kEpiWG;   // promotion warps arriving per release
    static_assert(!MERGED || NB <= STAGES, "a TMEM buffer is reused within the stage ring");
    constexpr uint32_t kSlots = C::kScaleSlots > 0 ? C::kScaleSlots : 1;   // divisor for the (SS) slot ring
    constexpr uint32_t kSfN = C::kSfSlots > 0 ? C::kSfSlots : 1;         // divisor for the (MX) slot ring
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = smem;                                        // STAGES x (P | Q)
    uint8_t* ytile = smem + size_t(STAGES) * C::kStageBytes;      // TS: bf16 Y tile, 8 KB per promotion warp
    float* slab = reinterpret_cast<float*>(ytile + C::kYBytes);
    uint8_t* sring = ytile + C::kYBytes + size_t(C::kSlabFloats) * 4;   // SS slots
    uint8_t* sfring = sring + size_t(C::kScaleSlots) * C::kScaleSlotBytes;   // MX scale-factor slots
    uint64_t* bars = reinterpret_cast<uint64_t*>(sfring + size_t(C::kSfSlots) * C::kSfSlotBytes);
    uint64_t* full = bars;                        // [STAGES] TMA landed
    uint64_t* empty = bars + STAGES;              // [STAGES] MMA done reading
    uint64_t* tfull = bars + 2 * STAGES;          // [NB] block partial ready in TMEM
    uint64_t* tempty = bars + 2 * STAGES + NB;    // [NB] promotion done reading TMEM
    uint64_t* sfull = bars + 2 * STAGES + 2 * NB;  // [kScaleSlots] scale slot landed (SS)
    uint64_t* sempty = sfull + C::kScaleSlots;     // [kScaleSlots] scale slot read by every promotion warp
    uint64_t* sffull = sempty + C::kScaleSlots;   // [kSfSlots] scale-factor slot written (MX)
    uint64_t* sfempty = sffull + C::kSfSlots;     // [kSfSlots] slot consumed by the MMAs (MX)
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(sfempty + C::kSfSlots);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    ptx::griddep_launch_dependents();    // the next kernel on the stream may begin launching
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA pair: rank 0 (the leader) issues the MMAs; both load, both promote.
    const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit0 = PAIR ? int(ptx::cluster_id_x()) : int(blockIdx.x);
    const int unit_step = PAIR ? int(ptx::num_clusters_x()) : int(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&full[s], MERGED ? 1 + kRelease : 1);
            ptx::mbar_init(&empty[s], 1);
        }
        if (MERGED)              // the first NB K blocks find their TMEM buffer free
            for (int j = 0; j < NB; ++j)
                for (uint32_t a = 0; a < kRelease; ++a) ptx::mbar_arrive(&full[j]);
        for (int b = 0; b < NB; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], (PAIR ? 2 : 1) * 4 * C::kEpiWG);
        }
        for (int i = 0; i < C::kScaleSlots; ++i) {
            ptx::mbar_init(&sfull[i], 1);
            ptx::mbar_init(&sempty[i], 4 * C::kEpiWG);
        }
        for (int i = 0; i < C::kSfSlots; ++i) {
            ptx::mbar_init(&sffull[i], 1);
            ptx::mbar_init(&sfempty[i], 1);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmP);
        ptx::prefetch_tmap(&tmQ);
        if (SS) { ptx::prefetch_tmap(&tmSA); ptx::prefetch_tmap(&tmSB); }
    }
    if (warp == 1) {
        if (PAIR) { ptx::tmem_alloc_pair(tmem_base_smem, C::kTmemCols); ptx::tmem_relinquish_pair(); }
        else { ptx::tmem_alloc(tmem_base_smem, C::kTmemCols); ptx::tmem_relinquish(); }
    }
    ptx::tc_fence_before();
    if (PAIR) ptx::cluster_sync();      // the peer may signal the leader's barriers from here on
    else __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;
    // Nothing above touched global memory.  Wait for the previous kernel on
    // the stream (programmatic dependent launch) before anything does; only
    // the producer of a launch whose weights do not depend on that kernel
    // (p.pdl) issues the weight loads of its first stages before it waits.
    const bool early_weights = !PAIR && SM == 0 && p.pdl && warp == 0 && lane == 0;
    if (!early_weights) ptx::griddep_wait();

    auto fail = [&]() { *abort_flag = 1; record_error(p.status_slot, 6 /* FP8Q_ERR_TIMEOUT */); };

    if (warp < 4) {
        if (C::kEpiWG > 1) ptx::regs_dec<C::kRegWG0>();
        if (MX && warp == 2) {
            // ------------------------------------ scale-slot writer (ue8m0)
            // All lanes write one slot per group of 4 K blocks, in the order
            // the MMA warp consumes them; wait results are broadcast from
            // lane 0 so the warp stays converged and stops together.
            uint32_t sg = 0;
            bool stop = false;
            for (int u = unit0; u < p.units && !stop; u += unit_step) {
                int tp, tq, kb0, kb1;
                unit_coords(p, u, tp, tq, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (kb != kb0 && (kb & 3) != 0) continue;
                    const uint32_t slot = sg % kSfN, sph = (sg / kSfN) & 1;
                    bool ok = true;
                    if (lane == 0) ok = ptx::mbar_wait(&sfempty[slot], sph ^ 1, p.wait_budget);
                    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                    if (!ok) { if (lane == 0) fail(); stop = true; break; }
                    __syncwarp();
                    build_sf_slot<BN, SWAP>(sfring + size_t(slot) * C::kSfSlotBytes, p, lane, tp, tq, kb >> 2);
                    ptx::fence_proxy_async_shared();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sffull[slot]);
                    ++sg;
                }
            }
            __syncwarp();
        } else if (warp == 0 && lane == 0) {
            // -------------------------------------------------------- producer
            // PDL: the weights do not depend on the previous kernel, so the
            // weight halves of the first STAGES stages go out before waiting
            // for it; the token halves (and all scales) follow the wait.
            uint32_t pre = 0;
            if (!PAIR && SM == 0 && p.pdl) {
                for (int u = unit0; u < p.units && pre < uint32_t(STAGES); u += unit_step) {
                    int tp, tq, kb0, kb1;
                    unit_coords(p, u, tp, tq, kb0, kb1);
                    for (int kb = kb0; kb < kb1 && pre < uint32_t(STAGES); ++kb, ++pre) {
                        uint8_t* dst = tiles + size_t(pre) * C::kStageBytes;
                        ptx::mbar_arrive_expect_tx(&full[pre], C::kStageBytes);
                        if (SWAP) ptx::tma_load_2d(dst, &tmP, &full[pre], kb * 128, tp * C::kTileRows);
                        else ptx::tma_load_2d(dst + C::kPBytes, &tmQ, &full[pre], kb * 128, tq * BN);
                    }
                }
                ptx::griddep_wait();
            }
            uint32_t it = 0;
            uint32_t sg = 0;             // scale groups issued (SS)
            bool stop = false;
            for (int u = unit0; u < p.units && !*abort_flag && !stop; u += unit_step) {
                int tp, tq, kb0, kb1;
                unit_coords(p, u, tp, tq, kb0, kb1);
                const int prow = tp * C::kTileRows + int(rank) * 128;
                const int qrow = tq * BN + int(rank) * C::kQRows;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    if (SS && (kb == kb0 || (kb & 3) == 0)) {
                        // scales of K blocks [4*(kb/4), 4*(kb/4)+4): x is a multiple of 4 fp32
                        const uint32_t slot = sg % kSlots, sph = (sg / kSlots) & 1;
                        if (!ptx::mbar_wait(&sempty[slot], sph ^ 1, p.wait_budget)) { fail(); stop = true; break; }
                        uint8_t* sdst = sring + size_t(slot) * C::kScaleSlotBytes;
                        ptx::mbar_arrive_expect_tx(&sfull[slot], C::kScaleTx);
                        ptx::tma_load_2d(sdst, &tmSA, &sfull[slot], (kb >> 2) * 4, prow);
                        ptx::tma_load_2d(sdst + 2048, &tmSB, &sfull[slot], (kb >> 2) * 4, tq * C::kSbRows);
                        ++sg;
                    }
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (it < pre) {                       // weight half already issued (PDL)
                        uint8_t* dst = tiles + size_t(s) * C::kStageBytes;
                        if (SWAP) ptx::tma_load_2d(dst + C::kPBytes, &tmQ, &full[s], kb * 128, qrow);
                        else ptx::tma_load_2d(dst, &tmP, &full[s], kb * 128, prow);
                        continue;
                    }
                    if (!ptx::mbar_wait(&empty[s], ph ^ 1, p.wait_budget)) { fail(); stop = true; break; }
                    uint8_t* dst = tiles + size_t(s) * C::kStageBytes;
                    if (PAIR) {
                        // both CTAs' copies complete on the leader's barrier
                        const uint32_t bar0 = ptx::mapa_shared(ptx::smem_u32(&full[s]), 0);
                        if (leader) ptx::mbar_arrive_expect_tx(&full[s], 2 * C::kStageBytes);
                        ptx::tma_load_2d_pair(dst, &tmP, bar0, kb * 128, prow);
                        ptx::tma_load_2d_pair(dst + C::kPBytes, &tmQ, bar0, kb * 128, qrow);
                    } else {
                        ptx::mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                        ptx::tma_load_2d(dst, &tmP, &full[s], kb * 128, prow);
                        ptx::tma_load_2d(dst + C::kPBytes, &tmQ, &full[s], kb * 128, qrow);
                    }
                }
            }
            if (*abort_flag && leader) {
                // Let this thread's own copies land before the CTA exits.
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j)
                    ptx::mbar_wait(&full[j % STAGES], (j / STAGES) & 1, 100000000LL);
                const uint32_t sfirst = sg > uint32_t(C::kScaleSlots) ? sg - C::kScaleSlots : 0;
                for (uint32_t g = sfirst; g < sg; ++g)
                    ptx::mbar_wait(&sfull[g % kSlots], (g / kSlots) & 1, 100000000LL);
            }
        } else if (warp == 1 && lane == 0 && leader) {
            // -------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = ptx::idesc_e4m3_f32(BN, C::kTileRows);
            uint32_t it = 0, c = 0;
            uint32_t sgm = 0, sf_slot = 0, sf_col = 0;   // scale-factor slots (MX)
            bool failed = false;
            // the most recent commit (a commit arrives once every MMA issued
            // before it has finished): what an abort must wait for
            uint64_t* last_bar = nullptr;
            uint32_t last_parity = 0;
            for (int u = unit0; u < p.units && !failed; u += unit_step) {
                int tp, tq, kb0, kb1;
                unit_coords(p, u, tp, tq, kb0, kb1);
                // One promotion step = one K block (block scales), or the
                // whole K range of the unit (per-tensor scales: the MMAs
                // accumulate every K block into one TMEM buffer).
                const int steps = ONE ? 1 : kb1 - kb0;
                int kb = kb0;
                for (int st = 0; st < steps && !failed; ++st, ++c) {
                    const uint32_t buf = c % NB, tph = (c / NB) & 1;
                    if (!MERGED) {          // merged: the full wait below covers the buffer
                        const bool freed = PAIR ? ptx::mbar_wait_cluster(&tempty[buf], tph ^ 1, p.wait_budget)
                                                : ptx::mbar_wait(&tempty[buf], tph ^ 1, p.wait_budget);
                        if (!freed) { fail(); failed = true; break; }
                    }
                    const uint32_t d = tmem_base + buf * BN;
                    const int kb_end = ONE ? kb1 : kb + 1;
                    for (; kb < kb_end; ++kb, ++it) {
                        if (MX && (kb == kb0 || (kb & 3) == 0)) {
                            // this group's scale bytes: shared slot -> TMEM slot
                            sf_slot = sgm % kSfN;
                            const uint32_t sph = (sgm / kSfN) & 1;
                            if (!ptx::mbar_wait(&sffull[sf_slot], sph, p.wait_budget)) { fail(); failed = true; break; }
                            ptx::tc_fence_after();
                            const uint32_t src = ptx::smem_u32(sfring + size_t(sf_slot) * C::kSfSlotBytes);
                            sf_col = tmem_base + C::kSfCol0 + sf_slot * 16;
                            ptx::tmem_cp_32x128b_x4(sf_col + 8, ptx::sf_block_desc(src));          // A
                            ptx::tmem_cp_32x128b_x4(sf_col, ptx::sf_block_desc(src + 512));        // B rows 0-127
                            if (BN > 128) ptx::tmem_cp_32x128b_x4(sf_col + 4, ptx::sf_block_desc(src + 1024));
                            ++sgm;
                        }
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1;
                        if (!ptx::mbar_wait(&full[s], ph, p.wait_budget)) { fail(); failed = true; break; }
                        ptx::tc_fence_after();
                        const uint32_t pa = ptx::smem_u32(tiles + size_t(s) * C::kStageBytes);
                        const uint32_t qa = pa + C::kPBytes;
                        const uint32_t first = (ONE && kb > kb0) ? 1u : 0u;  // accumulate across K blocks
                        if (MX) {
                            const uint32_t idx = ptx::idesc_mx_e4m3(BN, uint32_t(kb & 3));
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                ptx::mma_f8_mx(d, ptx::sw128_kmajor_desc(pa + 32 * k), ptx::sw128_kmajor_desc(qa + 32 * k),
                                               idx, sf_col + 8, sf_col, first | (k > 0));
                            ptx::mma_commit(&empty[s]);
                            if ((kb & 3) == 3 || kb == kb1 - 1) ptx::mma_commit(&sfempty[sf_slot]);
                        } else if (PAIR) {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                ptx::mma_f8_pair(d, ptx::sw128_kmajor_desc(pa + 32 * k),
                                                 ptx::sw128_kmajor_desc(qa + 32 * k), idesc, first | (k > 0));
                            const uint32_t e0 = ptx::smem_u32(&empty[s]);      // stage free, in both CTAs
                            ptx::mma_commit_pair(e0);
                            ptx::mma_commit_pair(ptx::mapa_shared(e0, 1));
                        } else {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                ptx::mma_f8(d, ptx::sw128_kmajor_desc(pa + 32 * k),
                                            ptx::sw128_kmajor_desc(qa + 32 * k), idesc, first | (k > 0));
                            ptx::mma_commit(&empty[s]);
                        }
                        last_bar = &empty[s];
                        last_parity = ph;
                    }
                    if (failed) break;
                    if (MERGED) continue;                                    // empty[s] said it
                    if (PAIR) {                                              // step ready, in both CTAs
                        const uint32_t f0 = ptx::smem_u32(&tfull[buf]);
                        ptx::mma_commit_pair(f0);
                        ptx::mma_commit_pair(ptx::mapa_shared(f0, 1));
                    } else {
                        ptx::mma_commit(&tfull[buf]);
                    }
                    last_bar = &tfull[buf];
                    last_parity = tph;
                }
            }
            if (*abort_flag && last_bar) ptx::mbar_wait(last_bar, last_parity, 100000000LL);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ promotion
        if (C::kEpiWG > 1) ptx::regs_inc<C::kRegEpi>();
        const int e = warp - 4;                   // 0 .. 4*kEpiWG-1
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int chalf = e >> 2;                 // which kCW-column slice
        const int row = quarter * 32 + lane;      // TMEM lane = tile row
        const int nthreads = 128 * C::kEpiWG;
        const int etid = threadIdx.x - 128;
        const bool vec4 = p.scale_vec4 != 0;
        uint32_t c = 0;
        uint32_t sg = 0;                          // scale groups consumed (SS)
        uint64_t acc2[C::kCW / 2];
        // the leader's tempty (merged: full) barriers, as cluster addresses (pair mode)
        const uint32_t tempty0 = PAIR ? ptx::mapa_shared(ptx::smem_u32(tempty), 0) : 0u;
        const uint32_t full0 = PAIR ? ptx::mapa_shared(ptx::smem_u32(full), 0) : 0u;
        for (int u = unit0; u < p.units; u += unit_step) {
            int tp, tq, kb0, kb1;
            unit_coords(p, u, tp, tq, kb0, kb1);
            const int nkb = kb1 - kb0;
            const int q0 = tq * BN;
            const int m_row = tp * C::kTileRows + int(rank) * 128 + row;   // normal: token row
            const int n_row = tp * 128 + row;                              // swapped: weight row
            if (PC) {
                // slab[j] = scale of tile column j: sb[q0+j] (normal) or sa[q0+j] (swapped)
                ptx::named_bar_sync(1, nthreads);
                for (int i = etid; i < BN; i += nthreads) {
                    const int qi = q0 + i;
                    slab[i] = SWAP ? (qi < p.M ? __ldg(p.sa + qi) : 0.0f) : (qi < p.N ? __ldg(p.sb + qi) : 0.0f);
                }
                ptx::named_bar_sync(1, nthreads);
            }
            if (SWAP && SM == 0) {
                // slab[kbl*BN + j] = sa[q0+j, kb0+kbl] * sb[tp, kb0+kbl]
                ptx::named_bar_sync(1, nthreads);
                for (int i = etid; i < nkb * BN; i += nthreads) {
                    const int kbl = i / BN, j = i - kbl * BN;
                    const int m = q0 + j;
                    const int kb = kb0 + kbl;
                    slab[i] = (m < p.M) ? __ldg(p.sa + int64_t(m) * p.G + kb) *
                                          __ldg(p.sb + int64_t(tp) * p.G + kb)
                                        : 0.0f;
                }
                ptx::named_bar_sync(1, nthreads);
            }
#pragma unroll
            for (int j = 0; j < C::kCW / 2; ++j) acc2[j] = 0ull;

            // Normal mode: row scale sa[m_row, kb] times the column block's
            // sb[nb, kb], fetched four K blocks at a time, one group ahead.
            const int nb = (q0 + chalf * C::kCW) >> 7;
            const bool row_ok = !SWAP && SM == 0 && m_row < p.M;
            const bool col_ok = !SWAP && SM == 0 && nb * 128 < p.N;
            const float* sa_row = p.sa + int64_t(SWAP ? 0 : (row_ok ? m_row : 0)) * p.G;
            const float* sb_row = p.sb + int64_t(col_ok ? nb : 0) * p.G;
            float4 sa_cur, sb_cur, sa_nxt, sb_nxt;
            if (!SWAP && SM == 0 && !SS) {
                sa_cur = load_scale4(sa_row, kb0 >> 2, p.G, vec4, row_ok);
                sb_cur = load_scale4(sb_row, kb0 >> 2, p.G, vec4, col_ok);
                sa_nxt = load_scale4(sa_row, (kb0 >> 2) + 1, p.G, vec4, row_ok);
                sb_nxt = load_scale4(sb_row, (kb0 >> 2) + 1, p.G, vec4, col_ok);
            }
            bool ok = true;
            // per-tensor scales: one step per unit, one scalar scale
            const int kb_last = ONE ? kb0 + 1 : kb1;
            // one-step modes: the scale applied to the whole accumulation
            // (per-channel: this thread's row; its column scales come later)
            const float s_pt = PT ? __ldg(p.sa) * __ldg(p.sb) : MX ? 1.0f
                             : PC ? (SWAP ? (n_row < p.N ? __ldg(p.sb + n_row) : 0.0f)
                                          : (m_row < p.M ? __ldg(p.sa + m_row) : 0.0f))
                             : 0.0f;
            for (int kb = kb0; kb < kb_last; ++kb, ++c) {
                float s = s_pt;
                if (SS) {
                    if (kb == kb0 || (kb & 3) == 0) {
                        // this group's scales: row `row` of the 128 x 4 box, and
                        // the column block of this thread's slice
                        const uint32_t slot = sg % kSlots, sph = (sg / kSlots) & 1;
                        if (!ptx::mbar_wait(&sfull[slot], sph, p.wait_budget)) { fail(); ok = false; break; }
                        const uint8_t* src = sring + size_t(slot) * C::kScaleSlotBytes;
                        sa_cur = *reinterpret_cast<const float4*>(src + row * 16);
                        sb_cur = *reinterpret_cast<const float4*>(src + 2048 + ((chalf * C::kCW) >> 7) * 16);
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sempty[slot]);
                        ++sg;
                    }
                    s = pick4(sa_cur, kb & 3) * pick4(sb_cur, kb & 3);
                } else if (!SWAP && SM == 0) {
                    if ((kb & 3) == 0 && kb != kb0) {
                        sa_cur = sa_nxt;
                        sb_cur = sb_nxt;
                        sa_nxt = load_scale4(sa_row, (kb >> 2) + 1, p.G, vec4, row_ok);
                        sb_nxt = load_scale4(sb_row, (kb >> 2) + 1, p.G, vec4, col_ok);
                    }
                    s = pick4(sa_cur, kb & 3) * pick4(sb_cur, kb & 3);
                }
                const uint64_t s2 = ptx::pack_f32x2(s, s);
                const uint32_t buf = c % NB, tph = (c / NB) & 1;
                const bool landed = MERGED ? ptx::mbar_wait(&empty[c % STAGES], (c / STAGES) & 1, p.wait_budget)
                                           : ptx::mbar_wait(&tfull[buf], tph, p.wait_budget);
                if (!landed) { fail(); ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16)
                                       + buf * BN + chalf * C::kCW;
                const float* sl = slab + (kb - kb0) * BN + chalf * C::kCW;
                // Hand the TMEM buffer back (all of this warp's loads have landed).
                auto release = [&]() {
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        const uint32_t j = (c + NB) % STAGES;           // merged: the K block reusing it
                        if (MERGED && PAIR) ptx::mbar_arrive_cluster(full0 + j * 8);
                        else if (MERGED) ptx::mbar_arrive(&full[j]);
                        else if (PAIR) ptx::mbar_arrive_cluster(tempty0 + buf * 8);
                        else ptx::mbar_arrive(&tempty[buf]);
                    }
                };
                if constexpr (C::kCW == 128) {
                    // 128 columns: 48, then 80 -- the fewest FMAs between
                    // the first load and the release that the registers
                    // (128 accumulators + 80 loaded values) allow
                    float v[80];
                    ptx::tmem_ld32(taddr, v);
                    ptx::tmem_ld16(taddr + 32, v + 32);
                    ptx::tmem_wait_ld();
                    fma_uniform<48>(acc2, v, s2);
                    ptx::tmem_ld64(taddr + 48, v);
                    ptx::tmem_ld16(taddr + 112, v + 64);
                    ptx::tmem_wait_ld();
                    release();
                    fma_uniform<80>(acc2 + 24, v, s2);
                } else {
                    // Loads of this thread's kCW columns in chunks of at most 64;
                    // the TMEM buffer is released as soon as the last chunk has
                    // landed, then that chunk's FMAs run.
                    constexpr int kChunk = C::kCW >= 64 ? 64 : C::kCW;
                    constexpr int kChunks = C::kCW / kChunk;
                    float v[kChunk];
#pragma unroll
                    for (int ch = 0; ch < kChunks; ++ch) {
                        if constexpr (kChunk == 64) ptx::tmem_ld64(taddr + ch * 64, v);
                        else if constexpr (kChunk == 32) ptx::tmem_ld32(taddr + ch * 32, v);
                        else ptx::tmem_ld16(taddr + ch * 16, v);
                        ptx::tmem_wait_ld();
                        if (ch == kChunks - 1) release();
                        if (SWAP && SM == 0) fma_columns<kChunk>(acc2 + ch * kChunk / 2, v, sl + ch * kChunk);
                        else fma_uniform<kChunk>(acc2 + ch * kChunk / 2, v, s2);
                    }
                }
            }
            if (!ok) break;

            // ---------------------------------------------------- epilogue
            float acc[C::kCW];
#pragma unroll
            for (int j = 0; j < C::kCW / 2; ++j) ptx::unpack_f32x2(acc2[j], acc[2 * j], acc[2 * j + 1]);
            if (PC) {
#pragma unroll
                for (int j = 0; j < C::kCW; ++j) acc[j] *= slab[chalf * C::kCW + j];
            }
            if (C::TS && p.ystore && p.splits == 1 && u < p.full_units) {
                // bf16 Y through shared memory: this warp's 32 rows x 128
                // columns as two 64-column boxes (32 rows of 128 bytes, 16-byte
                // chunk c of row r at chunk c ^ (r % 8)), then two bulk stores
                uint8_t* wreg = ytile + size_t(e) * 8192;
                if (lane == 0) ptx::bulk_wait_read_all();      // the previous tile's stores have read it
                __syncwarp();
#pragma unroll
                for (int b = 0; b < 2; ++b) {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const int j = b * 64 + cc * 8;
                        uint4 w;
                        w.x = ptx::pack_bf16x2(acc[j + 0], acc[j + 1]);
                        w.y = ptx::pack_bf16x2(acc[j + 2], acc[j + 3]);
                        w.z = ptx::pack_bf16x2(acc[j + 4], acc[j + 5]);
                        w.w = ptx::pack_bf16x2(acc[j + 6], acc[j + 7]);
                        *reinterpret_cast<uint4*>(wreg + b * 4096 + lane * 128 + ((cc ^ (lane & 7)) * 16)) = w;
                    }
                }
                ptx::fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    const int y0 = tp * C::kTileRows + int(rank) * 128 + quarter * 32;
                    const int x0 = q0 + chalf * C::kCW;
                    if (y0 < p.M) {
                        if (x0 < p.N) ptx::tma_store_2d(&tmY, ptx::smem_u32(wreg), x0, y0);
                        if (x0 + 64 < p.N) ptx::tma_store_2d(&tmY, ptx::smem_u32(wreg + 4096), x0 + 64, y0);
                    }
                    ptx::bulk_commit_group();
                }
            } else if (p.splits == 1 && u < p.full_units && !SWAP && C::kCW % 64 == 0) {
                // bf16 Y, 64 columns (8 chunks) per block, stored through
                // transpose8x8.  Writing a tile row by row took ~8000 clocks
                // per tile with the MMA stalled behind it; this takes ~3200.
                const int g8 = lane & 7;
                const int m_base = tp * C::kTileRows + int(rank) * 128 + quarter * 32 + (lane & ~7);
#pragma unroll
                for (int b = 0; b < C::kCW / 64; ++b) {
                    uint4 a[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int j = b * 64 + k * 8;
                        a[k].x = ptx::pack_bf16x2(acc[j + 0], acc[j + 1]);
                        a[k].y = ptx::pack_bf16x2(acc[j + 2], acc[j + 3]);
                        a[k].z = ptx::pack_bf16x2(acc[j + 4], acc[j + 5]);
                        a[k].w = ptx::pack_bf16x2(acc[j + 6], acc[j + 7]);
                    }
                    transpose8x8(a, g8);
                    const int n = q0 + chalf * C::kCW + b * 64 + g8 * 8;     // a[k] = chunk g8 of row m_base + k
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int m = m_base + k;
                        if (m >= p.M) continue;
                        uint16_t* yr = p.y + int64_t(m) * p.ldy;
                        if (n + 8 <= p.N) {
                            *reinterpret_cast<uint4*>(yr + n) = a[k];
                        } else {
                            const uint32_t wv[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
#pragma unroll
                            for (int t = 0; t < 8; ++t)
                                if (n + t < p.N) yr[n + t] = uint16_t(wv[t >> 1] >> (16 * (t & 1)));
                        }
                    }
                }
            } else if (p.splits == 1 && u < p.full_units) {
                if (!SWAP) {
                    const int m = m_row;
                    const int n_first = q0 + chalf * C::kCW;
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
                            const int m = q0 + chalf * C::kCW + j;
                            if (m < p.M)
                                p.y[int64_t(m) * p.ldy + n] =
                                    uint16_t(ptx::pack_bf16x2(acc[j], 0.0f) & 0xFFFF);
                        }
                    }
                }
            } else {
                // fp32 partial: split-K slot [split][M][ldw], or (split tail)
                // slot u - full_units laid out [tile rows][BN] per tile
                const bool tail = u >= p.full_units;
                const int split = u % p.splits;
                float* wsp = p.ws + int64_t(split) * p.M * p.ldw;
                if (!SWAP && C::kCW % 32 == 0) {
                    // 32 fp32 columns (8 chunks) per block, through transpose8x8
                    const int g8 = lane & 7;
                    const int r_base = quarter * 32 + (lane & ~7);          // tile row of a[0] after the transpose
                    const int m_base = tp * C::kTileRows + int(rank) * 128 + r_base;
#pragma unroll
                    for (int b = 0; b < C::kCW / 32; ++b) {
                        uint4 a[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int j = b * 32 + k * 4;
                            a[k] = make_uint4(__float_as_uint(acc[j]), __float_as_uint(acc[j + 1]),
                                              __float_as_uint(acc[j + 2]), __float_as_uint(acc[j + 3]));
                        }
                        transpose8x8(a, g8);
                        const int n = q0 + chalf * C::kCW + b * 32 + g8 * 4;  // a[k] = chunk g8 of row m_base + k
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int m = m_base + k;
                            if (m >= p.M) continue;
                            // row m, indexed by the output column n
                            float* wr = tail ? p.ws + (int64_t(u - p.full_units) * C::kTileRows + int(rank) * 128 + r_base + k) * BN - q0
                                             : wsp + int64_t(m) * p.ldw;
                            if (n + 4 <= p.N) {
                                *reinterpret_cast<uint4*>(wr + n) = a[k];
                            } else {
                                const uint32_t wv[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
#pragma unroll
                                for (int t = 0; t < 4; ++t)
                                    if (n + t < p.N) wr[n + t] = __uint_as_float(wv[t]);
                            }
                        }
                    }
                } else if (!SWAP) {
                    const int m = m_row;
                    const int n_first = q0 + chalf * C::kCW;
                    if (m < p.M) {
                        float* wr = tail ? p.ws + (int64_t(u - p.full_units) * C::kTileRows + int(rank) * 128 + row) * BN - q0
                                         : wsp + int64_t(m) * p.ldw;
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
                            const int m = q0 + chalf * C::kCW + j;
                            if (m < p.M) wsp[int64_t(m) * p.ldw + n] = acc[j];
                        }
                    }
                }
            }
        }
    }

    if (C::TS && warp >= 4 && lane == 0) ptx::bulk_wait_all();   // this warp's Y stores have completed
    __syncwarp();
    ptx::tc_fence_before();
    if (PAIR) ptx::cluster_sync();      // both CTAs done with TMEM and with each other's barriers
    else __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        if (PAIR) ptx::tmem_dealloc_pair(tmem_base, C::kTmemCols);
        else ptx::tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// Fixed-order sum of the split-K partials and conversion to bf16.
// Each thread handles 4 consecutive columns of one row.
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ ws, int splits, int M, int N, int64_t ldw,
                     uint16_t* __restrict__ y, int64_t ldy) {
    pdl_begin();
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

// Fixed-order sum of the split-tail partials (slot tt * splits + s holds
// split s of tail tile tt, tile_rows x bn fp32) and conversion to bf16 into Y.
// Each thread handles 4 consecutive columns of one tile row.
__global__ void __launch_bounds__(256)
tail_reduce_kernel(const float* __restrict__ ws, int tail_tiles, int splits, int full_tiles, int tiles_p,
                   int tile_rows, int bn, int M, int N, uint16_t* __restrict__ y, int64_t ldy) {
    pdl_begin();
    const int quads = bn / 4;
    const int64_t per_tile = int64_t(tile_rows) * quads;
    const int64_t total = int64_t(tail_tiles) * per_tile;
    const int64_t slot = int64_t(tile_rows) * bn;
    for (int64_t i = int64_t(blockIdx.x) * 256 + threadIdx.x; i < total; i += int64_t(gridDim.x) * 256) {
        const int tt = int(i / per_tile);
        const int rem = int(i - int64_t(tt) * per_tile);
        const int r = rem / quads;
        const int c = (rem - r * quads) * 4;
        const int tile = full_tiles + tt;
        const int64_t m = int64_t(tile % tiles_p) * tile_rows + r;
        const int n = (tile / tiles_p) * bn + c;
        if (m >= M || n >= N) continue;
        const float* src = ws + (int64_t(tt) * splits * tile_rows + r) * bn + c;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        // loads issued 18 at a time (all of them for the usual split
        // counts), added in split order
        for (int s0 = 0; s0 < splits; s0 += 18) {
            float4 v[18];
#pragma unroll
            for (int t = 0; t < 18; ++t)
                v[t] = s0 + t < splits ? __ldcs(reinterpret_cast<const float4*>(src + int64_t(s0 + t) * slot))
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int t = 0; t < 18; ++t)
                if (s0 + t < splits) { a[0] += v[t].x; a[1] += v[t].y; a[2] += v[t].z; a[3] += v[t].w; }
        }
        if (n + 4 <= N) {
            uint2 o;
            o.x = ptx::pack_bf16x2(a[0], a[1]);
            o.y = ptx::pack_bf16x2(a[2], a[3]);
            *reinterpret_cast<uint2*>(y + m * ldy + n) = o;
        } else {
            for (int t = 0; t < 4 && n + t < N; ++t)
                y[m * ldy + n + t] = uint16_t(ptx::pack_bf16x2(a[t], 0.0f) & 0xFFFF);
        }
    }
}

}  // namespace fp8q
