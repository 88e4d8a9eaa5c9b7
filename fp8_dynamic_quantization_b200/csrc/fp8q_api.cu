// C ABI of the fp8q library: argument checks, launch selection, launches.
// Declarations and the full contract are in include/fp8q.h.
#include "fp8q.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp8q_status.cuh"
#include "gemm_kernels.cuh"
#include "quant_kernels.cuh"

// Split-K partial sums of fp8_block_gemm_noalloc live in this file-scope
// device array instead of a caller-provided workspace.  Every device that
// loads the library holds it until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[FP8Q_NOALLOC_MAX_SCRATCH_BYTES / sizeof(float)];

namespace fp8q {
namespace {

// ------------------------------------------------------------------ helpers
bool log_enabled() {
    static const bool on = [] {
        const char* v = std::getenv("FP8Q_LOG");
        return v && v[0] && v[0] != '0';
    }();
    return on;
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

struct DeviceInfo {
    bool ready = false;
    int status = FP8Q_OK;
    int sms = 0;
    int index = 0;
    int64_t l2_bytes = 0;
};

// The per-tensor passes hold a tensor of at most half the L2 there between
// the amax pass and the apply pass (measured at 4096 x 7168, 58.7 MB of a
// 126 MB L2: 26.3 against 28.2 us per call; at 16384 x 7168, above L2, the
// same hints cost 3%).
bool keep_in_l2(const DeviceInfo* d, int64_t bytes) { return bytes <= d->l2_bytes / 2; }

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

constexpr int kClusterU = 8;        // vectors per thread in the one-cluster per-tensor kernel
constexpr int kStreamU = 4;         // vectors per thread per iteration elsewhere
constexpr int kMaxPartials = 4096;  // per-tensor workspace partial slots
constexpr int kBlocksPerSm = 8;     // 256-thread CTAs per SM for streaming kernels

// Programmatic dependent launch of every kernel (the kernels' side is
// pdl_begin / griddepcontrol in the device code): a launch may begin while
// the previous kernel on the stream finishes, and waits for it before it
// touches global memory.  FP8Q_PDL=0 launches without the attribute
// (measurement; same results).
bool pdl_enabled() {
    static const bool on = [] {
        const char* e = std::getenv("FP8Q_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

// cudaLaunchKernelEx with the programmatic-serialisation attribute and, for
// cluster > 1, a 1-D cluster of that many CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   unsigned cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int BN, bool SWAP, int STAGES, bool PAIR = false, int SM = 0, bool SS = false>
cudaError_t set_gemm_smem() {
    return cudaFuncSetAttribute(block_gemm_kernel<BN, SWAP, STAGES, PAIR, SM, SS>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(GemmCfg<BN, SWAP, STAGES, PAIR, SM, SS>::kSmemBytes));
}

// Device facts, queried once per device.  FP8Q_ERR_NO_DEVICE unless the
// current device is an sm_100 part.
int device_info(DeviceInfo** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FP8Q_ERR_NO_DEVICE;
    }
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        if (!d.ready) {
            cudaDeviceProp prop;
            if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
                cudaGetLastError();
                return FP8Q_ERR_NO_DEVICE;
            }
            d.status = FP8Q_OK;
            d.index = dev;
            if (prop.major != 10) d.status = FP8Q_ERR_NO_DEVICE;
            d.sms = prop.multiProcessorCount;
            d.l2_bytes = prop.l2CacheSize;
            if (d.status == FP8Q_OK) {
                cudaError_t e = cudaSuccess;
                if (e == cudaSuccess) e = set_gemm_smem<16, true, 12>();
                if (e == cudaSuccess) e = set_gemm_smem<32, true, 10>();
                if (e == cudaSuccess) e = set_gemm_smem<64, true, 8>();
                if (e == cudaSuccess) e = set_gemm_smem<128, true, 6>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 6>();
                if (e == cudaSuccess) e = set_gemm_smem<192, false, 5>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 4>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 4, false, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 6, false, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 5, true>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 8, true>();
                if (e == cudaSuccess) e = set_gemm_smem<16, true, 12, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<32, true, 10, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<64, true, 8, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<128, true, 6, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 6, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<192, false, 5, false, true>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 5, true, 1>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 8, true, 1>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 5, true, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 8, true, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<16, true, 12, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<32, true, 10, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<64, true, 8, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<128, true, 6, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 6, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<192, false, 5, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 4, false, 3>();
                if (e == cudaSuccess) e = set_gemm_smem<16, true, 12, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<32, true, 10, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<64, true, 8, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<128, true, 6, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<128, false, 6, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<192, false, 5, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 4, false, 2>();
                if (e == cudaSuccess) e = set_gemm_smem<256, false, 4, false, true>();
                if (e != cudaSuccess) { cudaGetLastError(); d.status = FP8Q_ERR_CUDA; }
            }
            d.ready = true;
        }
    }
    *out = &d;
    return d.status;
}

// Stream -> error-word slot (g_stream_status), per device.  Slots 1.. are
// handed out in the order streams first ask for one; once they are all
// taken, later streams share slot 0.  A stream handle that CUDA recycles
// for a new stream keeps the slot.
cudaStream_t g_slot_stream[kMaxDevices][kStatusSlots];
int g_slots_used[kMaxDevices];
std::mutex g_slot_mutex;

int status_slot(int dev, cudaStream_t st) {
    thread_local int last_dev = -1, last_slot = 0;
    thread_local cudaStream_t last_st = nullptr;
    if (dev == last_dev && st == last_st) return last_slot;
    int slot = 0;
    {
        std::lock_guard<std::mutex> lock(g_slot_mutex);
        const int n = g_slots_used[dev];
        for (int i = 1; i <= n && slot == 0; ++i)
            if (g_slot_stream[dev][i] == st) slot = i;
        if (slot == 0 && n + 1 < kStatusSlots) {
            slot = n + 1;
            g_slot_stream[dev][slot] = st;
            g_slots_used[dev] = slot;
        }
    }
    last_dev = dev;
    last_st = st;
    last_slot = slot;
    return slot;
}

std::atomic<unsigned long long> g_launches{0};

// Status of the launches just enqueued; counts them when they succeeded.
int launch_status(int n = 1) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return FP8Q_ERR_CUDA;
    g_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed);
    return FP8Q_OK;
}

// CTAs of `kernel` (kQuantThreads threads, no dynamic shared memory) that
// fit on the device at once: the grid of the chunked streaming kernels,
// which stride over their chunks.
template <auto kernel>
int64_t resident_ctas(int sms) {
    static const int per_sm = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kQuantThreads, 0) != cudaSuccess) n = 0;
        cudaGetLastError();
        return std::max(1, std::min(n, kBlocksPerSm));
    }();
    return int64_t(per_sm) * sms;
}

// Grid of a chunked kernel: one CTA per chunk, at most what fits at once.
// (A grid that gives every CTA the same number of chunks measured slower
// back to back: 21.6 against 20.0 us per-tensor at 4096 x 7168.)
template <auto kernel>
int chunk_grid(int64_t chunks, int sms) {
    return int(std::max<int64_t>(1, std::min(chunks, resident_ctas<kernel>(sms))));
}

// Streaming grid: enough CTAs for the data, capped at kBlocksPerSm per SM.
int stream_grid(int64_t nvec, int sms) {
    const int64_t need = (nvec + int64_t(kQuantThreads) * kStreamU - 1) /
                         (int64_t(kQuantThreads) * kStreamU);
    const int64_t cap = std::min<int64_t>(int64_t(sms) * kBlocksPerSm, kMaxPartials);
    return int(std::max<int64_t>(1, std::min(need, cap)));
}

// Checks shared by the bf16 -> code entry points.
int check_bf16_matrix(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                      const uint8_t* q, int64_t ldq, int64_t col_multiple) {
    if (rows < 0 || cols < 0) return FP8Q_ERR_INVALID_ARG;
    if (cols % col_multiple) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return FP8Q_OK;
    if (!x || !q) return FP8Q_ERR_INVALID_ARG;
    if (ldx < cols || ldq < cols) return FP8Q_ERR_INVALID_ARG;
    if (!aligned16(x) || (ldx * 2) % 16 || !aligned8(q) || ldq % 8) return FP8Q_ERR_MISALIGNED;
    return FP8Q_OK;
}

// ------------------------------------------------------------------ GEMM plan
enum Mode { kNormal = 0, kSwap = 1, kPair = 2 };
struct TableRow { int64_t m_lo, m_hi, n_lo, n_hi; int mode, bn, splits; };
const TableRow kGemmTable[] = {
#include "launch_table.inc"
};

struct GemmPlan {
    bool swap, pair;
    int bn, stages, splits, tiles_p, tiles_q, units, grid;
    int full_tiles, tail_tiles, tail_splits;   // split tail (normal and pair tiles)
    int64_t ldw;
    size_t ws_bytes;
};

// Measurement override: FP8Q_PER_TENSOR_PATH=twopass makes every per-tensor
// call take the amax + apply passes (same result).
bool per_tensor_two_pass_forced() {
    static const bool v = [] {
        const char* e = std::getenv("FP8Q_PER_TENSOR_PATH");
        return e && std::strcmp(e, "twopass") == 0;
    }();
    return v;
}

// Bound on every barrier wait inside the GEMM, in SM clock cycles (about
// two seconds by default).  FP8Q_WAIT_BUDGET_CYCLES overrides it for fault
// testing; it never changes the result of a call that completes.
std::atomic<long long> g_wait_budget_override{-1};

long long wait_budget_cycles() {
    const long long o = g_wait_budget_override.load(std::memory_order_relaxed);
    if (o >= 0) return o;
    static const long long v = [] {
        const char* e = std::getenv("FP8Q_WAIT_BUDGET_CYCLES");
        if (e && e[0]) {
            char* end = nullptr;
            const long long b = std::strtoll(e, &end, 10);
            if (end && *end == 0 && b >= 0) return b;
        }
        return 4000000000LL;
    }();
    return v;
}

// Tuning override of the table (FP8Q_GEMM_TILE="normal:128", "swap:64:4",
// ...: mode, tile width, optional split-K count).  For measuring launch
// choices only; every choice computes the same sums.
bool tile_override(TableRow* out) {
    static TableRow row;
    static const bool has = [] {
        const char* v = std::getenv("FP8Q_GEMM_TILE");
        if (!v || !v[0]) return false;
        char mode[16] = {0};
        int bn = 0, splits = 0;
        if (std::sscanf(v, "%15[a-z]:%d:%d", mode, &bn, &splits) < 2) return false;
        const bool swap = std::strcmp(mode, "swap") == 0;
        const bool pair = std::strcmp(mode, "pair") == 0;
        if (!swap && !pair && std::strcmp(mode, "normal") != 0) return false;
        if (swap ? !(bn == 16 || bn == 32 || bn == 64 || bn == 128)
                 : pair ? !(bn == 256 || bn == 128) : !(bn == 128 || bn == 192 || bn == 256))
            return false;
        row = TableRow{1, int64_t(1) << 30, 1, int64_t(1) << 30, swap ? kSwap : pair ? kPair : kNormal,
                       bn, pair ? 1 : splits};
        return true;
    }();
    if (has) *out = row;
    return has;
}

// no_pair: a pair row runs as the single-CTA tile of the same width (the
// scale modes other than fp32 block scales).
//
// Split tail: with one whole tile per unit, a tile count just above a
// multiple of the SM count leaves a last wave in which few SMs work for a
// whole tile time (4096 x 7168 with 128 x 256 tiles: 896 tiles = 6 waves of
// 148 + 8).  If that last wave holds at most half the SMs, its tiles are
// split along K into S = min(SMs / tail, K blocks / 2) ranges instead, so it
// takes about 1/S of a tile time; tail_reduce_kernel then adds the S fp32
// partials of each tail tile in fixed order.  ws_cap bounds the workspace
// either split may use: split-K shrinks to fit (to 1, except where the
// swapped kernel needs at least 2), the tail's S shrinks to fit (below 2 the
// tail stays whole).
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int sms, bool no_pair = false,
                   size_t ws_cap = ~size_t(0)) {
    GemmPlan pl{};
    const TableRow* row = &kGemmTable[0];
    for (const TableRow& r : kGemmTable)
        if (M >= r.m_lo && M <= r.m_hi && N >= r.n_lo && N <= r.n_hi) { row = &r; break; }
    TableRow forced;
    if (tile_override(&forced)) row = &forced;
    pl.swap = row->mode == kSwap;
    pl.pair = row->mode == kPair && !no_pair;
    pl.bn = row->bn;
    pl.stages = pl.swap ? (pl.bn == 16 ? 12 : pl.bn == 32 ? 10 : pl.bn == 64 ? 8 : 6)
                        : pl.pair ? (pl.bn == 256 ? 5 : 8) : (pl.bn == 192 ? 5 : pl.bn == 256 ? 4 : 6);
    const int G = int(K / 128);
    const int64_t rows_p = pl.swap ? N : M, rows_q = pl.swap ? M : N;
    const int tile_rows = pl.pair ? 256 : 128;
    pl.tiles_p = int((rows_p + tile_rows - 1) / tile_rows);
    pl.tiles_q = int((rows_q + pl.bn - 1) / pl.bn);
    const int64_t tiles = int64_t(pl.tiles_p) * pl.tiles_q;
    int splits = row->splits;
    if (pl.pair) splits = 1;
    if (splits <= 0) {
        splits = 1;
        if (tiles < sms) splits = int(std::max<int64_t>(1, sms / tiles));
        splits = std::min(splits, std::max(1, G / 2));   // at least 2 K blocks per split
    }
    splits = std::max(1, std::min(splits, G));
    if (splits > 1) {   // split-K partials must fit ws_cap: fewer splits if not
        const size_t per_split = size_t(M) * size_t((N + 7) / 8 * 8) * sizeof(float);
        splits = int(std::max<size_t>(1, std::min<size_t>(size_t(splits), ws_cap / per_split)));
    }
    if (pl.swap) {   // the swapped kernel stages at most 64 K blocks of scales per unit
        while ((G + splits - 1) / splits > 64) ++splits;
    }
    pl.splits = splits;
    pl.units = int(tiles * splits);
    pl.full_tiles = int(tiles);
    pl.tail_tiles = 0;
    pl.tail_splits = 1;
    const int slots = pl.pair ? sms / 2 : sms;          // tiles that run at once
    if (!pl.swap && splits == 1 && tiles > slots && tiles % slots != 0) {
        const int tail = int(tiles % slots);
        const size_t slot_bytes = size_t(tail) * tile_rows * size_t(pl.bn) * sizeof(float);   // one split of every tail tile
        const int s = int(std::min<size_t>(size_t(std::min(slots / tail, G / 2)), ws_cap / slot_bytes));
        if (s >= 2) {
            pl.tail_tiles = tail;
            pl.tail_splits = s;
            pl.full_tiles = int(tiles) - tail;
            pl.units = pl.full_tiles + tail * s;
        }
    }
    pl.grid = pl.pair ? 2 * std::max(1, std::min(pl.units, sms / 2))
                      : std::max(1, std::min(pl.units, sms));
    pl.ldw = (N + 7) / 8 * 8;
    pl.ws_bytes = splits > 1 ? size_t(splits) * size_t(M) * size_t(pl.ldw) * sizeof(float)
                : pl.tail_tiles > 0 ? size_t(pl.tail_tiles) * size_t(pl.tail_splits) * tile_rows * size_t(pl.bn) * sizeof(float)
                : 0;
    return pl;
}

// Map of the bf16 output Y [M, N] (row pitch ldy elements, 16-byte aligned
// base and pitch): boxes of 64 columns (128 bytes) x 32 rows, 128-byte
// swizzle, for bulk stores of the CTA-pair tiles' epilogue.
bool make_y_tmap(CUtensorMap* m, const void* base, int64_t M, int64_t N, int64_t ldy);

// cuTensorMapEncodeTiled through the runtime's driver entry point.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        cudaGetLastError();
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D map over an E4M3 [rows, K] matrix (row pitch ld bytes), box of
// 128 K-bytes x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int64_t ld, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(ld)};
    cuuint32_t box[2] = {128u, cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_y_tmap(CUtensorMap* m, const void* base, int64_t M, int64_t N, int64_t ldy) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(M)};
    cuuint64_t strides[1] = {cuuint64_t(ldy) * 2};
    cuuint32_t box[2] = {64u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map of an fp32 scale matrix [rows, G] (row pitch G floats, G % 4 == 0,
// 16-byte aligned base): boxes of 4 consecutive K-block scales x box_rows
// rows, no swizzle; rows past the end read as zero.
bool make_scale_tmap(CUtensorMap* m, const float* base, int64_t rows, int64_t G, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(G), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(G) * 4};
    cuuint32_t box[2] = {4u, cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// tsa/tsb: scale maps (staged-scale variants only; the others ignore them)
template <int BN, bool SWAP, int STAGES, bool PAIR = false, int SM = 0, bool SS = false>
void launch_gemm(const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& tsa, const CUtensorMap& tsb,
                 const GemmParams& p, int grid, cudaStream_t st, const CUtensorMap* ty = nullptr) {
    using C = GemmCfg<BN, SWAP, STAGES, PAIR, SM, SS>;
    launch(block_gemm_kernel<BN, SWAP, STAGES, PAIR, SM, SS>, dim3(unsigned(grid)), dim3(C::kThreads),
           C::kSmemBytes, st, PAIR ? 2u : 1u, tp, tq, tsa, tsb, ty ? *ty : tp, p);
}

// ------------------------------------------------------------------ no-alloc GEMM scratch
constexpr size_t kNoAllocScratchBytes = FP8Q_NOALLOC_MAX_SCRATCH_BYTES;

// Device address of g_noalloc_scratch on the current device.  In host code
// the symbol's name is only a host-side stand-in, so the address is looked
// up once per device (with that device current) and cached.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

int noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FP8Q_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, ::g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return FP8Q_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return FP8Q_OK;
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

// ====================================================================== ABI
extern "C" {

const char* fp8q_status_string(int status) {
    switch (status) {
        case FP8Q_OK: return "FP8Q_OK";
        case FP8Q_ERR_INVALID_ARG: return "FP8Q_ERR_INVALID_ARG";
        case FP8Q_ERR_UNSUPPORTED_SHAPE: return "FP8Q_ERR_UNSUPPORTED_SHAPE";
        case FP8Q_ERR_MISALIGNED: return "FP8Q_ERR_MISALIGNED";
        case FP8Q_ERR_WORKSPACE: return "FP8Q_ERR_WORKSPACE";
        case FP8Q_ERR_CUDA: return "FP8Q_ERR_CUDA";
        case FP8Q_ERR_TIMEOUT: return "FP8Q_ERR_TIMEOUT";
        case FP8Q_ERR_NO_DEVICE: return "FP8Q_ERR_NO_DEVICE";
        default: return "FP8Q_ERR_UNKNOWN";
    }
}

int fp8q_abi_version(void) { return (1 << 16) | 1; }

// Host only: the launch plan fp8_block_gemm would use on a device with
// `sms` SMs (the ue8m0 GEMM runs pair rows as single-CTA tiles).
int fp8q_gemm_plan(int64_t M, int64_t N, int64_t K, int sms, size_t ws_cap, int* plan, size_t* ws_bytes) {
    if (M <= 0 || N <= 0 || K <= 0 || sms <= 0 || !plan || !ws_bytes) return FP8Q_ERR_INVALID_ARG;
    if (K % 128 || M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    const GemmPlan pl = plan_gemm(M, N, K, sms, false, ws_cap);
    const int v[11] = {pl.swap ? 1 : 0, pl.pair ? 1 : 0, pl.bn, pl.stages, pl.splits, pl.tiles_p,
                       pl.tiles_q, pl.units, pl.grid, pl.tail_tiles, pl.tail_splits};
    for (int i = 0; i < 11; ++i) plan[i] = v[i];
    *ws_bytes = pl.ws_bytes;
    return FP8Q_OK;
}

// ------------------------------------------------------------ per-tensor
size_t fp8_act_quant_per_tensor_workspace_size(int64_t, int64_t) {
    return size_t(2 + kMaxPartials) * sizeof(uint32_t);
}

size_t fp8_act_amax_workspace_size(int64_t, int64_t) {
    return size_t(kMaxPartials) * sizeof(uint32_t);
}

int fp8_act_quant_per_tensor(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                             int64_t ldq, float* scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
    int rc = check_bf16_matrix(x, M, K, ldx, q, ldq, 8);
    if (rc != FP8Q_OK) return rc;
    if (!scale) return FP8Q_ERR_INVALID_ARG;
    if (!aligned4(scale)) return FP8Q_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < fp8_act_quant_per_tensor_workspace_size(M, K))
        return FP8Q_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP8Q_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d)) != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M == 0 || K == 0)
        return cudaMemsetAsync(scale, 0, sizeof(float), st) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;

    const int64_t vpr = K / 8, nvec = M * vpr;
    const bool contig = (ldx == K && ldq == K);
    uint32_t* ws = static_cast<uint32_t*>(workspace);
    // Single launch when the tensor fits in the registers of one cluster of
    // up to 8 CTAs; the partial maxima are exchanged through distributed
    // shared memory.
    constexpr int kClusterThreads = 256;
    const int64_t per_cta = int64_t(kClusterThreads) * kClusterU;
    const int64_t csize = (nvec + per_cta - 1) / per_cta;
    if (csize <= kClusterMax && !per_tensor_two_pass_forced()) {
        if (log_enabled())
            std::fprintf(stderr, "[fp8q] per_tensor M=%lld K=%lld: one cluster of %lld CTAs\n",
                         (long long)M, (long long)K, (long long)csize);
        const uint16_t* xs = static_cast<const uint16_t*>(x);
        const cudaError_t e =
            contig ? launch(per_tensor_cluster_kernel<kClusterU, true, kClusterThreads>, dim3(unsigned(csize)),
                            dim3(kClusterThreads), 0, st, unsigned(csize), xs, nvec, vpr, ldx, q, ldq, scale)
                   : launch(per_tensor_cluster_kernel<kClusterU, false, kClusterThreads>, dim3(unsigned(csize)),
                            dim3(kClusterThreads), 0, st, unsigned(csize), xs, nvec, vpr, ldx, q, ldq, scale);
        if (e != cudaSuccess) { cudaGetLastError(); return FP8Q_ERR_CUDA; }
        return launch_status(1);
    }
    uint32_t* partials = ws;
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    const bool keep = keep_in_l2(d, M * ldx * 2);
    if (contig) {
        // The amax pass takes chunks of 256 x 4 vectors, or of 256 x 2 when
        // that would leave fewer chunks than CTAs that fit at once
        // (1024 x 7168: 7.5 against 8.3 us per call; at 4096 x 7168 and
        // above the larger chunks are as fast or faster).
        constexpr int64_t kChunk = int64_t(kQuantThreads) * kStreamU;
        const int64_t chunks = (nvec + kChunk - 1) / kChunk;
        const bool half = chunks < resident_ctas<amax_contig_kernel<kStreamU, true>>(d->sms);
        const int64_t achunks = half ? (nvec + kChunk / 2 - 1) / (kChunk / 2) : chunks;
        const uint4* xv = static_cast<const uint4*>(x);
        uint2* qv = reinterpret_cast<uint2*>(q);
        const int ga = half ? (keep ? chunk_grid<amax_contig_kernel<kStreamU / 2, true>>(achunks, d->sms)
                                    : chunk_grid<amax_contig_kernel<kStreamU / 2, false>>(achunks, d->sms))
                            : (keep ? chunk_grid<amax_contig_kernel<kStreamU, true>>(achunks, d->sms)
                                    : chunk_grid<amax_contig_kernel<kStreamU, false>>(achunks, d->sms));
        const int gp = keep ? chunk_grid<apply_contig_kernel<kStreamU, false, true>>(chunks, d->sms)
                            : chunk_grid<apply_contig_kernel<kStreamU, false, false>>(chunks, d->sms);
        if (log_enabled())
            std::fprintf(stderr, "[fp8q] per_tensor M=%lld K=%lld: amax grid=%d (%lld chunks), apply grid=%d "
                                 "(%lld chunks)%s\n",
                         (long long)M, (long long)K, ga, (long long)achunks, gp, (long long)chunks,
                         keep ? ", kept in L2" : "");
        if (half && keep)
            launch(amax_contig_kernel<kStreamU / 2, true>, dim3(ga), dim3(kQuantThreads), 0, st, 1u, xv, nvec, partials);
        else if (half)
            launch(amax_contig_kernel<kStreamU / 2, false>, dim3(ga), dim3(kQuantThreads), 0, st, 1u, xv, nvec, partials);
        else if (keep)
            launch(amax_contig_kernel<kStreamU, true>, dim3(ga), dim3(kQuantThreads), 0, st, 1u, xv, nvec, partials);
        else
            launch(amax_contig_kernel<kStreamU, false>, dim3(ga), dim3(kQuantThreads), 0, st, 1u, xv, nvec, partials);
        if (keep)
            launch(apply_contig_kernel<kStreamU, false, true>, dim3(gp), dim3(kQuantThreads), 0, st, 1u, xv, nvec,
                   (const uint32_t*)partials, ga, qv, scale);
        else
            launch(apply_contig_kernel<kStreamU, false, false>, dim3(gp), dim3(kQuantThreads), 0, st, 1u, xv, nvec,
                   (const uint32_t*)partials, ga, qv, scale);
        return launch_status(2);
    }
    const int grid = stream_grid(nvec, d->sms);
    if (log_enabled())
        std::fprintf(stderr, "[fp8q] per_tensor M=%lld K=%lld: amax+apply grid=%d\n",
                     (long long)M, (long long)K, grid);
    if (keep) {
        launch(amax_partial_kernel<kStreamU, false, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx,
               partials);
        launch(apply_kernel<kStreamU, false, false, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx,
               partials, grid, q, ldq, scale);
    } else {
        launch(amax_partial_kernel<kStreamU, false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx, partials);
        launch(apply_kernel<kStreamU, false, false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx, partials,
                                                                             grid, q, ldq, scale);
    }
    return launch_status(2);
}

int fp8_act_amax(const void* x, int64_t M, int64_t K, int64_t ldx, uint32_t* amax_bits,
                 void* workspace, size_t workspace_bytes, void* stream) {
    if (M < 0 || K < 0) return FP8Q_ERR_INVALID_ARG;
    if (K % 8) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    if (!amax_bits) return FP8Q_ERR_INVALID_ARG;
    if (!aligned4(amax_bits)) return FP8Q_ERR_MISALIGNED;
    if (M > 0 && K > 0) {
        if (!x || ldx < K) return FP8Q_ERR_INVALID_ARG;
        if (!aligned16(x) || (ldx * 2) % 16) return FP8Q_ERR_MISALIGNED;
    }
    if (!workspace || workspace_bytes < fp8_act_amax_workspace_size(M, K)) return FP8Q_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP8Q_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M == 0 || K == 0)
        return cudaMemsetAsync(amax_bits, 0, 4, st) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
    const int64_t vpr = K / 8, nvec = M * vpr;
    uint32_t* partials = static_cast<uint32_t*>(workspace);
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    const bool keep = keep_in_l2(d, M * ldx * 2);      // for an apply call that follows
    if (ldx == K) {
        constexpr int64_t kChunk = int64_t(kQuantThreads) * kStreamU;
        const int64_t chunks = (nvec + kChunk - 1) / kChunk;
        const uint4* xv = static_cast<const uint4*>(x);
        const int ga = keep ? chunk_grid<amax_contig_kernel<kStreamU, true>>(chunks, d->sms)
                            : chunk_grid<amax_contig_kernel<kStreamU, false>>(chunks, d->sms);
        if (keep) launch(amax_contig_kernel<kStreamU, true>, dim3(ga), dim3(kQuantThreads), 0, st, 1u, xv, nvec, partials);
        else launch(amax_contig_kernel<kStreamU, false>, dim3(ga), dim3(kQuantThreads), 0, st, 1u, xv, nvec, partials);
        launch(reduce_partials_kernel, dim3(1), dim3(kQuantThreads), 0, st, 1u, (const uint32_t*)partials, ga, amax_bits);
        return launch_status(2);
    }
    const int grid = stream_grid(nvec, d->sms);
    if (keep)
        launch(amax_partial_kernel<kStreamU, false, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx,
               partials);
    else
        launch(amax_partial_kernel<kStreamU, false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx, partials);
    // Fold the partials into one word: a single CTA over `grid` words.
    launch(reduce_partials_kernel, dim3(1), dim3(kQuantThreads), 0, st, 1u, partials, grid, amax_bits);
    return launch_status(2);
}

int fp8_act_quant_apply(const void* x, int64_t M, int64_t K, int64_t ldx,
                        const uint32_t* amax_bits, uint8_t* q, int64_t ldq, float* scale,
                        void* stream) {
    int rc = check_bf16_matrix(x, M, K, ldx, q, ldq, 8);
    if (rc != FP8Q_OK) return rc;
    if (!amax_bits) return FP8Q_ERR_INVALID_ARG;
    if (!aligned4(amax_bits) || (scale && !aligned4(scale))) return FP8Q_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d)) != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t vpr = K / 8, nvec = M * vpr;
    if (nvec == 0) {
        if (scale) launch(scale_only_kernel, dim3(1), dim3(32), 0, st, 1u, amax_bits, scale);
        return launch_status();
    }
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    const bool keep = keep_in_l2(d, M * ldx * 2);      // an amax call before this one kept x in L2
    if (ldx == K && ldq == K) {
        constexpr int64_t kChunk = int64_t(kQuantThreads) * kStreamU;
        const int64_t chunks = (nvec + kChunk - 1) / kChunk;
        const uint4* xv = static_cast<const uint4*>(x);
        uint2* qv = reinterpret_cast<uint2*>(q);
        if (keep)
            launch(apply_contig_kernel<kStreamU, true, true>,
                   dim3(chunk_grid<apply_contig_kernel<kStreamU, true, true>>(chunks, d->sms)), dim3(kQuantThreads), 0,
                   st, 1u, xv, nvec, amax_bits, 1, qv, scale);
        else
            launch(apply_contig_kernel<kStreamU, true, false>,
                   dim3(chunk_grid<apply_contig_kernel<kStreamU, true, false>>(chunks, d->sms)), dim3(kQuantThreads), 0,
                   st, 1u, xv, nvec, amax_bits, 1, qv, scale);
        return launch_status();
    }
    const int grid = stream_grid(nvec, d->sms);
    if (keep)
        launch(apply_kernel<kStreamU, false, true, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx,
               amax_bits, 1, q, ldq, scale);
    else
        launch(apply_kernel<kStreamU, false, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, nvec, vpr, ldx, amax_bits, 1,
                                                                            q, ldq, scale);
    return launch_status();
}

// ------------------------------------------------------------ group / block
// e8: ue8m0 scales (E8M0 bytes) instead of fp32 amax/448.
static int run_group128(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                        void* scales, bool e8, void* stream) {
    int rc = check_bf16_matrix(x, M, K, ldx, q, ldq, 128);
    if (rc != FP8Q_OK) return rc;
    if (M == 0 || K == 0) return FP8Q_OK;
    if (!scales) return FP8Q_ERR_INVALID_ARG;
    if (!e8 && !aligned4(scales)) return FP8Q_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d)) != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t G = K / 128, groups = M * G;
    constexpr int kGroupU = 2;        // groups per thread per iteration (8 threads a group)
    const bool contig = ldx == K && ldq == K;
    if (contig && aligned32(x) && aligned16(q)) {
        // 4 threads a group, 32-byte loads: 4-13 % faster than 8 threads a
        // group at 1024-4096 x 7168 and 4000 x 1280, level at 16384 x 7168
        constexpr int64_t kChunk = int64_t(kQuantThreads / 4);
        const int64_t chunks = (groups + kChunk - 1) / kChunk;
        const uint4* xv = static_cast<const uint4*>(x);
        uint4* qv = reinterpret_cast<uint4*>(q);
        const int grid = e8 ? chunk_grid<group128_contig4_kernel<true>>(chunks, d->sms)
                            : chunk_grid<group128_contig4_kernel<false>>(chunks, d->sms);
        if (log_enabled())
            std::fprintf(stderr, "[fp8q] group128%s M=%lld K=%lld: 4 threads a group, grid=%d, %lld chunks\n",
                         e8 ? " ue8m0" : "", (long long)M, (long long)K, grid, (long long)chunks);
        if (e8) launch(group128_contig4_kernel<true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xv, qv, scales, groups);
        else launch(group128_contig4_kernel<false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xv, qv, scales, groups);
        return launch_status();
    }
    if (contig) {
        constexpr int64_t kChunk = int64_t(kQuantThreads / 8) * kGroupU;
        const int64_t chunks = (groups + kChunk - 1) / kChunk;
        const uint4* xv = static_cast<const uint4*>(x);
        uint2* qv = reinterpret_cast<uint2*>(q);
        const int grid = e8 ? chunk_grid<group128_contig_kernel<kGroupU, true>>(chunks, d->sms)
                            : chunk_grid<group128_contig_kernel<kGroupU, false>>(chunks, d->sms);
        if (log_enabled())
            std::fprintf(stderr, "[fp8q] group128%s M=%lld K=%lld: grid=%d, %lld chunks\n", e8 ? " ue8m0" : "",
                         (long long)M, (long long)K, grid, (long long)chunks);
        if (e8) launch(group128_contig_kernel<kGroupU, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xv, qv, scales, groups);
        else launch(group128_contig_kernel<kGroupU, false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xv, qv, scales, groups);
        return launch_status();
    }
    const int64_t need = (groups * 8 + int64_t(kQuantThreads) * kGroupU - 1) /
                         (int64_t(kQuantThreads) * kGroupU);
    const int grid = int(std::max<int64_t>(1, std::min<int64_t>(need, int64_t(d->sms) * kBlocksPerSm)));
    if (log_enabled())
        std::fprintf(stderr, "[fp8q] group128%s M=%lld K=%lld: grid=%d\n", e8 ? " ue8m0" : "",
                     (long long)M, (long long)K, grid);
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    if (e8)
        launch(group128_quant_kernel<kGroupU, false, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, ldx, q, ldq, scales, groups, G);
    else
        launch(group128_quant_kernel<kGroupU, false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, xs, ldx, q, ldq, scales, groups, G);
    return launch_status();
}

static int run_block128(const void* w, int64_t N, int64_t K, int64_t ldw, uint8_t* qb, int64_t ldqb,
                        void* sb, bool e8, void* stream) {
    int rc = check_bf16_matrix(w, N, K, ldw, qb, ldqb, 128);
    if (rc != FP8Q_OK) return rc;
    if (N == 0 || K == 0) return FP8Q_OK;
    if (!sb) return FP8Q_ERR_INVALID_ARG;
    if (!e8 && !aligned4(sb)) return FP8Q_ERR_MISALIGNED;
    if ((N + 127) / 128 > 65535) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d)) != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t G = K / 128;
    dim3 grid(unsigned(G), unsigned((N + 127) / 128));
    const uint16_t* ws = static_cast<const uint16_t*>(w);
    if (e8) launch(block128_quant_kernel<true>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, ws, N, ldw, qb, ldqb, sb, G);
    else launch(block128_quant_kernel<false>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, ws, N, ldw, qb, ldqb, sb, G);
    return launch_status();
}

int fp8_act_quant_group128(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                           int64_t ldq, float* scales, void* stream) {
    return run_group128(x, M, K, ldx, q, ldq, scales, false, stream);
}

int fp8_weight_quant_block128(const void* w, int64_t N, int64_t K, int64_t ldw, uint8_t* qb,
                              int64_t ldqb, float* sb, void* stream) {
    return run_block128(w, N, K, ldw, qb, ldqb, sb, false, stream);
}

int fp8_act_quant_per_channel(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                              int64_t ldq, float* scales, void* stream) {
    int rc = check_bf16_matrix(x, M, K, ldx, q, ldq, 8);
    if (rc != FP8Q_OK) return rc;
    if (M == 0) return FP8Q_OK;
    if (!scales) return FP8Q_ERR_INVALID_ARG;
    if (!aligned4(scales)) return FP8Q_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d)) != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int grid = int(std::max<int64_t>(1, std::min<int64_t>(M, int64_t(d->sms) * kBlocksPerSm)));
    if (log_enabled())
        std::fprintf(stderr, "[fp8q] per_channel M=%lld K=%lld: grid=%d\n", (long long)M, (long long)K, grid);
    launch(per_channel_quant_kernel<4>, dim3(grid), dim3(kQuantThreads), 0, st, 1u, static_cast<const uint16_t*>(x), M, K / 8, ldx,
                                                            q, ldq, scales);
    return launch_status();
}

int fp8_act_quant_group128_ue8m0(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                                 int64_t ldq, uint8_t* scales, void* stream) {
    return run_group128(x, M, K, ldx, q, ldq, scales, true, stream);
}

int fp8_weight_quant_block128_ue8m0(const void* w, int64_t N, int64_t K, int64_t ldw, uint8_t* qb,
                                    int64_t ldqb, uint8_t* sb, void* stream) {
    return run_block128(w, N, K, ldw, qb, ldqb, sb, true, stream);
}

// ------------------------------------------------------------ GEMM
size_t fp8_block_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 128) return 0;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != FP8Q_OK) return 0;
    // the ue8m0 GEMM never runs as CTA pairs: size for both plans
    return std::max(plan_gemm(M, N, K, d->sms).ws_bytes, plan_gemm(M, N, K, d->sms, true).ws_bytes);
}

}  // extern "C"

// Host-side argument checks shared by every GEMM entry point, run before
// anything touches the device, in this order: negative sizes, unsupported
// shapes (K % 128, sizes beyond INT_MAX), empty products (FP8Q_OK with
// *empty set: nothing to do), null pointers, leading dimensions, alignment.
// mode as in run_gemm.
static int check_gemm_args(int mode, const uint8_t* qa, int64_t lda, const float* sa, const uint8_t* qb,
                           int64_t ldb, const float* sb, const void* y, int64_t ldy, int64_t M, int64_t N,
                           int64_t K, bool* empty) {
    const bool ue8m0 = mode == 2;
    *empty = false;
    if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARG;
    if (K % 128) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) { *empty = true; return FP8Q_OK; }
    if (!qa || !sa || !qb || !sb || !y) return FP8Q_ERR_INVALID_ARG;
    if (lda < K || ldb < K || ldy < N) return FP8Q_ERR_INVALID_ARG;
    if (!aligned16(qa) || lda % 16 || !aligned16(qb) || !aligned16(y) || ldb % 16 || (ldy * 2) % 16 ||
        (!ue8m0 && (!aligned4(sa) || !aligned4(sb))))
        return FP8Q_ERR_MISALIGNED;
    return FP8Q_OK;
}

static int run_gemm(const uint8_t* qa, int64_t lda, const float* sa, const uint8_t* qb, int64_t ldb,
                    const float* sb, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                    void* workspace, size_t workspace_bytes, void* stream, int mode, bool pdl = false,
                    size_t ws_cap = ~size_t(0)) {
    // mode 0: fp32 block scales; 1: per-tensor fp32 scales; 2: ue8m0 bytes;
    // 3: per-channel fp32 scales.  pdl: the weights do not depend on the
    // previous kernel on the stream (it writes only qa and sa).
    const bool per_tensor = mode == 1, ue8m0 = mode == 2, per_channel = mode == 3;
    bool empty = false;
    int rc = check_gemm_args(mode, qa, lda, sa, qb, ldb, sb, y, ldy, M, N, K, &empty);
    if (rc != FP8Q_OK || empty) return rc;
    DeviceInfo* d = nullptr;
    rc = device_info(&d);
    if (rc != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        // Empty sum: Y = 0.
        return cudaMemset2DAsync(y, size_t(ldy) * 2, 0, size_t(N) * 2, size_t(M), st) == cudaSuccess
                   ? FP8Q_OK : FP8Q_ERR_CUDA;
    }
    // CTA pairs for every scale mode but ue8m0, which has none (with the
    // bulk-store epilogue the per-tensor GEMM runs 4096 x 7168 x 7168 in
    // 168.3 against 177.2 us with pairs, the same at N = 18432-24576)
    const GemmPlan pl = plan_gemm(M, N, K, d->sms, mode == 2, ws_cap);
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return FP8Q_ERR_WORKSPACE;
        if (!aligned16(workspace)) return FP8Q_ERR_MISALIGNED;
    }
    CUtensorMap tp, tq;
    const uint8_t* P = pl.swap ? qb : qa;
    const uint8_t* Q = pl.swap ? qa : qb;
    const int64_t rows_p = pl.swap ? N : M, rows_q = pl.swap ? M : N;
    const int64_t ld_p = pl.swap ? ldb : lda, ld_q = pl.swap ? lda : ldb;
    if (!make_tmap(&tp, P, rows_p, K, ld_p, 128)) return FP8Q_ERR_CUDA;
    if (!make_tmap(&tq, Q, rows_q, K, ld_q, pl.pair ? pl.bn / 2 : pl.bn)) return FP8Q_ERR_CUDA;
    GemmParams p;
    p.sa = sa;
    p.sb = sb;
    p.y = static_cast<uint16_t*>(y);
    p.ws = static_cast<float*>(workspace);
    p.ldy = ldy;
    p.ldw = pl.ldw;
    p.M = int(M);
    p.N = int(N);
    p.G = int(K / 128);
    p.tiles_p = pl.tiles_p;
    p.splits = pl.splits;
    p.units = pl.units;
    p.full_units = pl.tail_tiles > 0 ? pl.full_tiles : pl.units;
    p.full_tiles = pl.full_tiles;
    p.tail_splits = pl.tail_splits;
    p.scale_vec4 = mode == 0 && (p.G % 4 == 0) && aligned16(sa) && aligned16(sb);
    p.sf_words = ue8m0 && (p.G % 4 == 0) && aligned4(sa) && aligned4(sb);
    p.pdl = (pdl && mode == 0 && !pl.pair) ? 1 : 0;
    // Normal 128/256-wide tiles stage the block scales through shared memory
    // (TMA boxes of 4 K blocks) when the scale rows allow 16-byte boxes.
    const bool staged = p.scale_vec4 && !pl.swap && !pl.pair && (pl.bn == 128 || pl.bn == 256);
    CUtensorMap tsa = tp, tsb = tq;
    if (staged && (!make_scale_tmap(&tsa, sa, M, p.G, 128) ||
                   !make_scale_tmap(&tsb, sb, (N + 127) / 128, p.G, pl.bn / 128)))
        return FP8Q_ERR_CUDA;
    p.wait_budget = wait_budget_cycles();
    p.status_slot = uint8_t(status_slot(d->index, st));
    // CTA-pair 256 x 256 tiles store Y in bulk from shared memory
    // (check_gemm_args has made Y's base and row pitch 16-byte aligned, as
    // the tensor map needs).
    CUtensorMap ty = tp;
    p.ystore = 0;
    if (pl.pair && pl.bn == 256 && mode != 2) {
        if (!make_y_tmap(&ty, y, M, N, ldy)) return FP8Q_ERR_CUDA;
        p.ystore = 1;
    }
    if (log_enabled())
        std::fprintf(stderr, "[fp8q] gemm M=%lld N=%lld K=%lld: %s%s bn=%d stages=%d splits=%d units=%d grid=%d"
                             " tail=%dx%d\n",
                     (long long)M, (long long)N, (long long)K,
                     pl.swap ? "swap" : pl.pair ? "pair" : "normal", staged ? " (staged scales)" : "", pl.bn,
                     pl.stages, pl.splits, pl.units, pl.grid, pl.tail_tiles, pl.tail_splits);
    if (per_channel) {
        if (pl.pair) {
            if (pl.bn == 256) launch_gemm<256, false, 5, true, 3>(tp, tq, tsa, tsb, p, pl.grid, st, &ty);
            else launch_gemm<128, false, 8, true, 3>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else if (pl.swap) {
            switch (pl.bn) {
                case 16: launch_gemm<16, true, 12, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                case 32: launch_gemm<32, true, 10, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                case 64: launch_gemm<64, true, 8, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                default: launch_gemm<128, true, 6, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st); break;
            }
        } else if (pl.bn == 128) {
            launch_gemm<128, false, 6, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else if (pl.bn == 192) {
            launch_gemm<192, false, 5, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else {
            launch_gemm<256, false, 4, false, 3>(tp, tq, tsa, tsb, p, pl.grid, st);
        }
    } else if (ue8m0) {
        if (pl.swap) {
            switch (pl.bn) {
                case 16: launch_gemm<16, true, 12, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                case 32: launch_gemm<32, true, 10, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                case 64: launch_gemm<64, true, 8, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                default: launch_gemm<128, true, 6, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st); break;
            }
        } else if (pl.bn == 128) {
            launch_gemm<128, false, 6, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else if (pl.bn == 192) {
            launch_gemm<192, false, 5, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else {
            launch_gemm<256, false, 4, false, 2>(tp, tq, tsa, tsb, p, pl.grid, st);
        }
    } else if (per_tensor) {
        if (pl.pair) {
            if (pl.bn == 256) launch_gemm<256, false, 5, true, 1>(tp, tq, tsa, tsb, p, pl.grid, st, &ty);
            else launch_gemm<128, false, 8, true, 1>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else if (pl.swap) {
            switch (pl.bn) {
                case 16: launch_gemm<16, true, 12, false, true>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                case 32: launch_gemm<32, true, 10, false, true>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                case 64: launch_gemm<64, true, 8, false, true>(tp, tq, tsa, tsb, p, pl.grid, st); break;
                default: launch_gemm<128, true, 6, false, true>(tp, tq, tsa, tsb, p, pl.grid, st); break;
            }
        } else if (pl.bn == 128) {
            launch_gemm<128, false, 6, false, true>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else if (pl.bn == 192) {
            launch_gemm<192, false, 5, false, true>(tp, tq, tsa, tsb, p, pl.grid, st);
        } else {
            launch_gemm<256, false, 4, false, true>(tp, tq, tsa, tsb, p, pl.grid, st);
        }
    } else if (pl.swap) {
        switch (pl.bn) {
            case 16: launch_gemm<16, true, 12>(tp, tq, tsa, tsb, p, pl.grid, st); break;
            case 32: launch_gemm<32, true, 10>(tp, tq, tsa, tsb, p, pl.grid, st); break;
            case 64: launch_gemm<64, true, 8>(tp, tq, tsa, tsb, p, pl.grid, st); break;
            default: launch_gemm<128, true, 6>(tp, tq, tsa, tsb, p, pl.grid, st); break;
        }
    } else if (pl.pair) {
        if (pl.bn == 256) launch_gemm<256, false, 5, true>(tp, tq, tsa, tsb, p, pl.grid, st, &ty);
        else launch_gemm<128, false, 8, true>(tp, tq, tsa, tsb, p, pl.grid, st);
    } else {
        if (pl.bn == 192) launch_gemm<192, false, 5>(tp, tq, tsa, tsb, p, pl.grid, st);
        else if (pl.bn == 256 && staged) launch_gemm<256, false, 4, false, false, true>(tp, tq, tsa, tsb, p, pl.grid, st);
        else if (pl.bn == 256) launch_gemm<256, false, 4>(tp, tq, tsa, tsb, p, pl.grid, st);
        else if (staged) launch_gemm<128, false, 6, false, false, true>(tp, tq, tsa, tsb, p, pl.grid, st);
        else launch_gemm<128, false, 6>(tp, tq, tsa, tsb, p, pl.grid, st);
    }
    if ((rc = launch_status()) != FP8Q_OK) return rc;
    if (pl.splits > 1) {
        const int64_t total = M * ((N + 3) / 4);
        const int g = int(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, int64_t(d->sms) * 8)));
        launch(splitk_reduce_kernel, dim3(g), dim3(256), 0, st, 1u, p.ws, pl.splits, p.M, p.N, pl.ldw, p.y, ldy);
        rc = launch_status();
    } else if (pl.tail_tiles > 0) {
        const int tile_rows = pl.pair ? 256 : 128;
        const int64_t total = int64_t(pl.tail_tiles) * tile_rows * (pl.bn / 4);
        const int g = int(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, int64_t(d->sms) * 8)));
        launch(tail_reduce_kernel, dim3(g), dim3(256), 0, st, 1u, p.ws, pl.tail_tiles, pl.tail_splits, pl.full_tiles,
                                              pl.tiles_p, tile_rows, pl.bn, p.M, p.N, p.y, ldy);
        rc = launch_status();
    }
    return rc;
}

extern "C" {

int fp8_block_gemm(const uint8_t* qa, int64_t lda, const float* sa, const uint8_t* qb, int64_t ldb,
                   const float* sb, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                   void* workspace, size_t workspace_bytes, void* stream) {
    return run_gemm(qa, lda, sa, qb, ldb, sb, y, ldy, M, N, K, workspace, workspace_bytes, stream, 0);
}

int fp8_gemm_per_tensor(const uint8_t* qa, int64_t lda, const float* sa, const uint8_t* qb, int64_t ldb,
                        const float* sb, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, void* stream) {
    return run_gemm(qa, lda, sa, qb, ldb, sb, y, ldy, M, N, K, workspace, workspace_bytes, stream, 1);
}

// ------------------------------------------------------------ one-call linear
// Group-128 quantisation of x into the workspace, then the block GEMM on
// it, launched as a programmatic dependent of the quantisation: its
// producer issues the weight loads of its first pipeline stages (weights
// do not depend on the quantisation) before it waits for the codes.
// Workspace layout: codes [M, K], then the group scales [M, K/128] fp32,
// then the GEMM's split-K partials.
static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

size_t fp8_linear_group128_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 128) return 0;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != FP8Q_OK) return 0;
    const GemmPlan pl = plan_gemm(M, N, K, d->sms);
    return round256(size_t(M) * size_t(K)) + round256(size_t(M) * size_t(K / 128) * 4) + pl.ws_bytes;
}

int fp8_linear_group128(const void* x, int64_t ldx, const uint8_t* qb, int64_t ldb, const float* sb,
                        void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, void* stream) {
    if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARG;
    if (K % 128 || M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return FP8Q_OK;
    if (!x || !qb || !sb || !y) return FP8Q_ERR_INVALID_ARG;
    if (ldx < K || ldb < K || ldy < N) return FP8Q_ERR_INVALID_ARG;
    if (!aligned16(x) || (ldx * 2) % 16 || !aligned16(qb) || ldb % 16 || !aligned4(sb) || !aligned16(y) ||
        (ldy * 2) % 16)
        return FP8Q_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc != FP8Q_OK) return rc;
    const GemmPlan pl = plan_gemm(M, N, K, d->sms);
    const size_t need = fp8_linear_group128_workspace_size(M, N, K);
    if (!workspace || workspace_bytes < need) return FP8Q_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP8Q_ERR_MISALIGNED;
    uint8_t* qa = static_cast<uint8_t*>(workspace);
    float* sa = reinterpret_cast<float*>(qa + round256(size_t(M) * size_t(K)));
    uint8_t* gws = reinterpret_cast<uint8_t*>(sa) + round256(size_t(M) * size_t(K / 128) * 4);
    if ((rc = run_group128(x, M, K, ldx, qa, K, sa, false, stream)) != FP8Q_OK) return rc;
    return run_gemm(qa, K, sa, qb, ldb, sb, y, ldy, M, N, K, gws, pl.ws_bytes, stream, 0, true);
}

int fp8_gemm_per_channel(const uint8_t* qa, int64_t lda, const float* sa, const uint8_t* qb, int64_t ldb,
                         const float* sb, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream) {
    return run_gemm(qa, lda, sa, qb, ldb, sb, y, ldy, M, N, K, workspace, workspace_bytes, stream, 3);
}

int fp8_block_gemm_ue8m0(const uint8_t* qa, int64_t lda, const uint8_t* sa, const uint8_t* qb, int64_t ldb,
                         const uint8_t* sb, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream) {
    return run_gemm(qa, lda, reinterpret_cast<const float*>(sa), qb, ldb, reinterpret_cast<const float*>(sb),
                    y, ldy, M, N, K, workspace, workspace_bytes, stream, 2);
}

// ------------------------------------------------------------ GEMM, no allocation
int fp8_block_gemm_noalloc(const uint8_t* qa, int64_t lda, const float* sa, const uint8_t* qb,
                           int64_t ldb, const float* sb, void* y, int64_t ldy, int64_t M, int64_t N,
                           int64_t K, void* stream) {
    // Argument errors first, with fp8_block_gemm's checks and codes, before
    // the device is queried or the launch is planned against the scratch.
    bool empty = false;
    int rc = check_gemm_args(0, qa, lda, sa, qb, ldb, sb, y, ldy, M, N, K, &empty);
    if (rc != FP8Q_OK || empty) return rc;
    DeviceInfo* d = nullptr;
    rc = device_info(&d);
    if (rc != FP8Q_OK) return rc;
    // the launch is planned to fit the scratch (fewer K splits); only a swapped
    // skinny shape that needs 2+ splits larger than the scratch is refused
    if (plan_gemm(M, N, K, d->sms, false, kNoAllocScratchBytes).ws_bytes > kNoAllocScratchBytes)
        return FP8Q_ERR_WORKSPACE;
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != FP8Q_OK) return rc;
    return run_gemm(qa, lda, sa, qb, ldb, sb, y, ldy, M, N, K, scratch, kNoAllocScratchBytes, stream, 0,
                    false, kNoAllocScratchBytes);
}

// ------------------------------------------------------------ status
unsigned long long fp8q_launch_count(void) {
    return g_launches.load(std::memory_order_relaxed);
}

int fp8q_device_status(int* status, int reset) {
    if (!status) return FP8Q_ERR_INVALID_ARG;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc != FP8Q_OK) return rc;
    if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); return FP8Q_ERR_CUDA; }
    int v[kStatusSlots];
    if (cudaMemcpyFromSymbol(v, g_stream_status, sizeof(v)) != cudaSuccess) { cudaGetLastError(); return FP8Q_ERR_CUDA; }
    *status = FP8Q_OK;
    for (int i = 0; i < kStatusSlots && *status == FP8Q_OK; ++i) *status = v[i];
    if (reset) {
        std::memset(v, 0, sizeof(v));
        if (cudaMemcpyToSymbol(g_stream_status, v, sizeof(v)) != cudaSuccess) { cudaGetLastError(); return FP8Q_ERR_CUDA; }
    }
    return FP8Q_OK;
}

long long fp8q_set_wait_budget_cycles(long long cycles) {
    const long long prev = wait_budget_cycles();
    g_wait_budget_override.store(cycles < 0 ? -1 : cycles, std::memory_order_relaxed);
    return prev;
}

int fp8q_get_last_device_status(void* stream, int* status) {
    if (!status) return FP8Q_ERR_INVALID_ARG;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc != FP8Q_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t off = size_t(status_slot(d->index, st)) * sizeof(int);
    int v = 0;
    const int z = 0;
    // the copies are ordered after this stream's kernels; only this stream waits
    if (cudaMemcpyFromSymbolAsync(&v, g_stream_status, sizeof(int), off, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    if (v != 0 && (cudaMemcpyToSymbolAsync(g_stream_status, &z, sizeof(int), off, cudaMemcpyHostToDevice, st) != cudaSuccess ||
                   cudaStreamSynchronize(st) != cudaSuccess)) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    *status = v;
    return FP8Q_OK;
}

}  // extern "C"
