/*
 * fp8q -- C ABI of the FP8 (E4M3) dynamic-quantisation linear path on
 * NVIDIA B200 (sm_100a).
 *
 * The path has two halves:
 *   1. dynamic activation quantisation: an exact amax reduction (over the
 *      whole tensor, or per 1x128 group along K), scale = fl32(amax / 448),
 *      codes = e4m3_rne_sat(fl32(x / scale));
 *   2. the block-scaled FP8 GEMM that consumes those codes: A scaled per
 *      1x128 group, B per 128x128 block, fp32 accumulation, bf16 output.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "How to Profile DeepSeek-V3 Inference Kernels Using Triton
 *        Autotuning": "Understanding the Autotuned Kernels in DeepSeek-V3"
 *        (block-wise activation quantisation producing FP8 values and
 *        per-block scales; FP8 GEMM with per-block scaling), "Benchmarking
 *        the FP8 GEMM Kernel" (BLOCK_SIZE_K = 128; codes plus scale tensors
 *        a_s, b_s), "Benchmarking the Activation Quantization Kernel"
 *        (act_quant(x, block_size=128) returns codes and scales).
 *   [P2] "Size the per-tensor FP8 dynamic-quant amax grid to the input"
 *        (TensorRT-LLM pull request 16569): "Description" (per-tensor amax
 *        with an input-sized grid, then an apply-only pass), "Test Coverage"
 *        (amax is exact; scale = amax / 448; bitwise-identical bytes), the
 *        review comments (strided 2-D inputs; NaN handling).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library allocates nothing per call; it enqueues work on `stream`
 *     (a cudaStream_t; NULL means the legacy default stream) and returns
 *     before the work completes.
 *   - Matrices are row-major with unit inner stride; `ld*` is the row
 *     stride in ELEMENTS (>= the row length).  bf16 tensors are passed as
 *     `const void*` holding IEEE bfloat16 bit patterns; E4M3 codes as
 *     uint8_t (OCP FP8 E4M3: 1 sign, 4 exponent, 3 mantissa bits, bias 7,
 *     no infinity, NaN = 0x7F/0xFF, max finite 448).
 *   - Alignment: bf16 matrices (inputs and the GEMM output) and the GEMM's
 *     code operands must be 16-byte aligned with row pitches (ld * element
 *     size) that are multiples of 16 bytes; code OUTPUTS of the quantisation
 *     calls 8-byte aligned with row pitches that are multiples of 8 bytes;
 *     scale pointers 4-byte aligned.  Otherwise FP8Q_ERR_MISALIGNED.
 *   - Arguments are checked on the host before anything is enqueued; on
 *     any error nothing is enqueued.  A failed launch returns FP8Q_ERR_CUDA.
 *   - Zero convention: an all-zero tensor (per-tensor path) or group (group
 *     and block paths) gets scale 0.0f and signed-zero codes (0x00, or 0x80
 *     where x is -0).  The GEMM consumes a zero scale as a zero
 *     contribution.
 *   - NaN / Inf: amax propagates NaN (any NaN makes amax NaN), else Inf.
 *     The scale is then non-finite and the codes are E4M3 of x / scale
 *     (NaN codes, or signed zeros for finite x over an infinite scale).
 *   - Determinism: the same inputs give the same bytes, whatever the
 *     launch configuration chosen.
 *   - Launches: every kernel is launched as a programmatic dependent of the
 *     work before it on `stream`.  It may be placed on the GPU while the
 *     previous kernel finishes, and waits for that kernel to complete
 *     before it touches global memory, so stream order holds as usual and
 *     the gap between back-to-back kernels shrinks.
 *   - Environment: FP8Q_LOG=1 prints the launch chosen for every call to
 *     stderr.  FP8Q_GEMM_TILE forces a GEMM launch mode and
 *     FP8Q_PER_TENSOR_PATH=twopass the two-pass per-tensor path (measurement);
 *     FP8Q_PDL=0 launches every kernel without programmatic dependent
 *     launch (measurement; see "Launches" below);
 *     FP8Q_WAIT_BUDGET_CYCLES bounds the GEMM's device-side waits (fault
 *     testing; fp8q_set_wait_budget_cycles changes it at run time); these
 *     are read once per process.  No environment variable changes the
 *     result of a call that completes.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned (as int) by every call. */
typedef enum fp8q_status {
    FP8Q_OK = 0,
    FP8Q_ERR_INVALID_ARG = 1,       /* null pointer, negative size, ld < row length */
    FP8Q_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of the required width */
    FP8Q_ERR_MISALIGNED = 3,        /* pointer or row pitch alignment violated */
    FP8Q_ERR_WORKSPACE = 4,         /* workspace missing or too small */
    FP8Q_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    FP8Q_ERR_TIMEOUT = 6,           /* a bounded device-side wait gave up */
    FP8Q_ERR_NO_DEVICE = 7          /* no usable sm_100 device */
} fp8q_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* fp8q_status_string(int status);

/* ABI version of this header, (major << 16) | minor. */
int fp8q_abi_version(void);

/* ------------------------------------------------------------------ */
/* Per-tensor dynamic quantisation  ([P2] Description, Test Coverage)  */
/* ------------------------------------------------------------------ */

/* Bytes of device workspace fp8_act_quant_per_tensor needs for an [M,K]
 * input (partial maxima of the amax pass; no zero fill needed).  Calls
 * sharing one workspace must be ordered (same stream, or joined). */
size_t fp8_act_quant_per_tensor_workspace_size(int64_t M, int64_t K);

/* x: bf16 [M,K], row stride ldx.  Writes codes q: uint8 [M,K], row stride
 * ldq, and *scale (one fp32 on the device) = fl32(amax / 448), with
 * amax = max |x| over the whole tensor (exact).  K must be a multiple of 8.
 * M == 0 or K == 0 writes scale 0 and nothing else.  Tensors of up to
 * 128K elements take a single launch of one thread-block cluster (up to 8
 * CTAs exchange their partial maxima through distributed shared memory);
 * larger ones take an amax pass with an input-sized grid and then an apply
 * pass that re-reads x in reverse order (its tail is still in L2). */
int fp8_act_quant_per_tensor(const void* x, int64_t M, int64_t K, int64_t ldx,
                             uint8_t* q, int64_t ldq, float* scale,
                             void* workspace, size_t workspace_bytes,
                             void* stream);

/* The two halves of the per-tensor path, for callers that combine the amax
 * of several shards (e.g. a max all-reduce across ranks) before applying.
 *
 * fp8_act_amax: writes *amax_bits (one uint32 on the device) = the bf16 bit
 * pattern of max |x| over x[M,K] (NaN > Inf > finite under unsigned order),
 * so the max of several shards' words is the amax of their union.
 * Workspace: fp8_act_amax_workspace_size(M, K) bytes; needs no zero fill. */
size_t fp8_act_amax_workspace_size(int64_t M, int64_t K);
int fp8_act_amax(const void* x, int64_t M, int64_t K, int64_t ldx,
                 uint32_t* amax_bits, void* workspace, size_t workspace_bytes,
                 void* stream);

/* fp8_act_quant_apply: scale = fl32(amax / 448) from *amax_bits (device),
 * written to *scale (device, may be NULL), and codes of x[M,K] into q. */
int fp8_act_quant_apply(const void* x, int64_t M, int64_t K, int64_t ldx,
                        const uint32_t* amax_bits, uint8_t* q, int64_t ldq,
                        float* scale, void* stream);

/* ------------------------------------------------------------------ */
/* Per-1x128-group quantisation along K ([P1] act_quant, block 128)    */
/* ------------------------------------------------------------------ */

/* x: bf16 [M,K] (row stride ldx), K a multiple of 128.  Writes codes
 * q: uint8 [M,K] (row stride ldq) and scales: fp32 [M, K/128] row-major
 * contiguous, scales[m*(K/128)+g] = fl32(amax(x[m,128g:128g+128]) / 448).
 * One pass over x; no workspace. */
int fp8_act_quant_group128(const void* x, int64_t M, int64_t K, int64_t ldx,
                           uint8_t* q, int64_t ldq, float* scales, void* stream);

/* ------------------------------------------------------------------ */
/* Per-128x128-block weight quantisation ([P1] b_s: one scale per      */
/* 128x128 block of the weight).  Auxiliary (offline) step.            */
/* ------------------------------------------------------------------ */

/* w: bf16 [N,K] (row stride ldw), K a multiple of 128.  Writes codes
 * qb: uint8 [N,K] (row stride ldqb) and sb: fp32 [ceil(N/128), K/128]
 * row-major contiguous; the last row block may hold fewer than 128 rows. */
int fp8_weight_quant_block128(const void* w, int64_t N, int64_t K, int64_t ldw,
                              uint8_t* qb, int64_t ldqb, float* sb, void* stream);

/* ------------------------------------------------------------------ */
/* The dynamic FP8 linear in one call: activation quantisation, then   */
/* the GEMM on its codes ([P1] "Analyzing FP8 Quantization Sensitivity": */
/* act_quant produces the scales that feed fp8_gemm, and its latency     */
/* matters at small batch).                                              */
/* ------------------------------------------------------------------ */

/* Workspace bytes fp8_linear_group128 needs for (M, N, K) on the current
 * device (0 when unused; no zero fill needed). */
size_t fp8_linear_group128_workspace_size(int64_t M, int64_t N, int64_t K);

/* y = block_gemm(act_quant_group128(x), sa; qb, sb): the result of
 * fp8_act_quant_group128 followed by fp8_block_gemm, bit for bit.
 *   x : bf16 [M,K] (row stride ldx, a multiple of 8; 16-byte aligned)
 *   qb: E4M3 [N,K] (row stride ldb), sb: fp32 [ceil(N/128), K/128]
 *   y : bf16 [M,N] (row stride ldy)
 * The quantisation kernel runs first and the GEMM is launched as its
 * programmatic dependent: the GEMM starts while the quantisation runs,
 * issues the weight halves of its first pipeline stages, and waits for the
 * quantisation only before reading the codes and scales (kept in the
 * workspace).  Argument errors as fp8_act_quant_group128 and
 * fp8_block_gemm; FP8Q_ERR_WORKSPACE for a missing or short workspace. */
int fp8_linear_group128(const void* x, int64_t ldx, const uint8_t* qb, int64_t ldb,
                        const float* sb, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* Per-channel scales ([P2] Description names a PER_CHANNEL mode of the */
/* dynamic-quant path and defines nothing more).  Reading: one fp32      */
/* scale per row of the quantised matrix -- a token of X, an output     */
/* channel of a weight W[N,K] -- scale = amax(row)/448, codes as in the */
/* per-tensor path (zero row: scale 0, signed-zero codes).              */
/* ------------------------------------------------------------------ */

/* x: bf16 [M,K] (row stride ldx, K a multiple of 8).  Writes q: uint8
 * [M,K] (row stride ldq) and scales: fp32 [M].  No workspace. */
int fp8_act_quant_per_channel(const void* x, int64_t M, int64_t K, int64_t ldx,
                              uint8_t* q, int64_t ldq, float* scales, void* stream);

/* Y[m,n] = bf16_rne( sa[m] * sb[n] * sum_k A[m,k] * B[n,k] ), fp32
 * accumulation of the sum in TMEM, the two scales applied in the epilogue.
 *   qa: E4M3 [M,K] (row stride lda), sa: fp32 [M] on the device
 *   qb: E4M3 [N,K] (row stride ldb), sb: fp32 [N] on the device
 *   y : bf16 [M,N] (row stride ldy)
 * Shapes, alignment, launch selection, workspace and errors as
 * fp8_block_gemm. */
int fp8_gemm_per_channel(const uint8_t* qa, int64_t lda, const float* sa,
                         const uint8_t* qb, int64_t ldb, const float* sb,
                         void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* ue8m0 (power-of-two) scales ([P1] Benchmarking the Activation        */
/* Quantization Kernel: act_quant(..., scale_fmt="ue8m0")).  The page   */
/* names the format only.  Reading: the scale is the smallest power of  */
/* two 2^e >= amax/448, e clamped to [-127, 127], stored as the E8M0    */
/* byte e + 127 (value 2^(b-127); 255 = NaN).  An all-zero group gets   */
/* byte 0; an Inf or NaN amax gives byte 255 and NaN codes (0x7F).      */
/* Codes are e4m3_rne(x * 2^-e): x * 2^-e is exact, so the one rounding  */
/* is the conversion, and |x * 2^-e| <= 448 means nothing saturates.     */
/* ------------------------------------------------------------------ */

/* As fp8_act_quant_group128, with E8M0 scale bytes: scales[m*(K/128)+g]
 * (uint8, contiguous).  No alignment requirement on scales. */
int fp8_act_quant_group128_ue8m0(const void* x, int64_t M, int64_t K, int64_t ldx,
                                 uint8_t* q, int64_t ldq, uint8_t* scales, void* stream);

/* As fp8_weight_quant_block128, with E8M0 scale bytes sb[nb*(K/128)+kb]
 * (uint8, [ceil(N/128), K/128] contiguous). */
int fp8_weight_quant_block128_ue8m0(const void* w, int64_t N, int64_t K, int64_t ldw,
                                    uint8_t* qb, int64_t ldqb, uint8_t* sb, void* stream);

/* ------------------------------------------------------------------ */
/* Block-scaled FP8 GEMM ([P1] FP8 GEMM with per-block scaling,         */
/* BLOCK_SIZE_K = 128)                                                  */
/* ------------------------------------------------------------------ */

/* Bytes of device workspace fp8_block_gemm needs for (M, N, K) on the
 * current device (split-K partial sums for skinny M, or those of a split
 * last wave; 0 when unused).  The workspace needs no zero fill. */
size_t fp8_block_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/* Y = A * B^T with block scales:
 *   Y[m,n] = bf16_rne( sum_kb sa[m,kb] * sb[n/128,kb]
 *                       * sum_{k in block kb} A[m,k] * B[n,k] )
 * accumulated in fp32 (the per-block partial from the tensor cores is
 * multiplied by sa*sb in fp32 registers and added to an fp32 sum).
 *   qa: E4M3 [M,K], row stride lda        sa: fp32 [M, K/128] contiguous
 *   qb: E4M3 [N,K], row stride ldb        sb: fp32 [ceil(N/128), K/128]
 *   y : bf16 [M,N], row stride ldy
 * K must be a multiple of 128; M, N >= 0 arbitrary (tails handled).
 * The launch (tile shape, operand swap, split-K) is chosen per shape from
 * a compiled table.  When whole 128-row tiles would leave a last wave that
 * fills at most half the SMs, the tiles of that wave are split along K and
 * their fp32 partials are added in fixed order by a second kernel (the
 * call then enqueues two kernels); results are deterministic for a given
 * shape and device.  A bounded device wait that gives up records
 * FP8Q_ERR_TIMEOUT in the error word of `stream`, read by
 * fp8q_get_last_device_status (or fp8q_device_status for every stream);
 * the call's output is then unspecified (the GEMM kernel stops writing it,
 * but a split-K or split-tail reduce that follows may write sums of
 * partials that were never computed). */
int fp8_block_gemm(const uint8_t* qa, int64_t lda, const float* sa,
                   const uint8_t* qb, int64_t ldb, const float* sb,
                   void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* Per-tensor-scaled FP8 GEMM ([P2] Description and walkthrough: the   */
/* linear method's dynamic path quantises the input per tensor, then    */
/* runs the projection GEMM on the codes with the tensor scales)         */
/* ------------------------------------------------------------------ */

/* Y = bf16_rne( sa * sb * sum_k A[m,k] * B[n,k] ), fp32 accumulation.
 *   qa: E4M3 [M,K] (row stride lda), sa: ONE fp32 on the device (A's scale)
 *   qb: E4M3 [N,K] (row stride ldb), sb: ONE fp32 on the device (B's scale)
 *   y : bf16 [M,N] (row stride ldy)
 * Shapes, alignment, launch selection and errors as fp8_block_gemm; the
 * workspace size is fp8_block_gemm_workspace_size(M, N, K).  With scalar
 * scales there is no per-block promotion: the tensor cores accumulate the
 * whole K range in TMEM and the epilogue multiplies by sa*sb once. */
int fp8_gemm_per_tensor(const uint8_t* qa, int64_t lda, const float* sa,
                        const uint8_t* qb, int64_t ldb, const float* sb,
                        void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* Block-scaled FP8 GEMM with ue8m0 scales (the GEMM of the ue8m0       */
/* variant above; scales applied by the tensor cores)                   */
/* ------------------------------------------------------------------ */

/* Y[m,n] = bf16_rne( sum_kb 2^(sa[m,kb]-127) * 2^(sb[n/128,kb]-127)
 *                     * sum_{k in block kb} A[m,k] * B[n,k] ), fp32 accumulation.
 *   qa: E4M3 [M,K], row stride lda     sa: E8M0 bytes [M, K/128] contiguous
 *   qb: E4M3 [N,K], row stride ldb     sb: E8M0 bytes [ceil(N/128), K/128]
 *   y : bf16 [M,N], row stride ldy
 * A scale byte of 255 (NaN) makes the outputs it touches NaN.  Shapes,
 * alignment (none on sa/sb), launch selection, workspace (size from
 * fp8_block_gemm_workspace_size) and errors as fp8_block_gemm.  The power-of-
 * two scales multiply the E4M3 products exactly inside the tensor cores
 * (tcgen05.mma kind::mxf8f6f4.block_scale), so the whole K range
 * accumulates in TMEM with no per-block promotion. */
int fp8_block_gemm_ue8m0(const uint8_t* qa, int64_t lda, const uint8_t* sa,
                         const uint8_t* qb, int64_t ldb, const uint8_t* sb,
                         void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* Block-scaled FP8 GEMM without any allocation                         */
/* ------------------------------------------------------------------ */

/* The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory: host frameworks and plugin interfaces that
 * hand a kernel only its input and output buffers and own every other byte
 * of the device; serving processes that reserve the whole device pool at
 * start-up, so that a later cudaMalloc would fail; and latency-critical
 * loops that cannot afford cudaMalloc/cudaFree (cudaFree synchronises the
 * device).
 *
 * Same operation, arguments, layouts and errors as fp8_block_gemm, minus
 * the workspace.  The split-K partial sums that fp8_block_gemm would put in
 * the caller's workspace go to a fixed scratch array inside the library
 * instead: FP8Q_NOALLOC_MAX_SCRATCH_BYTES (8 MiB) per device, reserved by
 * every device that loads the library until the process exits.  The launch
 * is planned to fit that scratch: where fp8_block_gemm would split K (or
 * its last wave, see fp8_block_gemm) into more partial sums than the
 * scratch holds, this call uses fewer K ranges, so its bytes can differ
 * from fp8_block_gemm's in rounding, within the same tolerance.  A shape is
 * rejected with FP8Q_ERR_WORKSPACE, before anything is enqueued, only when
 * even the fewest K ranges its launch allows do not fit: skinny M (at most
 * 32 rows, run with the operands swapped) with K > 8192 needs at least two
 * ranges, 2 * M * N * 4 bytes (N rounded up to a multiple of 8).  Use
 * fp8_block_gemm for those.
 *
 * The call allocates nothing: no cudaMalloc, cudaFree or allocating
 * library routine.  The first call on each device looks up the scratch
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture begins.  The scratch is
 * part of the library's device code, which CUDA loads onto a device when
 * a call first touches the library there (lazy module loading); that load
 * claims the 8 MiB.  A process that reserves the whole device pool at
 * start-up must therefore make its first fp8_block_gemm_noalloc call (with
 * real operands) or one fp8q_device_status call on each device before it
 * reserves the pool, as it must before any stream capture.
 *
 * All calls on a device share the one scratch array, which keeps the last
 * call's contents; each call overwrites every partial sum it reads, so no
 * clearing is needed.  Two calls whose executions overlap on the GPU (e.g.
 * on different streams without ordering) race on the scratch array and may
 * produce wrong results: order them. */
#define FP8Q_NOALLOC_MAX_SCRATCH_BYTES ((size_t)8 << 20)
int fp8_block_gemm_noalloc(const uint8_t* qa, int64_t lda, const float* sa,
                           const uint8_t* qb, int64_t ldb, const float* sb,
                           void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           void* stream);

/* ------------------------------------------------------------------ */
/* Device status                                                       */
/* ------------------------------------------------------------------ */

/* The launch plan fp8_block_gemm uses for (M, N, K) on a device with `sms`
 * SMs (fp8_gemm_per_tensor and fp8_gemm_per_channel use the same plan; the
 * ue8m0 GEMM runs one CTA where this plan has a CTA pair), with
 * the split-K partials (or those of a split last wave) limited to ws_cap
 * bytes (SIZE_MAX: no limit; fp8_block_gemm_noalloc plans with its
 * scratch size).  Host only: no device is touched, so it runs anywhere.
 * plan[0..10] receives: operands swapped (0/1), CTA pair (0/1), tile
 * width BN, pipeline stages, K splits, tiles along the MMA's M operand,
 * tiles along its N operand, work units, grid size, tail tiles split along
 * K, K ranges per tail tile.  *ws_bytes receives the workspace the plan
 * needs.  FP8Q_ERR_INVALID_ARG for non-positive sizes or null outputs,
 * FP8Q_ERR_UNSUPPORTED_SHAPE for K % 128 != 0.  The pages have no
 * counterpart: it exposes this library's launch selection for tests. */
int fp8q_gemm_plan(int64_t M, int64_t N, int64_t K, int sms, size_t ws_cap,
                   int* plan, size_t* ws_bytes);

/* Device-side errors.  A kernel that meets an error it cannot report
 * through its return value (a bounded wait that gave up: FP8Q_ERR_TIMEOUT)
 * records it in the error word of the stream it was launched on, and the
 * first error recorded stays until it is read and cleared.  Streams get
 * their own word in the order they first use one (255 per device); streams
 * beyond that share one word.  The pages have no counterpart: they define
 * no device-side failure. */

/* Waits for the work enqueued on `stream` (only that stream: it does not
 * synchronise the device), then stores in *status the first error a kernel
 * launched on it recorded since the last read (FP8Q_OK if none), and clears
 * it.  FP8Q_ERR_INVALID_ARG for a null status, FP8Q_ERR_CUDA if the stream
 * failed. */
int fp8q_get_last_device_status(void* stream, int* status);

/* Synchronises the current device and stores in *status the first error
 * recorded on any stream of it since the last reset (FP8Q_OK if none).
 * reset != 0 clears every stream's word afterwards. */
int fp8q_device_status(int* status, int reset);

/* Sets the bound on every device-side wait of the GEMM kernels launched
 * from now on, in SM clock cycles (default about two seconds, or
 * FP8Q_WAIT_BUDGET_CYCLES); a negative value restores the default.
 * Returns the bound in force before the call.  For fault testing: a bound
 * of 0 makes the first wait that is not already satisfied give up.  It
 * never changes the result of a call that completes. */
long long fp8q_set_wait_budget_cycles(long long cycles);

/* Number of kernels this library has launched in the process so far (all
 * devices, all streams); a diagnostic for benchmarks. */
unsigned long long fp8q_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
