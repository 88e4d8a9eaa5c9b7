/*
 * fp8q oracle -- plain, slow, obviously-correct CPU definition of the FP8
 * dynamic-quantisation linear path.  TEST INFRASTRUCTURE ONLY: it is called by
 * the test-suite, by the smoke check and by the benchmark's CPU-baseline leg,
 * never by the product path.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *  [P1] "How to Profile DeepSeek-V3 Inference Kernels Using Triton Autotuning"
 *       -- "Understanding the Autotuned Kernels in DeepSeek-V3" (block-wise
 *       activation quant producing FP8 values plus per-block scales; FP8 GEMM
 *       with per-block scaling), "Benchmarking the FP8 GEMM Kernel" (BLOCK_K =
 *       128, scale tensors a_s / b_s), "Benchmarking the Activation
 *       Quantization Kernel" (act_quant(x, block_size=128) returns (y, s)).
 *  [P2] "Size the per-tensor FP8 dynamic-quant amax grid to the input"
 *       (TensorRT-LLM pull request 16569) -- "Description" (per-tensor amax,
 *       then a separate apply pass), "Test Coverage / Correctness" (amax is an
 *       exact reduction, scale = amax / 448, bytes bitwise-identical), review
 *       comments (strided 2-D inputs; NaN parity between implementations).
 *  [P4] "The Surgical Precision Flip: Converting DeepSeek-V4's Indexer GEMM
 *       from FP32 to bf16 on Blackwell GPUs" -- "Assumptions and Their
 *       Validity", assumption 1: E4M3 is 1 sign, 4 exponent and 3 mantissa
 *       bits and widens to bf16 without loss.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes): scale = fl32(amax / 448) with one IEEE division, no bf16 rounding of
 * the scale; codes = e4m3_rne_sat(fl32(x / scale)) -- two roundings by
 * definition; an all-zero tensor or group gets scale 0 and signed-zero codes;
 * NaN propagates through amax; NaN codes are 0x7F (sign not significant).
 *
 * The ue8m0 variant ([P1] "Benchmarking the Activation Quantization Kernel"
 * passes scale_fmt="ue8m0" and says nothing more): the scale is a power of two
 * stored as an E8M0 byte b (value 2^(b-127), b = 255 is NaN), namely the
 * smallest 2^e >= amax/448, with e clamped to [-127, 127]; an all-zero group
 * gets b = 0; an Inf or NaN amax gives b = 255 and NaN codes (0x7F).  Codes
 * are e4m3_rne(x * 2^-e), exact before the one rounding.
 *
 * Everything below is loops over elements.  No SIMD intrinsics, no blocking,
 * no reordering beyond what the definitions say.  OpenMP only splits
 * independent rows / groups across threads.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* bf16 and fp32 bit views                                             */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an fp32 word, so widening is a 16-bit shift. */
static float bf16_bits_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t f32_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

int oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* E4M3 decode, from the format definition ([P4] assumption 1 gives   */
/* the 1/4/3 split; the exponent bias 7, the subnormals and the single */
/* NaN mantissa pattern with no infinity are the OCP FP8 E4M3 rules).  */
/* ------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 0x7;
    double v;
    if (e == 15 && m == 7) return NAN;          /* 0x7F and 0xFF */
    if (e == 0)
        v = ldexp((double)m, -9);               /* m/8 * 2^(1-7) */
    else
        v = ldexp((double)(8 + m), e - 10);     /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* ------------------------------------------------------------------ */
/* E4M3 encode with round-to-nearest-even and saturation to +-448.      */
/* Exact integer arithmetic on the fp32 bit pattern.                    */
/*   NaN            -> 0x7F                                             */
/*   |v| >= 448     -> sign | 0x7E (448); this includes +-Inf           */
/*   otherwise      -> nearest of the 127 finite magnitudes, ties to    */
/*                     the even significand, sign kept (so -0 and tiny  */
/*                     negatives give 0x80).                            */
/* ------------------------------------------------------------------ */
uint8_t oracle_e4m3_encode(float v) {
    uint32_t u = f32_bits(v);
    uint8_t sign = (uint8_t)((u >> 24) & 0x80);
    uint32_t a = u & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return 0x7F;                 /* NaN */
    if (a >= 0x43E00000u) return (uint8_t)(sign | 0x7E); /* |v| >= 448.0 */
    if (a == 0) return sign;

    /* |v| = M * 2^e2 exactly. */
    uint32_t E = a >> 23;
    uint64_t M;
    int e2;
    if (E == 0) { M = a & 0x7FFFFFu; e2 = -149; }
    else        { M = (a & 0x7FFFFFu) | 0x800000u; e2 = (int)E - 150; }

    /* k = floor(log2 |v|) */
    int bl = 0;
    for (uint64_t t = M; t; t >>= 1) bl++;
    int k = e2 + bl - 1;

    /* Spacing of E4M3 values around |v|: 2^(k-3) in the normal binades
       (k >= -6), 2^-9 in the subnormal range (k < -6). */
    int qe = (k < -6 ? -6 : k) - 3;
    int shift = qe - e2;            /* bits of M below the E4M3 quantum; >= 20 */
    uint64_t n;
    if (shift >= 64) {
        n = 0;                      /* far below half a quantum */
    } else {
        n = M >> shift;
        uint64_t rem = M & ((1ull << shift) - 1ull);
        uint64_t half = 1ull << (shift - 1);
        if (rem > half || (rem == half && (n & 1ull))) n++;
    }

    /* |q| = n * 2^qe.  Subnormal range: code = n (n == 8 is 2^-6, the
       smallest normal, whose code is also 8).  Normal range: n in [8,16];
       code = (biased exponent << 3) + (n - 8), which also carries n == 16
       into the next binade. */
    uint32_t code;
    if (k < -6) code = (uint32_t)n;
    else        code = ((uint32_t)(k + 7) << 3) + (uint32_t)(n - 8);
    return (uint8_t)(sign | code);
}

/* Bulk helpers used by the exhaustive tests. */
void oracle_e4m3_encode_bits(const uint32_t* bits, int64_t n, uint8_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        float f;
        memcpy(&f, &bits[i], 4);
        out[i] = oracle_e4m3_encode(f);
    }
}

void oracle_e4m3_encode_range(uint32_t first, int64_t n, uint8_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        uint32_t b = first + (uint32_t)i;
        float f;
        memcpy(&f, &b, 4);
        out[i] = oracle_e4m3_encode(f);
    }
}

/* ------------------------------------------------------------------ */
/* amax and scale ([P2] Description; Test Coverage / Correctness)       */
/* ------------------------------------------------------------------ */

/* max |x| over the slice x[r0:r1, c0:c1] of a row-major bf16 matrix with
   row stride ld.  -0 counts as 0.  Any NaN makes the result NaN, else any
   Inf makes it +Inf. */
static float amax_bf16(const uint16_t* x, int64_t ld, int64_t r0, int64_t r1,
                       int64_t c0, int64_t c1) {
    float best = 0.0f;
    int has_nan = 0;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t c = c0; c < c1; c++) {
            float v = bf16_bits_to_f32(x[r * ld + c]);
            if (isnan(v)) { has_nan = 1; continue; }
            float a = fabsf(v);
            if (a > best) best = a;
        }
    }
    return has_nan ? NAN : best;
}

/* scale = fl32(amax / 448): one IEEE fp32 division. */
float oracle_scale_from_amax(float amax) {
    volatile float num = amax;   /* keep the division in fp32 */
    return num / 448.0f;
}

/* One element's code given its scale: signed zero when the scale is 0
   (all-zero tensor or group), else e4m3_rne_sat(fl32(x / scale)). */
static uint8_t quant_one(uint16_t xb, float s) {
    float xv = bf16_bits_to_f32(xb);
    if (s == 0.0f) return (uint8_t)((xb >> 8) & 0x80);
    volatile float qv = xv / s;
    return oracle_e4m3_encode(qv);
}

float oracle_amax(const uint16_t* x, int64_t M, int64_t K, int64_t ldx) {
    /* Row maxima are independent; their max is order-free. */
    float best = 0.0f;
    int has_nan = 0;
    for (int64_t r = 0; r < M; r++) {
        float a = amax_bf16(x, ldx, r, r + 1, 0, K);
        if (isnan(a)) has_nan = 1;
        else if (a > best) best = a;
    }
    return has_nan ? NAN : best;
}

/* Per-tensor dynamic quantisation ([P2]): amax over the whole tensor,
   scale = amax/448, then the apply pass. */
void oracle_quant_per_tensor(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                             uint8_t* q, int64_t ldq, float* scale_out) {
    float amax = 0.0f;
    int has_nan = 0;
    #pragma omp parallel
    {
        float local = 0.0f;
        int lnan = 0;
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < M; r++) {
            float a = amax_bf16(x, ldx, r, r + 1, 0, K);
            if (isnan(a)) lnan = 1;
            else if (a > local) local = a;
        }
        #pragma omp critical
        {
            if (lnan) has_nan = 1;
            if (local > amax) amax = local;
        }
    }
    if (has_nan) amax = NAN;
    float s = oracle_scale_from_amax(amax);
    *scale_out = s;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; r++)
        for (int64_t c = 0; c < K; c++)
            q[r * ldq + c] = quant_one(x[r * ldx + c], s);
}

/* The apply-only step of the per-tensor path ([P2] Description: a separate
   pass quantises the input with the scale computed from the amax): amax is
   given as the bf16 bit pattern of its magnitude. */
void oracle_quant_apply(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                        uint16_t amax_bits, uint8_t* q, int64_t ldq, float* scale_out) {
    float s = oracle_scale_from_amax(bf16_bits_to_f32((uint16_t)(amax_bits & 0x7FFF)));
    *scale_out = s;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; r++)
        for (int64_t c = 0; c < K; c++)
            q[r * ldq + c] = quant_one(x[r * ldx + c], s);
}

/* Per-channel quantisation ([P2] Description names a PER_CHANNEL mode of the
   same dynamic-quant path and defines nothing more): one scale per row of the
   matrix -- a token of an activation, an output channel of a weight [N, K] --
   scale = amax(row) / 448, codes as in the per-tensor path. */
void oracle_quant_per_channel(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                              uint8_t* q, int64_t ldq, float* scales) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; r++) {
        float s = oracle_scale_from_amax(amax_bf16(x, ldx, r, r + 1, 0, K));
        scales[r] = s;
        for (int64_t c = 0; c < K; c++)
            q[r * ldq + c] = quant_one(x[r * ldx + c], s);
    }
}

/* Per-1x128-group quantisation along K ([P1] act_quant with block_size 128):
   for every row m and group g, amax over x[m, 128g : 128g+128], its own
   scale, and codes.  scales is [M, K/128] row-major. */
void oracle_quant_group128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                           uint8_t* q, int64_t ldq, float* scales) {
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; r++) {
        for (int64_t g = 0; g < G; g++) {
            float a = amax_bf16(x, ldx, r, r + 1, 128 * g, 128 * g + 128);
            float s = oracle_scale_from_amax(a);
            scales[r * G + g] = s;
            for (int64_t c = 128 * g; c < 128 * g + 128; c++)
                q[r * ldq + c] = quant_one(x[r * ldx + c], s);
        }
    }
}

/* Per-128x128-block weight quantisation ([P1] b_s holds one scale per
   128x128 block of the weight): W is [N, K] row-major; sb is
   [ceil(N/128), K/128] row-major; the last row-block may be short. */
void oracle_quant_block128(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                           uint8_t* q, int64_t ldq, float* sb) {
    int64_t G = K / 128;
    int64_t NB = (N + 127) / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t nb = 0; nb < NB; nb++) {
        int64_t r0 = nb * 128, r1 = (nb * 128 + 128 < N) ? nb * 128 + 128 : N;
        for (int64_t g = 0; g < G; g++) {
            float a = amax_bf16(w, ldw, r0, r1, 128 * g, 128 * g + 128);
            float s = oracle_scale_from_amax(a);
            sb[nb * G + g] = s;
            for (int64_t r = r0; r < r1; r++)
                for (int64_t c = 128 * g; c < 128 * g + 128; c++)
                    q[r * ldq + c] = quant_one(w[r * ldw + c], s);
        }
    }
}

/* ------------------------------------------------------------------ */
/* ue8m0 (power-of-two) scales ([P1] "Benchmarking the Activation        */
/* Quantization Kernel": act_quant(..., scale_fmt="ue8m0")).  The pages  */
/* name the format only; the reading is in the header comment above.    */
/* ------------------------------------------------------------------ */

/* E8M0 byte of the scale for a group amax: the smallest e in
   [-127, 127] with 448 * 2^e >= amax, plus the bias 127; 255 for Inf/NaN. */
int oracle_e8m0_from_amax(float amax) {
    if (isnan(amax) || isinf(amax)) return 255;
    double a = (double)amax;
    int e = -127;
    while (e < 127 && ldexp(448.0, e) < a) e++;
    return e + 127;
}

/* One element's code for an E8M0 scale byte: NaN (0x7F) for byte 255,
   else e4m3_rne(x * 2^-(b-127)) -- the product is exact in double. */
static uint8_t quant_one_e8m0(uint16_t xb, int b) {
    if (b == 255) return 0x7F;
    double v = (double)bf16_bits_to_f32(xb) * ldexp(1.0, 127 - b);
    return oracle_e4m3_encode((float)v);   /* |v| <= 448: exact in fp32 unless below 2^-126 */
}

void oracle_quant_group128_ue8m0(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                 uint8_t* q, int64_t ldq, uint8_t* sbytes) {
    int64_t G = K / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; r++) {
        for (int64_t g = 0; g < G; g++) {
            int b = oracle_e8m0_from_amax(amax_bf16(x, ldx, r, r + 1, 128 * g, 128 * g + 128));
            sbytes[r * G + g] = (uint8_t)b;
            for (int64_t c = 128 * g; c < 128 * g + 128; c++)
                q[r * ldq + c] = quant_one_e8m0(x[r * ldx + c], b);
        }
    }
}

void oracle_quant_block128_ue8m0(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                                 uint8_t* q, int64_t ldq, uint8_t* sbytes) {
    int64_t G = K / 128;
    int64_t NB = (N + 127) / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t nb = 0; nb < NB; nb++) {
        int64_t r0 = nb * 128, r1 = (nb * 128 + 128 < N) ? nb * 128 + 128 : N;
        for (int64_t g = 0; g < G; g++) {
            int b = oracle_e8m0_from_amax(amax_bf16(w, ldw, r0, r1, 128 * g, 128 * g + 128));
            sbytes[nb * G + g] = (uint8_t)b;
            for (int64_t r = r0; r < r1; r++)
                for (int64_t c = 128 * g; c < 128 * g + 128; c++)
                    q[r * ldq + c] = quant_one_e8m0(w[r * ldw + c], b);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Block-scaled FP8 GEMM ([P1] "FP8 GEMM with per-block scaling",       */
/* BLOCK_K = 128):                                                      */
/*   Y[m,n] = sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in kb} A[m,k]B[n,k]*/
/* A = qa [M,K] (row stride lda), B = qb [N,K] (row stride ldb), so      */
/* Y = A * B^T.  The inner per-block sum is exact in float64: every      */
/* product of two E4M3 values has at most 8 significant bits and lies in */
/* [2^-18, 448^2], so 128 of them sum without rounding.                  */
/* R receives the float64 result, T the same sum over |products| (the   */
/* magnitude term of the tolerance).  Either may be NULL.               */
/* ------------------------------------------------------------------ */
static void decode_table(double* t) {
    for (int c = 0; c < 256; c++) t[c] = oracle_e4m3_decode((uint8_t)c);
}

static void gemm_point(const double* dec, const uint8_t* qa, int64_t lda,
                       const float* sa, const uint8_t* qb, int64_t ldb,
                       const float* sb, int64_t K, int64_t m, int64_t n,
                       double* r_out, double* t_out) {
    int64_t G = K / 128;
    double R = 0.0, T = 0.0;
    for (int64_t kb = 0; kb < G; kb++) {
        double p = 0.0, pa = 0.0;
        for (int64_t k = kb * 128; k < kb * 128 + 128; k++) {
            double prod = dec[qa[m * lda + k]] * dec[qb[n * ldb + k]];
            p += prod;
            pa += fabs(prod);
        }
        double s = (double)sa[m * G + kb] * (double)sb[(n / 128) * G + kb];
        R += s * p;
        T += fabs(s) * pa;
    }
    *r_out = R;
    *t_out = T;
}

void oracle_block_gemm(const uint8_t* qa, int64_t lda, const float* sa,
                       const uint8_t* qb, int64_t ldb, const float* sb,
                       int64_t M, int64_t N, int64_t K, double* R, double* T) {
    double dec[256];
    decode_table(dec);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double r, t;
            gemm_point(dec, qa, lda, sa, qb, ldb, sb, K, m, n, &r, &t);
            if (R) R[m * N + n] = r;
            if (T) T[m * N + n] = t;
        }
    }
}

/* The same definition evaluated only at the listed (m, n) points. */
void oracle_block_gemm_points(const uint8_t* qa, int64_t lda, const float* sa,
                              const uint8_t* qb, int64_t ldb, const float* sb,
                              int64_t K, const int64_t* ms, const int64_t* ns,
                              int64_t npts, double* R, double* T) {
    double dec[256];
    decode_table(dec);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < npts; i++)
        gemm_point(dec, qa, lda, sa, qb, ldb, sb, K, ms[i], ns[i], &R[i], &T[i]);
}

/* bf16 round-to-nearest-even of a float64 value (the GEMM's output type).
   Integer arithmetic on the float64 bits; NaN -> 0x7FC0; overflow -> Inf. */
uint16_t oracle_f64_to_bf16(double v) {
    uint64_t u;
    memcpy(&u, &v, 8);
    uint16_t sign = (uint16_t)((u >> 48) & 0x8000);
    uint64_t a = u & 0x7FFFFFFFFFFFFFFFull;
    if (a > 0x7FF0000000000000ull) return 0x7FC0;
    if (a == 0x7FF0000000000000ull) return (uint16_t)(sign | 0x7F80);
    if (a == 0) return sign;
    int E = (int)(a >> 52);
    uint64_t M;
    int e2;
    if (E == 0) { M = a & 0xFFFFFFFFFFFFFull; e2 = -1074; }
    else        { M = (a & 0xFFFFFFFFFFFFFull) | (1ull << 52); e2 = E - 1075; }
    int bl = 0;
    for (uint64_t t = M; t; t >>= 1) bl++;
    int k = e2 + bl - 1;                      /* floor(log2 |v|) */
    /* bf16: 8 significant bits, min normal 2^-126, subnormal quantum 2^-133 */
    int qe = (k < -126 ? -126 : k) - 7;
    int shift = qe - e2;
    uint64_t n;
    if (shift <= 0) {
        n = M << (-shift);
    } else if (shift >= 64) {
        n = 0;
    } else {
        n = M >> shift;
        uint64_t rem = M & ((1ull << shift) - 1ull);
        uint64_t half = 1ull << (shift - 1);
        if (rem > half || (rem == half && (n & 1ull))) n++;
    }
    uint32_t code;
    if (k < -126) code = (uint32_t)n;                        /* subnormal */
    else          code = ((uint32_t)(k + 127) << 7) + (uint32_t)(n - 128);
    if (code >= 0x7F80u) return (uint16_t)(sign | 0x7F80);   /* overflow */
    return (uint16_t)(sign | code);
}

void oracle_f64_to_bf16_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; i++) out[i] = oracle_f64_to_bf16(v[i]);
}
