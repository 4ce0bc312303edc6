/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for NVFP4 block-scaled quantisation and
 * matrix multiplication.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library. The product path (libnvfp4 and its Python
 * binding) never calls it, and the two share no source: no header, table or helper.
 *
 * What is computed, and where the reference pages fix it:
 *   - Operands are NVFP4: 4-bit e2m1 values packed two per uint8 byte, with one
 *     float8_e4m3fn scale per block of 16 consecutive K elements.
 *     ("When a Benchmark Crashes: The Elusive FP4 GEMM Comparison on Blackwell SM120",
 *      section "Input Knowledge Required", item 3; "The Art of Reading the Manual",
 *      section "The Message": block_size=16, and section "Assumptions": two values per
 *      byte, scale shape (rows, K/16).)
 *   - The product is out[m,n] = alpha * sum_k deq(A)[m,k] * deq(B)[n,k] with bf16
 *     output and an explicit fp32 alpha ("The Moment the Zeros Disappeared",
 *     section "The Subject Message", items 1-3; "The Art of Reading the Manual",
 *     section "The Message", the mm_fp4 signature).
 *   - The pages give no quantisation recipe. The one used here is the common two-level
 *     NVFP4 recipe: a per-tensor global scale gs = 448*6/amax, a per-block scale
 *     amax_block/6*gs rounded to e4m3, and e2m1 codes of x*gs/scale. The order of the
 *     fp32 operations, the tie rule and the sign of zero codes are readings of this
 *     build, listed in the design notes; each function below states the one it uses.
 *   - MXFP4 (use_nvfp4=False): OCP MX e2m1 elements with an E8M0 power-of-two scale per
 *     32 elements (the MXFP4 section below). The CUDA library does not implement it; the
 *     functions are here so that a kernel can be checked against them.
 *
 * Parity pins (tests/test_oracle.py, tests/test_oracle_mx.py) check every function here
 * against something other than itself: torch's float8_e4m3fn conversion, brute-force nearest-value search, exact
 * rational arithmetic on small products, closed forms and invariants.
 *
 * Floating point: compile with -ffp-contract=off and without -ffast-math; every fp32
 * operation is then a single IEEE round-to-nearest-even operation (x86-64 SSE).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------
 * Value tables, written from the bit-field definitions of the two formats.
 * e2m1: sign | 2-bit exponent (bias 1) | 1-bit mantissa; exponent 0 is subnormal
 *       (value = m * 0.5). Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 * e4m3fn: sign | 4-bit exponent (bias 7) | 3-bit mantissa; exponent 0 is subnormal
 *       (value = m * 2^-9); S.1111.111 is NaN; there is no infinity; max = 448.
 * ---------------------------------------------------------------------------------- */
double oracle_e2m1_decode(int code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
    return s ? -mag : mag;
}

double oracle_e4m3_decode(int byte)
{
    int s = (byte >> 7) & 1;
    int e = (byte >> 3) & 15;
    int m = byte & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? m * ldexp(1.0, -9) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -mag : mag;
}

/* Round a non-negative double that holds an exact small multiple of 1/2 or finer to the
 * nearest integer, ties to the even integer. */
static double round_half_even(double q)
{
    double f = floor(q);
    double r = q - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* fp32 -> e4m3fn byte, round to nearest even, saturating finite values to +-448.
 * NaN maps to 0x7F (never produced by the quantiser for finite inputs). */
uint8_t oracle_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    int s = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(s | 0x7E);   /* anything at or above the max is max */
    if (a == 0.0) return (uint8_t)s;
    int e2;
    frexp(a, &e2);                                  /* a = f * 2^e2 with f in [0.5, 1) */
    int E = e2 - 1;                                 /* a in [2^E, 2^(E+1)) */
    if (E < -6) {
        /* subnormal range: values are n * 2^-9, n = 0..7; n = 8 is the smallest normal */
        double n = round_half_even(a * 512.0);
        return (uint8_t)(s | (int)n);
    }
    double n = round_half_even(ldexp(a, 3 - E));    /* 8 <= n <= 16 */
    if (n == 16.0) { n = 8.0; E += 1; }
    return (uint8_t)(s | ((E + 7) << 3) | ((int)n - 8));
}

/* fp32 -> e2m1 code, round to nearest with ties to the even code, saturating at +-6.
 * The thresholds are the midpoints of consecutive table values; at a midpoint the code
 * with mantissa bit 0 wins. The sign bit is the sign of the input, so a negative value
 * that rounds to zero gives code 0x8 (negative zero). */
uint8_t oracle_e2m1_encode(float y)
{
    int s = signbit(y) ? 8 : 0;
    float a = fabsf(y);
    int c;
    if (a <= 0.25f) c = 0;        /* tie 0.25: codes 0 (0.0) and 1 (0.5) -> 0 */
    else if (a < 0.75f) c = 1;    /* tie 0.75: codes 1 (0.5) and 2 (1.0) -> 2 */
    else if (a <= 1.25f) c = 2;   /* tie 1.25: codes 2 (1.0) and 3 (1.5) -> 2 */
    else if (a < 1.75f) c = 3;    /* tie 1.75: codes 3 (1.5) and 4 (2.0) -> 4 */
    else if (a <= 2.5f) c = 4;    /* tie 2.5:  codes 4 (2.0) and 5 (3.0) -> 4 */
    else if (a < 3.5f) c = 5;     /* tie 3.5:  codes 5 (3.0) and 6 (4.0) -> 6 */
    else if (a <= 5.0f) c = 6;    /* tie 5.0:  codes 6 (4.0) and 7 (6.0) -> 6 */
    else c = 7;                   /* (5, inf): 6.0, saturating */
    return (uint8_t)(s | c);
}

/* Elementwise versions over arrays (used by the exhaustive rounding checks), split over
 * nthreads threads by contiguous ranges. */
typedef struct {
    const float* x;
    uint8_t* out;
    int64_t begin, end;
    int which;         /* 0: e4m3, 1: e2m1 */
} encode_job;

static void* encode_range(void* arg)
{
    encode_job* j = (encode_job*)arg;
    if (j->which == 0)
        for (int64_t i = j->begin; i < j->end; ++i) j->out[i] = oracle_e4m3_encode(j->x[i]);
    else
        for (int64_t i = j->begin; i < j->end; ++i) j->out[i] = oracle_e2m1_encode(j->x[i]);
    return NULL;
}

static void encode_array(const float* x, int64_t n, uint8_t* out, int which, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    encode_job jobs[256];
    int64_t per = (n + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].x = x; jobs[t].out = out; jobs[t].which = which;
        jobs[t].begin = t * per < n ? t * per : n;
        jobs[t].end = (t + 1) * per < n ? (t + 1) * per : n;
        if (nthreads == 1) encode_range(&jobs[t]);
        else pthread_create(&th[t], NULL, encode_range, &jobs[t]);
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out, int nthreads)
{
    encode_array(x, n, out, 0, nthreads);
}

void oracle_e2m1_encode_array(const float* x, int64_t n, uint8_t* out, int nthreads)
{
    encode_array(x, n, out, 1, nthreads);
}

/* ------------------------------------------------------------------------------------
 * Quantisation (two-level NVFP4), step by step, fp32 round-to-nearest-even throughout.
 * ---------------------------------------------------------------------------------- */

/* Step 1: per-tensor global scale. gs = (448 * 6) / amax, or 1 when the tensor is all
 * zero, so that the largest block scale (amax/6 * gs) lands on e4m3's maximum, 448. */
float oracle_global_scale(const float* x, int64_t numel)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < numel; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) return 1.0f;
    return 2688.0f / amax;
}

/* Steps 2-7 for one row-major tensor x[rows, K] (row stride ld elements).
 * Output: q[rows, K/2] packed codes (element 2i in the low nibble of byte i),
 *         sf[rows, K/16] e4m3 block scales. K must be a multiple of 16. */
void oracle_quantize(const float* x, int64_t rows, int64_t K, int64_t ld, float gs,
                     uint8_t* q, uint8_t* sf)
{
    int64_t nblk = K / 16;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < nblk; ++j) {
            const float* blk = x + r * ld + 16 * j;
            /* step 2: block amax */
            float amax_b = 0.0f;
            for (int k = 0; k < 16; ++k) {
                float a = fabsf(blk[k]);
                if (a > amax_b) amax_b = a;
            }
            /* step 3: block scale in fp32, two separately rounded operations */
            float t = amax_b / 6.0f;
            float sf32 = t * gs;
            /* step 4: round the scale to e4m3 */
            uint8_t sfq = oracle_e4m3_encode(sf32);
            /* step 5: the decoded scale and the reciprocal used for the elements */
            float sfd = (float)oracle_e4m3_decode(sfq);
            float rcp = (sfd == 0.0f) ? 0.0f : gs / sfd;
            /* steps 6-7: element codes, packed two per byte, even k in the low nibble */
            for (int k = 0; k < 8; ++k) {
                float y0 = blk[2 * k] * rcp;
                float y1 = blk[2 * k + 1] * rcp;
                uint8_t c0 = oracle_e2m1_encode(y0);
                uint8_t c1 = oracle_e2m1_encode(y1);
                q[r * (K / 2) + 8 * j + k] = (uint8_t)(c0 | (c1 << 4));
            }
            sf[r * nblk + j] = sfq;
        }
    }
}

/* alpha = 1 / (gsA * gsB) in fp32: undoes both global scales in the GEMM epilogue. */
float oracle_alpha(float gs_a, float gs_b)
{
    float p = gs_a * gs_b;
    return 1.0f / p;
}

/* ------------------------------------------------------------------------------------
 * Dequantisation and the matrix product.
 * ---------------------------------------------------------------------------------- */

/* deq[r, k] = e2m1(q[r, k]) * e4m3(sf[r, k/16]) as doubles (exact: at most 6
 * significant bits). */
void oracle_dequantize(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t K,
                       double* deq)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = q[r * (K / 2) + k / 2];
            int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double s = oracle_e4m3_decode(sf[r * (K / 16) + k / 16]);
            deq[r * K + k] = oracle_e2m1_decode(code) * s;
        }
    }
}

typedef struct {
    const double* a;   /* [M, K] dequantised */
    const double* b;   /* [N, K] dequantised */
    double alpha;
    int64_t M, N, K;
    int64_t row_begin, row_end;
    double* v;         /* [M, N] alpha * sum_k a*b, one rounding of the exact sum */
    double* S;         /* [M, N] sum_k |a*b| (may be NULL) */
    int inexact;       /* set when a partial sum could exceed the exact fp64 range */
} gemm_job;

/* Every product a*b is an integer multiple of 2^-20 below 2^23 in magnitude, so fp64
 * accumulation is exact while |partial sums| <= sum |a*b| < 2^33. */
static const double EXACT_LIMIT = 8589934592.0; /* 2^33 */

static void* gemm_rows(void* arg)
{
    gemm_job* j = (gemm_job*)arg;
    for (int64_t m = j->row_begin; m < j->row_end; ++m) {
        const double* ar = j->a + m * j->K;
        for (int64_t n = 0; n < j->N; ++n) {
            const double* br = j->b + n * j->K;
            double acc = 0.0, s = 0.0;
            for (int64_t k = 0; k < j->K; ++k) {
                double p = ar[k] * br[k];
                acc += p;
                s += fabs(p);
            }
            if (s >= EXACT_LIMIT) j->inexact = 1;
            j->v[m * j->N + n] = j->alpha * acc;
            if (j->S) j->S[m * j->N + n] = s;
        }
    }
    return NULL;
}

/* v[m, n] = alpha * sum_k deqA[m, k] * deqB[n, k]; S[m, n] = sum_k |deqA*deqB|.
 * Rows of the output are split across nthreads threads; each element is summed in
 * ascending k by a single thread. Returns 1 if every sum was exact, 0 otherwise. */
int oracle_gemm_dequantized(const double* deqA, const double* deqB, double alpha,
                            int64_t M, int64_t N, int64_t K, double* v, double* S,
                            int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (M < nthreads) nthreads = (M > 0) ? (int)M : 1;
    pthread_t th[256];
    gemm_job jobs[256];
    int64_t per = (M + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        gemm_job* j = &jobs[t];
        j->a = deqA; j->b = deqB; j->alpha = alpha;
        j->M = M; j->N = N; j->K = K;
        j->row_begin = t * per;
        j->row_end = (t + 1) * per < M ? (t + 1) * per : M;
        j->v = v; j->S = S; j->inexact = 0;
        if (j->row_begin >= j->row_end) continue;
        if (nthreads == 1) { gemm_rows(j); continue; }
        pthread_create(&th[t], NULL, gemm_rows, j);
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t)
            if (jobs[t].row_begin < jobs[t].row_end) pthread_join(th[t], NULL);
    int exact = 1;
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].row_begin < jobs[t].row_end && jobs[t].inexact) exact = 0;
    return exact;
}

/* The full product from packed operands: dequantise both, then the plain sum. */
int oracle_gemm(const uint8_t* Aq, const uint8_t* sfA, const uint8_t* Bq, const uint8_t* sfB,
                float alpha, int64_t M, int64_t N, int64_t K, double* v, double* S,
                int nthreads)
{
    double* da = (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)K);
    double* db = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * (size_t)K);
    if (!da || !db) { free(da); free(db); return -1; }
    oracle_dequantize(Aq, sfA, M, K, da);
    oracle_dequantize(Bq, sfB, N, K, db);
    int exact = oracle_gemm_dequantized(da, db, (double)alpha, M, N, K, v, S, nthreads);
    free(da);
    free(db);
    return exact;
}

/* Grouped product for mixture-of-experts: rows [off[e], off[e+1]) of A (sorted by
 * expert) multiply expert e's weights B[e] (N rows of K) and scale by alpha[e].
 * Returns 1 if every sum was exact, 0 otherwise, -1 on allocation failure. */
int oracle_grouped_gemm(const uint8_t* Aq, const uint8_t* sfA, const uint8_t* Bq,
                        const uint8_t* sfB, const float* alpha, const int32_t* off,
                        int32_t E, int64_t N, int64_t K, double* v, double* S, int nthreads)
{
    int exact = 1;
    for (int32_t e = 0; e < E; ++e) {
        int64_t r0 = off[e], r1 = off[e + 1];
        if (r1 <= r0) continue;
        int ex = oracle_gemm(Aq + r0 * (K / 2), sfA + r0 * (K / 16),
                             Bq + (int64_t)e * N * (K / 2), sfB + (int64_t)e * N * (K / 16),
                             alpha[e], r1 - r0, N, K, v + r0 * N, S ? S + r0 * N : NULL,
                             nthreads);
        if (ex < 0) return -1;
        if (!ex) exact = 0;
    }
    return exact;
}

/* ------------------------------------------------------------------------------------
 * MXFP4: the variant the pages select with use_nvfp4=False ("The Art of Reading the
 * Manual", section "The Message", the mm_fp4 signature). The pages name the flag but do not
 * define the format; this is the OCP Microscaling (MX) v1.0 FP4 format: e2m1 elements, one
 * E8M0 scale (a bare power of two, 2^(byte - 127); byte 255 is NaN) per block of 32
 * consecutive K elements, no per-tensor scale. Quantisation follows the MX conversion
 * rule: shared_exp = floor(log2(amax_block)) - 2 (2 = the largest e2m1 exponent), clamped
 * to the E8M0 range [-127, 127], and codes = e2m1_rn_satfinite(x / 2^shared_exp). A block
 * of zeros gets byte 0 (the spec leaves log2(0) open; the smallest scale is the plainest
 * choice, and its codes are 0 whatever the scale).
 * ---------------------------------------------------------------------------------- */

/* E8M0 byte -> scale (exact). */
double oracle_e8m0_decode(int byte)
{
    if (byte == 255) return NAN;
    return ldexp(1.0, byte - 127);
}

/* x[rows, K] (row stride ld) -> q[rows, K/2] codes (element 2i in the low nibble of byte
 * i) and sf[rows, K/32] E8M0 bytes. */
void oracle_mx_quantize(const float* x, int64_t rows, int64_t K, int64_t ld, uint8_t* q,
                        uint8_t* sf)
{
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * ld;
        for (int64_t b = 0; b < K / 32; ++b) {
            float amax = 0.0f;
            for (int k = 0; k < 32; ++k) {
                float a = fabsf(xr[b * 32 + k]);
                if (a > amax) amax = a;
            }
            int shared_exp = -127;
            if (amax > 0.0f) {
                int e;
                frexp((double)amax, &e);             /* amax = f * 2^e, f in [0.5, 1) */
                shared_exp = (e - 1) - 2;            /* floor(log2(amax)) - 2 */
                if (shared_exp < -127) shared_exp = -127;
                if (shared_exp > 127) shared_exp = 127;
            }
            sf[r * (K / 32) + b] = (uint8_t)(shared_exp + 127);
            for (int k = 0; k < 32; k += 2) {
                /* x / 2^shared_exp is exact in double; below 2^-126 it is far under the
                 * smallest e2m1 step, so the conversion to float changes no code */
                float y0 = (float)ldexp((double)xr[b * 32 + k], -shared_exp);
                float y1 = (float)ldexp((double)xr[b * 32 + k + 1], -shared_exp);
                q[r * (K / 2) + (b * 32 + k) / 2] =
                    (uint8_t)(oracle_e2m1_encode(y0) | (oracle_e2m1_encode(y1) << 4));
            }
        }
    }
}

/* deq[r, k] = e2m1(q[r, k]) * 2^(sf[r, k/32] - 127) as doubles (exact). */
void oracle_mx_dequantize(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t K,
                          double* deq)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = q[r * (K / 2) + k / 2];
            int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            deq[r * K + k] = oracle_e2m1_decode(code) * oracle_e8m0_decode(sf[r * (K / 32) + k / 32]);
        }
    }
}

/* Exponent of the smallest nonzero unit of a dequantised operand: every nonzero element is
 * a multiple of 2^lsb (e2m1 values are multiples of 0.5). Returns 1 << 20 if all are zero. */
static int min_unit_exponent(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t K)
{
    int lsb = 1 << 20;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            int any = 0;
            for (int k = 0; k < 16; ++k)
                if (q[r * (K / 2) + b * 16 + k] & 0x77) any = 1;
            int e = (int)sf[r * (K / 32) + b] - 127 - 1;
            if (any && e < lsb) lsb = e;
        }
    return lsb;
}

/* v[m, n] = alpha * sum_k deqA[m, k] * deqB[n, k] with 32-element E8M0 blocks; S as for
 * NVFP4. Every product is a multiple of 2^(lsbA + lsbB), so the fp64 sum is exact while
 * sum |a*b| < 2^(53 + lsbA + lsbB). Returns 1 if every sum was exact, 0 otherwise, -1 on
 * allocation failure. */
int oracle_mx_gemm(const uint8_t* Aq, const uint8_t* sfA, const uint8_t* Bq, const uint8_t* sfB,
                   float alpha, int64_t M, int64_t N, int64_t K, double* v, double* S,
                   int nthreads)
{
    double* da = (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)K);
    double* db = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * (size_t)K);
    double* s = S ? S : (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)(N > 0 ? N : 1));
    if (!da || !db || !s) { free(da); free(db); if (!S) free(s); return -1; }
    oracle_mx_dequantize(Aq, sfA, M, K, da);
    oracle_mx_dequantize(Bq, sfB, N, K, db);
    oracle_gemm_dequantized(da, db, (double)alpha, M, N, K, v, s, nthreads);
    int lsb = min_unit_exponent(Aq, sfA, M, K) + min_unit_exponent(Bq, sfB, N, K);
    int exact = 1;
    if (lsb < (1 << 19)) {
        double limit = ldexp(1.0, 53 + lsb);
        for (int64_t i = 0; i < M * N; ++i)
            if (s[i] >= limit) exact = 0;
    }
    free(da);
    free(db);
    if (!S) free(s);
    return exact;
}

/* ------------------------------------------------------------------------------------
 * bf16 rounding of a double, directly (one rounding, nearest-even), as 16 raw bits.
 * bf16: sign | 8-bit exponent (bias 127) | 7-bit mantissa, IEEE subnormals and inf.
 * ---------------------------------------------------------------------------------- */
uint16_t oracle_bf16_bits(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t s = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;                                  /* a in [2^E, 2^(E+1)) */
    if (E < -126) {
        /* subnormal: multiples of 2^-133; n = 128 is the smallest normal (exponent 1) */
        double n = round_half_even(ldexp(a, 133));
        return (uint16_t)(s | (uint16_t)n);
    }
    double n = round_half_even(ldexp(a, 7 - E));     /* 128 <= n <= 256 */
    if (n == 256.0) { n = 128.0; E += 1; }
    if (E > 127) return (uint16_t)(s | 0x7F80);     /* overflow to infinity */
    return (uint16_t)(s | ((E + 127) << 7) | ((int)n - 128));
}

void oracle_bf16_bits_array(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_bits(v[i]);
}

/* ------------------------------------------------------------------------------------
 * fp16 rounding of a double (the out_dtype=float16 option of the mm_fp4 signature, "The Art
 * of Reading the Manual", section "The Message"), one rounding, nearest-even, as raw bits.
 * fp16: sign | 5-bit exponent (bias 15) | 10-bit mantissa, subnormals, inf above 65504.
 * ---------------------------------------------------------------------------------- */
uint16_t oracle_fp16_bits(double v)
{
    if (isnan(v)) return 0x7E00;
    uint16_t s = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;                                  /* a in [2^E, 2^(E+1)) */
    if (E < -14) {
        /* subnormal: multiples of 2^-24; n = 1024 is the smallest normal (exponent 1) */
        double n = round_half_even(ldexp(a, 24));
        return (uint16_t)(s | (uint16_t)n);
    }
    double n = round_half_even(ldexp(a, 10 - E));    /* 1024 <= n <= 2048 */
    if (n == 2048.0) { n = 1024.0; E += 1; }
    if (E > 15) return (uint16_t)(s | 0x7C00);      /* overflow to infinity */
    return (uint16_t)(s | ((E + 15) << 10) | ((int)n - 1024));
}

void oracle_fp16_bits_array(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_fp16_bits(v[i]);
}
