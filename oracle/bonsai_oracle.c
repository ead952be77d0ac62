/*
 * bonsai_oracle.c -- plain CPU checker for the Bonsai 2 ternary linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline / reference leg may load this library.  The
 * CUDA library never includes, links or calls it, and this file uses nothing
 * of the CUDA library: no header, table, constant or helper is shared.
 *
 * Everything here is the plain definition, written as scalar loops in float64:
 *
 *   1. packing / unpacking of trits t in {-1, 0, +1}:
 *        PTQ1_0 -- five trits per byte as a base-3 number, 26 bytes per group
 *                  of 128 weights (25 full bytes + one byte holding 3 trits);
 *        PQ2_0  -- one trit per 2-bit slot, 32 bytes per group of 128.
 *      Source: "27B 模型压到 5.95GB，推理能力还保住 98%" (allhereai.com), the
 *      paragraph on the two file packings (PTQ1_0 1.75 bits/weight, PQ2_0
 *      "each trit in a 2-bit slot", 2.13 bits/weight); and "Bonsai把 27B 大模型
 *      塞进手机的极端量化方案到底靠不靠谱" (wmrh.cn), section 关键机制 (the
 *      5 trits / 8 bits storage bound).
 *      PQ2_0 g64 -- PQ2_0's 2-bit slots with one FP16 scale per 64 weights instead of
 *                per 128 (the pages' Q2_0_g64 file, wmrh.cn page, 快速上手 and 后端支持
 *                现状): only the scale plane (N x K/64) and the group of each scale change.
 *      Q1_0   -- the 1-bit sibling: weights w in {-1, +1}, one bit each, 16 bytes
 *                per group of 128.  Source: "Bonsai把 27B 大模型塞进手机的极端量化
 *                方案到底靠不靠谱" (wmrh.cn), section 核心观点 (1-bit Bonsai, about
 *                1.125 bits/weight, 3.9 GB) and section 关键机制 (weights held to
 *                {-1, 1} or {-1, 0, 1} with an FP16 group-wise scale).
 *   2. the block Hadamard rotation of the activations, x' = blockdiag(Hn) x,
 *      with Hn = H_128 / sqrt(128) and H_128 the Sylvester matrix, written out
 *      as an explicit 128 x 128 matrix.  Source: allhereai.com page, the
 *      paragraph describing the method (block Hadamard rotation folded into
 *      storage) and the one on running the files (a Hadamard activation
 *      runtime is required); "Bonsai 2，把27B压进6个G" (10100.com), section
 *      它怎么做到的 (the input must receive the matching transform).
 *   3. the grouped product y[m][n] = sum_g s[n][g] * sum_j t[n][128g+j] x'[m][128g+j],
 *      one FP16 scale per 128 weights.  Source: allhereai.com page, the
 *      paragraph describing the method (ternary weights, one FP16 scale shared
 *      by every 128 weights).
 *   4. the SwiGLU step after a fused gate/up product, h = silu(gate) * up.
 *
 * Readings where the pages are silent (block size of the rotation, Sylvester
 * order and 1/sqrt(128) normalisation, base-3 digit order least significant
 * first, 2-bit slot order least significant first, code = trit + 1, padding
 * digits zero, 1-bit order least significant first with bit 1 = +1) are fixed here
 * exactly as the CUDA library's header states them, and are listed with their
 * reasons in the design notes.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -o liboracle.so bonsai_oracle.c -lm
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 128
#define ORACLE_FMT_PTQ1_0 1
#define ORACLE_FMT_PQ2_0 2
#define ORACLE_FMT_Q1_0 3
#define ORACLE_FMT_PQ2_0_G64 4 /* PQ2_0 codes, one scale per 64 weights */
#define ORACLE_PTQ1_GROUP_BYTES 26 /* 25 bytes x 5 trits + 1 byte x 3 trits */
#define ORACLE_INVALID_TRIT (-128) /* written by the unpackers for an invalid code */

/* ------------------------------------------------------------------ sizes */

/* Bytes of the packed trit plane (scales not included); -1 on a bad shape. */
long long oracle_packed_bytes(int fmt, long long N, long long K)
{
    if (N < 0 || K < 0 || K % ORACLE_GROUP != 0) return -1;
    if (fmt == ORACLE_FMT_PTQ1_0) return N * (K / ORACLE_GROUP) * ORACLE_PTQ1_GROUP_BYTES;
    if (fmt == ORACLE_FMT_PQ2_0) return N * (K / 4);
    if (fmt == ORACLE_FMT_Q1_0) return N * (K / 8);
    if (fmt == ORACLE_FMT_PQ2_0_G64) return N * (K / 4);
    return -1;
}

/* ------------------------------------------------------------------ PTQ1_0 */

/* Trits 'count' (<= 5) into one byte: digit d_i = t_i + 1, byte = sum_i d_i * 3^i.
 * Returns 0xFF (not a valid base-3 byte) if a trit is outside {-1, 0, +1}. */
static int ptq1_encode_byte(const int8_t *t, int count)
{
    int value = 0, power = 1;
    for (int i = 0; i < count; i++) {
        if (t[i] < -1 || t[i] > 1) return 0xFF;
        value += (t[i] + 1) * power;
        power *= 3;
    }
    return value;
}

/* One byte back into 'count' trits: d_i = floor(byte / 3^i) mod 3, t_i = d_i - 1.
 * A byte >= 243 = 3^5 is not a base-3 code: its trits become ORACLE_INVALID_TRIT
 * and the function returns 1. */
static int ptq1_decode_byte(int byte, int8_t *t, int count)
{
    if (byte >= 243) {
        for (int i = 0; i < count; i++) t[i] = ORACLE_INVALID_TRIT;
        return 1;
    }
    int rest = byte;
    for (int i = 0; i < count; i++) {
        t[i] = (int8_t)(rest % 3 - 1);
        rest /= 3;
    }
    return 0;
}

/* Trits of weight row 'n' occupy group g's bytes b = 0..25; byte b holds
 * weights 128g + 5b ... 128g + 5b + 4 (byte 25: the last three weights). */
static int ptq1_trits_in_byte(int b) { return b < 25 ? 5 : 3; }

/* N x K trits -> N x (K/128) x 26 bytes.  Returns the number of invalid trits. */
long long oracle_pack_ptq1(const int8_t *trits, uint8_t *packed, long long N, long long K)
{
    long long G = K / ORACLE_GROUP, bad = 0;
    for (long long n = 0; n < N; n++)
        for (long long g = 0; g < G; g++)
            for (int b = 0; b < ORACLE_PTQ1_GROUP_BYTES; b++) {
                const int8_t *t = trits + n * K + g * ORACLE_GROUP + 5 * b;
                int v = ptq1_encode_byte(t, ptq1_trits_in_byte(b));
                if (v == 0xFF) bad++;
                packed[(n * G + g) * ORACLE_PTQ1_GROUP_BYTES + b] = (uint8_t)v;
            }
    return bad;
}

/* Unpacks one row of PTQ1_0 bytes into K trits; returns the count of invalid bytes. */
static long long ptq1_unpack_row(const uint8_t *row, int8_t *t, long long K)
{
    long long G = K / ORACLE_GROUP, bad = 0;
    for (long long g = 0; g < G; g++)
        for (int b = 0; b < ORACLE_PTQ1_GROUP_BYTES; b++)
            bad += ptq1_decode_byte(row[g * ORACLE_PTQ1_GROUP_BYTES + b],
                                    t + g * ORACLE_GROUP + 5 * b, ptq1_trits_in_byte(b));
    return bad;
}

long long oracle_unpack_ptq1(const uint8_t *packed, int8_t *trits, long long N, long long K)
{
    long long bad = 0, row_bytes = (K / ORACLE_GROUP) * ORACLE_PTQ1_GROUP_BYTES;
    for (long long n = 0; n < N; n++)
        bad += ptq1_unpack_row(packed + n * row_bytes, trits + n * K, K);
    return bad;
}

/* Validator: counts bytes that are not canonical PTQ1_0 codes -- any byte >= 243,
 * and a last byte of a group whose padding digits 3 and 4 are not zero (>= 27). */
long long oracle_check_ptq1(const uint8_t *packed, long long N, long long K)
{
    long long groups = N * (K / ORACLE_GROUP), bad = 0;
    for (long long q = 0; q < groups; q++)
        for (int b = 0; b < ORACLE_PTQ1_GROUP_BYTES; b++) {
            int v = packed[q * ORACLE_PTQ1_GROUP_BYTES + b];
            if (v >= 243 || (b == ORACLE_PTQ1_GROUP_BYTES - 1 && v >= 27)) bad++;
        }
    return bad;
}

/* ------------------------------------------------------------------ PQ2_0 */

/* Weight k of a row sits in byte k/4 of the row, bits 2(k mod 4) and 2(k mod 4)+1,
 * as code c = t + 1.  An invalid trit is stored as code 3 (never a valid code). */
long long oracle_pack_pq2(const int8_t *trits, uint8_t *packed, long long N, long long K)
{
    long long bad = 0;
    for (long long n = 0; n < N; n++)
        for (long long byte = 0; byte < K / 4; byte++) {
            int v = 0;
            for (int i = 0; i < 4; i++) {
                int t = trits[n * K + 4 * byte + i];
                int code = (t >= -1 && t <= 1) ? t + 1 : 3;
                if (code == 3) bad++;
                v |= code << (2 * i);
            }
            packed[n * (K / 4) + byte] = (uint8_t)v;
        }
    return bad;
}

static long long pq2_unpack_row(const uint8_t *row, int8_t *t, long long K)
{
    long long bad = 0;
    for (long long k = 0; k < K; k++) {
        int code = (row[k / 4] >> (2 * (k % 4))) & 3;
        if (code == 3) {
            t[k] = ORACLE_INVALID_TRIT;
            bad++;
        } else {
            t[k] = (int8_t)(code - 1);
        }
    }
    return bad;
}

long long oracle_unpack_pq2(const uint8_t *packed, int8_t *trits, long long N, long long K)
{
    long long bad = 0;
    for (long long n = 0; n < N; n++) bad += pq2_unpack_row(packed + n * (K / 4), trits + n * K, K);
    return bad;
}

/* Validator: counts 2-bit slots holding the invalid code 3. */
long long oracle_check_pq2(const uint8_t *packed, long long N, long long K)
{
    long long bad = 0;
    for (long long i = 0; i < N * (K / 4); i++)
        for (int s = 0; s < 4; s++)
            if (((packed[i] >> (2 * s)) & 3) == 3) bad++;
    return bad;
}

/* ------------------------------------------------------------------ Q1_0 */

/* Weight k of a row is bit (k mod 8) of byte k/8 of the row: 1 for +1, 0 for -1.  One
 * bit has no invalid value, so a weight other than +1 or -1 is stored as -1 and counted
 * in the return value. */
long long oracle_pack_q1(const int8_t *trits, uint8_t *packed, long long N, long long K)
{
    long long bad = 0;
    for (long long n = 0; n < N; n++)
        for (long long byte = 0; byte < K / 8; byte++) {
            int v = 0;
            for (int i = 0; i < 8; i++) {
                int t = trits[n * K + 8 * byte + i];
                if (t == 1)
                    v |= 1 << i;
                else if (t != -1)
                    bad++;
            }
            packed[n * (K / 8) + byte] = (uint8_t)v;
        }
    return bad;
}

static long long q1_unpack_row(const uint8_t *row, int8_t *t, long long K)
{
    for (long long k = 0; k < K; k++) t[k] = ((row[k / 8] >> (k % 8)) & 1) ? 1 : -1;
    return 0;
}

long long oracle_unpack_q1(const uint8_t *packed, int8_t *trits, long long N, long long K)
{
    for (long long n = 0; n < N; n++) q1_unpack_row(packed + n * (K / 8), trits + n * K, K);
    return 0;
}

/* Validator: every bit pattern is a valid Q1_0 plane. */
long long oracle_check_q1(const uint8_t *packed, long long N, long long K)
{
    (void)packed;
    (void)N;
    (void)K;
    return 0;
}

long long oracle_unpack(int fmt, const uint8_t *packed, int8_t *trits, long long N, long long K)
{
    if (fmt == ORACLE_FMT_PTQ1_0) return oracle_unpack_ptq1(packed, trits, N, K);
    if (fmt == ORACLE_FMT_PQ2_0) return oracle_unpack_pq2(packed, trits, N, K);
    if (fmt == ORACLE_FMT_Q1_0) return oracle_unpack_q1(packed, trits, N, K);
    if (fmt == ORACLE_FMT_PQ2_0_G64) return oracle_unpack_pq2(packed, trits, N, K);
    return -1;
}

/* ------------------------------------------------------------------ Hadamard */

static int parity_of_and(int i, int j)
{
    int v = i & j, p = 0;
    while (v) {
        p ^= v & 1;
        v >>= 1;
    }
    return p;
}

/* Explicit normalised Sylvester matrix: Hn[i][j] = (-1)^popcount(i & j) / sqrt(128).
 * Symmetric and orthonormal, so it is its own inverse. */
void oracle_sylvester128(double *H)
{
    const double norm = 1.0 / sqrt((double)ORACLE_GROUP);
    for (int i = 0; i < ORACLE_GROUP; i++)
        for (int j = 0; j < ORACLE_GROUP; j++)
            H[i * ORACLE_GROUP + j] = (parity_of_and(i, j) ? -1.0 : 1.0) * norm;
}

/* x' = blockdiag(Hn) x for every row of the M x K matrix x: each run of 128
 * activations starting at a multiple of 128 is multiplied by the explicit Hn. */
void oracle_hadamard128(const double *x, double *xr, long long M, long long K)
{
    double *H = (double *)malloc(sizeof(double) * ORACLE_GROUP * ORACLE_GROUP);
    oracle_sylvester128(H);
    for (long long m = 0; m < M; m++)
        for (long long b = 0; b < K / ORACLE_GROUP; b++) {
            const double *in = x + m * K + b * ORACLE_GROUP;
            double *out = xr + m * K + b * ORACLE_GROUP;
            for (int i = 0; i < ORACLE_GROUP; i++) {
                double s = 0.0;
                for (int j = 0; j < ORACLE_GROUP; j++) s += H[i * ORACLE_GROUP + j] * in[j];
                out[i] = s;
            }
        }
    free(H);
}

/* Second, independent route to the same transform (used only to pin the first):
 * the unnormalised Sylvester recursion H_2n [u; w] = [H_n (u + w); H_n (u - w)],
 * applied in place to a vector of length n (a power of two). */
void oracle_fwht_recursive(double *v, long long n)
{
    if (n <= 1) return;
    long long h = n / 2;
    for (long long i = 0; i < h; i++) {
        double a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
    }
    oracle_fwht_recursive(v, h);
    oracle_fwht_recursive(v + h, h);
}

/* ------------------------------------------------------------------ linear */

/* y (M x N, float64) = x'(M x K) . Wdeq^T with Wdeq[n][k] = s[n][k/128] * t[n][k],
 * summed group by group exactly as the definition reads:
 *     y[m][n] = sum_g s[n][g] * ( sum_{j<128} t[n][128g+j] * x'[m][128g+j] ).
 * x and scales arrive as float64 copies of the FP16 inputs.  If apply_hadamard
 * is 0, x' = x (the transform is skipped: used only by the negative tests).
 * nthreads <= 0 means the OpenMP default.  Returns the count of invalid bytes
 * met while unpacking (their trits read as ORACLE_INVALID_TRIT), or -1 on a bad
 * argument. */
long long oracle_ternary_linear(const double *x, const uint8_t *packed, const double *scales,
                                double *y, long long M, long long N, long long K, int fmt,
                                int apply_hadamard, int nthreads)
{
    long long row_bytes = oracle_packed_bytes(fmt, 1, K);
    if (row_bytes < 0 || M < 0 || N < 0) return -1;
    const int gs = fmt == ORACLE_FMT_PQ2_0_G64 ? 64 : ORACLE_GROUP; /* weights per scale */
    long long G = K / gs;
    double *xr = (double *)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    if (apply_hadamard)
        oracle_hadamard128(x, xr, M, K);
    else
        memcpy(xr, x, sizeof(double) * (size_t)(M * K));

    long long bad = 0;
#ifdef _OPENMP
    int threads = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 16) num_threads(threads) reduction(+ : bad)
#endif
    for (long long n = 0; n < N; n++) {
        int8_t *t = (int8_t *)malloc((size_t)(K > 0 ? K : 1));
        if (fmt == ORACLE_FMT_PTQ1_0)
            bad += ptq1_unpack_row(packed + n * row_bytes, t, K);
        else if (fmt == ORACLE_FMT_PQ2_0 || fmt == ORACLE_FMT_PQ2_0_G64)
            bad += pq2_unpack_row(packed + n * row_bytes, t, K);
        else
            bad += q1_unpack_row(packed + n * row_bytes, t, K);
        for (long long m = 0; m < M; m++) {
            double acc = 0.0;
            for (long long g = 0; g < G; g++) {
                double dot = 0.0;
                for (int j = 0; j < gs; j++) dot += (double)t[g * gs + j] * xr[m * K + g * gs + j];
                acc += scales[n * G + g] * dot;
            }
            y[m * N + n] = acc;
        }
        free(t);
    }
    free(xr);
    return bad;
}

/* ------------------------------------------------------------------ SwiGLU */

/* The MLP step that follows the fused gate/up projection: with y the M x 2F output of
 * one linear layer whose rows 0 .. F-1 are the gate projection and F .. 2F-1 the up
 * projection, h[m][f] = silu(y[m][f]) * y[m][F + f], silu(z) = z / (1 + e^-z).  Written
 * out in float64.  Source of the fused gate/up projection (N = 2 x 17408): the 27B-class
 * shapes this layer is built for (d = 5120, ffn = 17408). */
void oracle_swiglu(const double *y, double *h, long long M, long long F)
{
    for (long long m = 0; m < M; m++)
        for (long long f = 0; f < F; f++) {
            double g = y[m * 2 * F + f], u = y[m * 2 * F + F + f];
            h[m * F + f] = g / (1.0 + exp(-g)) * u;
        }
}

/* Threads an OpenMP region would use by default (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
