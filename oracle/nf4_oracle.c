/*
 * CPU oracle for the frozen-NF4 QLoRA linear layer: quantisation half.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The CUDA library
 * shares no code, table or constant generator with it.
 *
 * Plain, slow, obviously correct: every step is written the way the pages
 * state it, in the pages' order, with no blocking or fusion. Sources are the
 * five pages on QLoRA:
 *   [p1] "QLoRA - 650億パラメータのモデルをGPU 1枚で微調整する" (ta-paperlens),
 *        sections "量子化を1段落で" (blockwise absmax, c = max|x_i|),
 *        "NF4" (quantile levels, exact zero, ends at +-1),
 *        "二重量子化" (8-bit constants in groups of 256, mean subtracted first).
 *   [p4] "QLoRA" glossary (ultralytics), the NF4 level snippet
 *        (normal quantiles from 0.9677083 to 0.5, 8 positive, 7 negative, zero,
 *        divided by the max) and the nearest-level argmin.
 * Readings where the pages are silent (nibble order, 8-bit float format,
 * rounding of midpoints, zero blocks, mean summation order) are stated at
 * each function.
 *
 * Build: gcc -std=c11 -O2 -fPIC -shared -fopenmp -ffp-contract=off
 * (no fast-math: every fp32 operation below is one IEEE round-to-nearest step).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BLOCK 64   /* [p1] 量子化を1段落で: QLoRA cuts W into blocks of 64 */
#define ORACLE_GROUP 256  /* [p1] 二重量子化: constants grouped 256 at a time     */

/* ------------------------------------------------------------------------- */
/* Standard normal distribution                                              */
/* ------------------------------------------------------------------------- */

/* Phi(x) = P(Z <= x) = erfc(-x / sqrt 2) / 2 (definition of the normal CDF). */
static double normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Inverse normal CDF by bisection on the monotone Phi: the plain definition
 * "the x with Phi(x) = p", solved to the last fp64 bit. */
double oracle_normal_icdf(double p)
{
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 4000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    /* lo and hi are adjacent doubles; return the one whose CDF is closer */
    return (fabs(normal_cdf(lo) - p) <= fabs(normal_cdf(hi) - p)) ? lo : hi;
}

/* ------------------------------------------------------------------------- */
/* NF4 levels and decision thresholds                                        */
/* ------------------------------------------------------------------------- */

static int cmp_double(const void* a, const void* b)
{
    double x = *(const double*)a, y = *(const double*)b;
    return (x > y) - (x < y);
}

/* [p4] NF4 snippet: positive levels are the normal quantiles at
 * linspace(0.9677083, 0.5, 9) without its last point (8 values), negative
 * levels are minus the quantiles at linspace(0.9677083, 0.5, 8) without its
 * last point (7 values), plus an exact zero; sort, divide by the max.
 * [p1] NF4: zero is exact and the ends are exactly -1 and +1.
 * Reading: all of it in fp64, each level rounded once to fp32 at the end.
 * out64 may be NULL. */
void oracle_nf4_levels(double* out64, float* out32)
{
    const double p0 = 0.9677083;
    double v[16];
    int n = 0;
    for (int k = 0; k < 8; ++k) v[n++] = oracle_normal_icdf(p0 - k * ((p0 - 0.5) / 8.0));
    for (int k = 0; k < 7; ++k) v[n++] = -oracle_normal_icdf(p0 - k * ((p0 - 0.5) / 7.0));
    v[n++] = 0.0;
    qsort(v, 16, sizeof(double), cmp_double);
    double vmax = v[15];
    for (int k = 0; k < 16; ++k) {
        double l = v[k] / vmax;
        if (out64) out64[k] = l;
        out32[k] = (float)l;
    }
}

/* Decision thresholds for nearest-level search over a sorted fp32 table L.
 * m_k = the exact midpoint (L[k] + L[k+1]) / 2 (exact in fp64), rounded
 * toward -infinity to fp32. For an fp32 value v, "v > m_k" is then exactly
 * "v is strictly closer to L[k+1] than to L[k]", and an exact tie goes to the
 * lower index, which is the first-index rule of argmin ([p4] snippet). */
void oracle_midpoints(const float* L, int nlev, float* mids)
{
    for (int k = 0; k + 1 < nlev; ++k) {
        double m = ((double)L[k] + (double)L[k + 1]) * 0.5;
        float f = (float)m;
        if ((double)f > m) f = nextafterf(f, -INFINITY);
        mids[k] = f;
    }
}

/* ------------------------------------------------------------------------- */
/* Blockwise absmax + nearest-level codes + nibble packing                   */
/* ------------------------------------------------------------------------- */

/* [p1] 量子化を1段落で: c = max_i |x_i| over one block, kept in full fp32. */
float oracle_block_absmax(const float* w, int64_t n)
{
    float c = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(w[i]);
        if (a > c) c = a;
    }
    return c;
}

/* Code of one value: the number of thresholds strictly below v/c, i.e. the
 * index of the nearest level of x/c ([p1] 量子化を1段落で; [p4] argmin).
 * v = w / c is one IEEE fp32 division. Reading: a zero block (c == 0) codes
 * every element as the exact-zero level ([p1] NF4: zero stays zero), which is
 * index `zero_code`. */
static uint8_t encode_one(float w, float c, const float* mids, int nmid, uint8_t zero_code)
{
    if (c == 0.0f) return zero_code;
    float v = w / c;
    uint8_t code = 0;
    for (int k = 0; k < nmid; ++k)
        if (v > mids[k]) ++code;
    return code;
}

/* Encode nblocks consecutive blocks of `block` values with the level table
 * L[nlev] (nlev <= 16): absmax[b] and codes[b*block + i] (one code per byte,
 * unpacked). zero_code is the index of the exact-zero level (7 for NF4). */
void oracle_encode_blocks(const float* w, int64_t nblocks, int block,
                          const float* L, int nlev, uint8_t zero_code,
                          float* absmax, uint8_t* codes)
{
    float mids[15];
    oracle_midpoints(L, nlev, mids);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        const float* wb = w + b * block;
        float c = oracle_block_absmax(wb, block);
        absmax[b] = c;
        for (int i = 0; i < block; ++i)
            codes[b * block + i] = encode_one(wb[i], c, mids, nlev - 1, zero_code);
    }
}

/* Reading (the pages give no order): element 2j goes to the high nibble of
 * byte j, element 2j+1 to the low nibble. */
void oracle_pack_nibbles(const uint8_t* codes, int64_t n, uint8_t* packed)
{
    for (int64_t j = 0; j < n / 2; ++j)
        packed[j] = (uint8_t)(((codes[2 * j] & 15u) << 4) | (codes[2 * j + 1] & 15u));
}

void oracle_unpack_nibbles(const uint8_t* packed, int64_t n, uint8_t* codes)
{
    for (int64_t j = 0; j < n / 2; ++j) {
        codes[2 * j] = (uint8_t)(packed[j] >> 4);
        codes[2 * j + 1] = (uint8_t)(packed[j] & 15u);
    }
}

/* ------------------------------------------------------------------------- */
/* OCP FP8 E4M3 (the "8-bit float" of the constants)                         */
/* ------------------------------------------------------------------------- */

/* Value of an E4M3 byte (OCP 8-bit floating point, E4M3: bias 7, no
 * infinities, S.1111.111 is NaN, largest finite 448). */
double oracle_e4m3_decode(uint8_t q)
{
    int s = q >> 7, e = (q >> 3) & 15, m = q & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);          /* subnormal: m/8 * 2^(1-7) */
    else        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round-to-nearest-even onto the finite E4M3 values, saturating to +-448:
 * the plain definition, by searching all 127 non-negative finite magnitudes
 * (their values in `vals`) for the nearest one; ties go to the even code. */
static uint8_t e4m3_nearest(float x, const double* vals)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a > 448.0) a = 448.0;  /* saturate to the largest finite magnitude */
    int best = 0;
    double bestd = INFINITY;
    for (int q = 0; q <= 0x7E; ++q) {
        double d = fabs(a - vals[q]);
        if (d < bestd || (d == bestd && (q & 1) == 0 && (best & 1) == 1)) {
            best = q;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

static void e4m3_values(double* vals)
{
    for (int q = 0; q <= 0x7E; ++q) vals[q] = oracle_e4m3_decode((uint8_t)q);
}

uint8_t oracle_e4m3_encode(float x)
{
    double vals[127];
    e4m3_values(vals);
    return e4m3_nearest(x, vals);
}

/* ------------------------------------------------------------------------- */
/* Double quantisation of the absmax constants                               */
/* ------------------------------------------------------------------------- */

/* Mean of the constants. Reading: one global mean per tensor ([p1] 二重量子化
 * subtracts "their mean"); the sum is fp64, accumulated by the stride-doubling
 * pairwise tree over the values zero-padded to a power of two (level s = 1,
 * 2, 4, ...: x[i] += x[i + s] for every i that is a multiple of 2s), then
 * divided by n in fp64 and rounded once to fp32. */
float oracle_dq_mean(const float* c, int64_t n, double* sum_out)
{
    int64_t size = 1;
    while (size < n) size <<= 1;
    double* x = (double*)calloc((size_t)size, sizeof(double));
    for (int64_t i = 0; i < n; ++i) x[i] = (double)c[i];
    for (int64_t s = 1; s < size; s <<= 1)
        for (int64_t i = 0; i + s < size; i += 2 * s)
            x[i] += x[i + s];
    double total = x[0];
    free(x);
    if (sum_out) *sum_out = total;
    return (float)(total / (double)n);
}

/* [p1] 二重量子化: the fp32 constants, centred by their mean, are stored as
 * 8-bit floats in groups of 256, with one fp32 second-level constant per group.
 * Per group g: d_b = c_b - mean (fp32), c2 = max |d_b| over the group's entries
 * (a short last group uses the entries it has), s2 = c2 / 448 (fp32), and the
 * code is E4M3(d_b / s2) (fp32 division, then round-to-nearest-even onto E4M3).
 * Reading: E4M3 is scaled so the group absmax maps to its largest finite 448;
 * a group with s2 == 0 stores code 0x00. */
void oracle_double_quant(const float* c, int64_t nb, uint8_t* qabsmax, float* s2, float* mean)
{
    float mu = oracle_dq_mean(c, nb, NULL);
    double vals[127];
    e4m3_values(vals);
    *mean = mu;
    int64_t ng = (nb + ORACLE_GROUP - 1) / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ng; ++g) {
        int64_t b0 = g * ORACLE_GROUP;
        int64_t b1 = b0 + ORACLE_GROUP < nb ? b0 + ORACLE_GROUP : nb;
        float c2 = 0.0f;
        for (int64_t b = b0; b < b1; ++b) {
            float d = c[b] - mu;
            if (fabsf(d) > c2) c2 = fabsf(d);
        }
        float sg = c2 / 448.0f;
        s2[g] = sg;
        for (int64_t b = b0; b < b1; ++b) {
            float d = c[b] - mu;
            qabsmax[b] = (sg == 0.0f) ? (uint8_t)0x00 : e4m3_nearest(d / sg, vals);
        }
    }
}

/* Constant actually used at dequantisation: c' = E4M3 value * s2 + mean,
 * one fused multiply-add with a single fp32 rounding (C99 fmaf). */
float oracle_dq_constant(uint8_t q, float s2, float mean)
{
    return fmaf((float)oracle_e4m3_decode(q), s2, mean);
}

/* ------------------------------------------------------------------------- */
/* Dequantisation to bf16                                                    */
/* ------------------------------------------------------------------------- */

/* fp32 -> bf16 bits, round to nearest even (the compute dtype of [p1]
 * 勾配は実際どこへ行くのか: stored NF4, computed in BF16). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;  /* NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* [p1] 量子化を1段落で: restore x_hat = c * level[code]; with double
 * quantisation c is the decoded constant c'. The product is one fp32 rounding,
 * then one bf16 rounding. W is [N, K] row-major, K a multiple of 64, so block b
 * covers flat elements 64b .. 64b+63. */
void oracle_dequant_bf16(const uint8_t* packed, const uint8_t* qabsmax, const float* s2,
                         float mean, int64_t N, int64_t K, uint16_t* out)
{
    float L[16];
    oracle_nf4_levels(NULL, L);
    int64_t nb = N * K / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        float cp = oracle_dq_constant(qabsmax[b], s2[b / ORACLE_GROUP], mean);
        for (int i = 0; i < ORACLE_BLOCK; ++i) {
            int64_t e = b * ORACLE_BLOCK + i;
            uint8_t byte = packed[e / 2];
            uint8_t code = (e % 2 == 0) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
            float v = L[code] * cp;
            out[e] = oracle_f32_to_bf16(v);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Whole quantiser: W fp32 -> (packed codes, qabsmax, s2, mean)              */
/* ------------------------------------------------------------------------- */

/* absmax_out (nb floats) may be NULL; it returns the first-level constants. */
int oracle_quantize_nf4(const float* W, int64_t N, int64_t K, uint8_t* packed,
                        uint8_t* qabsmax, float* s2, float* mean, float* absmax_out)
{
    if (N <= 0 || K <= 0 || K % ORACLE_BLOCK != 0) return -1;
    int64_t n = N * K, nb = n / ORACLE_BLOCK;
    float L[16];
    oracle_nf4_levels(NULL, L);
    float* c = (float*)malloc((size_t)nb * sizeof(float));
    uint8_t* codes = (uint8_t*)malloc((size_t)n);
    oracle_encode_blocks(W, nb, ORACLE_BLOCK, L, 16, 7, c, codes);
    oracle_pack_nibbles(codes, n, packed);
    oracle_double_quant(c, nb, qabsmax, s2, mean);
    if (absmax_out) memcpy(absmax_out, c, (size_t)nb * sizeof(float));
    free(codes);
    free(c);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Storage without double quantisation                                       */
/* ------------------------------------------------------------------------- */

/* [p1] 二重量子化, first paragraph: before the constants are themselves
 * quantised, each block of 64 keeps its absmax c as one fp32 (4 + 32/64 = 4.5
 * bits per weight). The codes are those of the whole quantiser above; the
 * constants are the block absmax values, unchanged. */
int oracle_quantize_nf4_nodq(const float* W, int64_t N, int64_t K, uint8_t* packed, float* absmax)
{
    if (N <= 0 || K <= 0 || K % ORACLE_BLOCK != 0) return -1;
    int64_t n = N * K, nb = n / ORACLE_BLOCK;
    float L[16];
    oracle_nf4_levels(NULL, L);
    uint8_t* codes = (uint8_t*)malloc((size_t)n);
    oracle_encode_blocks(W, nb, ORACLE_BLOCK, L, 16, 7, absmax, codes);
    oracle_pack_nibbles(codes, n, packed);
    free(codes);
    return 0;
}

/* [p1] 量子化を1段落で: x_hat = c * level[code] with c the block's own fp32
 * absmax, one fp32 rounding (the restore of the glossary's snippet). */
void oracle_dequant_f32_nodq(const uint8_t* packed, const float* absmax, int64_t N, int64_t K, float* out)
{
    float L[16];
    oracle_nf4_levels(NULL, L);
    int64_t nb = N * K / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        for (int i = 0; i < ORACLE_BLOCK; ++i) {
            int64_t e = b * ORACLE_BLOCK + i;
            uint8_t byte = packed[e / 2];
            uint8_t code = (e % 2 == 0) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
            out[e] = L[code] * absmax[b];
        }
    }
}

/* The same restore, then one bf16 rounding (computed in BF16, [p1]
 * 勾配は実際どこへ行くのか). */
void oracle_dequant_bf16_nodq(const uint8_t* packed, const float* absmax, int64_t N, int64_t K, uint16_t* out)
{
    int64_t n = N * K;
    float* f = (float*)malloc((size_t)n * sizeof(float));
    oracle_dequant_f32_nodq(packed, absmax, N, K, f);
    for (int64_t e = 0; e < n; ++e) out[e] = oracle_f32_to_bf16(f[e]);
    free(f);
}

/* ------------------------------------------------------------------------- */
/* fp64 -> bf16, one rounding (for the adapter merge)                        */
/* ------------------------------------------------------------------------- */

/* Round x to the nearest bf16 value, ties to the even significand, in one
 * step from the fp64 value. bf16 keeps 8 significant bits; for |x| in
 * [2^(e-1), 2^e) neighbouring values are 2^(e-8) apart, and below the
 * smallest normal 2^-126 they are 2^-133 apart (subnormals). A result of
 * 2^128 or more overflows to infinity. nearbyint rounds to nearest even in the
 * default rounding mode; dividing by a power of two is exact. */
uint16_t oracle_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e);
    int qe = e - 8 < -133 ? -133 : e - 8;
    double r = ldexp(nearbyint(ldexp(a, -qe)), qe);
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    float f = (float)r;  /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (u >> 16));
}

void oracle_f64_to_bf16_array(const double* x, int64_t n, uint16_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16(x[i]);
}

/* Storage of one quantised N x K weight, in bytes: packed codes (4 bits per
 * weight), one 8-bit constant per block of 64, one fp32 per group of 256
 * blocks, one fp32 mean ([p1] 二重量子化). Without double quantisation the
 * constants are fp32 per block of 64 ([p1] 4 + 32/64 = 4.5 bits). */
int64_t oracle_storage_bytes(int64_t N, int64_t K, int double_quant)
{
    int64_t n = N * K, nb = n / ORACLE_BLOCK, ng = (nb + ORACLE_GROUP - 1) / ORACLE_GROUP;
    if (!double_quant) return n / 2 + 4 * nb;
    return n / 2 + nb + 4 * ng + 4;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* The E4M3 encoder above, applied to an array (for wide sweeps in tests). */
void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* q)
{
    double vals[127];
    e4m3_values(vals);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) q[i] = e4m3_nearest(x[i], vals);
}
