/*
 * Oracle for group-wise affine weight-only quantization and the quantized
 * matmul that consumes it.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * CPU statement of what the CUDA library computes.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark may load it.  It shares
 * no code, header, table or helper with the CUDA path, and it never calls it.
 *
 * What it follows (page titles and sections of the source pages):
 *  - "Quantizing a Model for MLX", section "What MLX quantization stores":
 *    weights are cut into contiguous groups; each group has its own scale and
 *    offset, stored in fp16 beside the integer codes, which are packed several
 *    to a machine word.
 *  - "metalworking — MLX Quantization", section "Mechanics": each group of
 *    32/64/128 values along a row stores one scale, one bias and 2..8-bit
 *    codes, with w ~= code * scale + bias.
 *  - "anllm Tutorial 10: Quantization", section 3 "Packing Multiple Weights into
 *    One Word": code j of a word sits at bit shift bits*j (shift, then mask);
 *    dequantization is values * scales + biases with the group's scale and
 *    bias repeated over its group_size values (section 2 "Group Quantization":
 *    groups run along in_features, i.e. along K within one output row).
 *  - Same tutorial, section 5 "Quantized Matrix Multiply": y = x @ W^T, and the
 *    fused product equals dequantize-then-multiply.
 *  - "metalworking — MLX Quantization" (newer modes) and "Quantizing a Model
 *    for MLX", section "Modes, bits and mixed recipes": the mxfp4 block-scaled
 *    mode (oracle_mxfp4_*; encodings and readings beside them).
 *  - the same two pages on mxfp8 (oracle_mxfp8_*; encodings beside them).
 *  - "ExecuTorch MLX backend — Quantization" (NVFP4 config) and "Quantizing a
 *    Model for MLX", section "Modes, bits and mixed recipes": the nvfp4 mode
 *    (oracle_nvfp4_*; encodings and readings beside them).
 *  - "mlx-gptq" page, section "How it works": the range search (--mse) that
 *    shrinks a group's min-max range when clipping its extremes costs less
 *    error than the coarser step (oracle_quantize_mse; readings beside it).
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *  - scale = (max - min) / (2^bits - 1) and bias = min, both computed in fp32
 *    and rounded to fp16 (round to nearest, ties to even, subnormals kept).
 *    A group extreme equal to zero is taken as +0.0 (the sign of a zero min or
 *    max is not a property of the set of values).
 *  - codes are computed from the STORED (fp16) scale and bias:
 *        q = clamp(rint_even(fp32(fp32(w - bias16) / scale16)), 0, 2^bits - 1)
 *    with IEEE correctly rounded fp32 subtraction and division.
 *    A group whose fp16 scale is zero gets all codes 0.
 *  - 3-bit codes form one contiguous LSB-first bitstream per row (32 codes in
 *    3 words); every row starts on a word boundary.
 *  - dequantized value: fp32(q * scale16 + bias16) with a single rounding (the
 *    exact product-sum fits in fp64, so it is formed there and rounded once),
 *    then rounded to bf16 for the bf16 output.
 *  - matmul reference: y[m][n] = sum_k x[m][k] * (q*scale16 + bias16), exact
 *    terms summed in fp64.
 *
 * Parity status: every function here is pinned by the not-gpu tests (closed
 * forms from the pages, hand-derived fixtures, brute force, an independent
 * NumPy implementation); none is "parity unpinned".
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* ------------------------------------------------------------------------ */
/* IEEE binary16 / bfloat16 rounding written out from the format definitions */
/* ------------------------------------------------------------------------ */

/* Round a finite double to the nearest value with `mant_bits` fraction bits
 * and minimum normal exponent `emin` (ties to even), returning the rounded
 * value as a double.  Values below 2^emin are rounded on the subnormal grid
 * 2^(emin - mant_bits).  rint() runs in the default round-to-nearest-even mode. */
static double round_to_format(double v, int mant_bits, int emin)
{
    if (v == 0.0 || !isfinite(v)) return v;
    double a = fabs(v);
    int ex;
    frexp(a, &ex);          /* a = f * 2^ex with f in [0.5, 1) */
    int e = ex - 1;         /* a in [2^e, 2^(e+1)) */
    if (e < emin) e = emin; /* subnormal range shares the quantum of 2^emin */
    double quantum = ldexp(1.0, e - mant_bits);
    double r = rint(a / quantum) * quantum; /* a/quantum is exact (power of 2) */
    return copysign(r, v);
}

/* fp16 bit pattern of the nearest binary16 value to v (v exactly a float). */
static uint16_t f16_bits_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return 0x7e00u;
    double r = fabs(round_to_format(v, 10, -14));
    if (isinf(v) || r >= 65536.0) return sign | 0x7c00u; /* overflow -> inf */
    if (r == 0.0) return sign;
    int ex;
    frexp(r, &ex);
    int e = ex - 1;
    if (e < -14) { /* subnormal: value = m * 2^-24 */
        uint16_t m = (uint16_t)ldexp(r, 24);
        return sign | m;
    }
    uint16_t mant = (uint16_t)(ldexp(r, 10 - e) - 1024.0);
    return sign | (uint16_t)((e + 15) << 10) | mant;
}

static double f16_value(uint16_t h)
{
    int sign = (h >> 15) & 1, exp = (h >> 10) & 0x1f, mant = h & 0x3ff;
    double v;
    if (exp == 0)
        v = ldexp((double)mant, -24);
    else if (exp == 31)
        v = mant ? NAN : INFINITY;
    else
        v = ldexp(1024.0 + mant, exp - 25);
    return sign ? -v : v;
}

/* bf16 bit pattern of the nearest bfloat16 value to v. */
static uint16_t bf16_bits_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return 0x7fc0u;
    double r = fabs(round_to_format(v, 7, -126));
    if (isinf(v) || r >= ldexp(1.0, 128)) return sign | 0x7f80u;
    if (r == 0.0) return sign;
    int ex;
    frexp(r, &ex);
    int e = ex - 1;
    if (e < -126) {
        uint16_t m = (uint16_t)ldexp(r, 133);
        return sign | m;
    }
    uint16_t mant = (uint16_t)(ldexp(r, 7 - e) - 128.0);
    return sign | (uint16_t)((e + 127) << 7) | mant;
}

static double bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Exposed for the pins: element-wise conversions. */
void oracle_f16_round(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = f16_bits_from_double((double)in[i]);
}

void oracle_bf16_round(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = bf16_bits_from_double((double)in[i]);
}

void oracle_f16_to_double(const uint16_t *in, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = f16_value(in[i]);
}

/* ------------------------------------------------------------------------ */
/* Argument checks shared by the entry points of this file                  */
/* ------------------------------------------------------------------------ */

static int bad_shape(int64_t N, int64_t K, int G, int bits)
{
    if (N <= 0 || K <= 0) return 1;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return 1;
    if (!(G == 32 || G == 64 || G == 128)) return 1;
    if (K % G != 0) return 1;
    return 0;
}

/* Words per packed row: K codes of `bits` bits, LSB-first bitstream. */
static int64_t row_words(int64_t K, int bits) { return K * bits / 32; }

/* ------------------------------------------------------------------------ */
/* Quantize: per group min/max, fp16 scale and bias, codes, packing          */
/* ------------------------------------------------------------------------ */

/* Put code q of element k into row n's bitstream: bits [k*bits, k*bits+bits). */
static void put_code(uint32_t *row, int64_t k, int bits, uint32_t q)
{
    for (int t = 0; t < bits; t++) {
        int64_t bit = k * bits + t;
        if ((q >> t) & 1u) row[bit / 32] |= (1u << (bit % 32));
    }
}

static uint32_t get_code(const uint32_t *row, int64_t k, int bits)
{
    uint32_t q = 0;
    for (int t = 0; t < bits; t++) {
        int64_t bit = k * bits + t;
        q |= ((row[bit / 32] >> (bit % 32)) & 1u) << t;
    }
    return q;
}

/* Group extremes, with a zero extreme taken as +0.0 (-0.0 and +0.0 are the
 * same number, and the sign of a zero min or max is not a property of the set
 * of values). */
static void group_min_max(const float *v, int G, float *mn_out, float *mx_out)
{
    float mn = v[0], mx = v[0];
    for (int i = 1; i < G; i++) {
        if (v[i] < mn) mn = v[i];
        if (v[i] > mx) mx = v[i];
    }
    if (mn == 0.0f) mn = 0.0f;
    if (mx == 0.0f) mx = 0.0f;
    *mn_out = mn;
    *mx_out = mx;
}

/* Stored fp16 scale and bias of the affine grid spanning [lo, hi]:
 * scale = fp32(fp32(hi - lo) / qmax), bias = lo, each rounded to fp16. */
static void grid_params(float lo, float hi, uint32_t qmax, uint16_t *s16, uint16_t *b16)
{
    float d = hi - lo;                 /* fp32 subtraction */
    float s32 = d / (float)qmax;       /* fp32 IEEE division */
    *s16 = f16_bits_from_double((double)s32);
    *b16 = f16_bits_from_double((double)lo);
}

/* Code of one value against the stored grid (sf, bf): the nearest grid point,
 * ties to even, clamped to [0, qmax]; a zero scale gives code 0. */
static uint32_t grid_code(float w, float sf, float bf, uint32_t qmax)
{
    if (sf == 0.0f) return 0u;
    float t = (w - bf) / sf;   /* fp32 sub, fp32 div */
    float r = rintf(t);        /* ties to even */
    if (r < 0.0f) r = 0.0f;
    if (r > (float)qmax) r = (float)qmax;
    return (uint32_t)r;
}

int oracle_quantize(const float *w, int64_t N, int64_t K, int G, int bits,
                    uint32_t *packed, uint16_t *scales, uint16_t *biases)
{
    if (!w || !packed || !scales || !biases || bad_shape(N, K, G, bits)) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits), Gn = K / G;
    const uint32_t qmax = (1u << bits) - 1u;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        const float *wr = w + n * K;
        uint32_t *pr = packed + n * P;
        for (int64_t j = 0; j < P; j++) pr[j] = 0u;
        for (int64_t g = 0; g < Gn; g++) {
            /* group = G contiguous elements of row n along K */
            float mn, mx;
            group_min_max(wr + g * G, G, &mn, &mx);
            uint16_t s16, b16;
            grid_params(mn, mx, qmax, &s16, &b16);
            scales[n * Gn + g] = s16;
            biases[n * Gn + g] = b16;
            float sf = (float)f16_value(s16), bf = (float)f16_value(b16);
            for (int64_t i = 0; i < G; i++)
                put_code(pr, g * G + i, bits, grid_code(wr[g * G + i], sf, bf, qmax));
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Range-search quantize: per group, the shrunk [min, max] of least error     */
/* ------------------------------------------------------------------------ */

/* "mlx-gptq" page, "How it works": the range search shrinks a group's min-max
 * range whenever clipping its extremes costs less error than the coarser step
 * of the full range costs the rest of the group.  The page gives neither the
 * grid of candidate ranges nor the error's arithmetic; the readings taken:
 *  - candidates i = 0 .. 31 with shrink factor p_i = 1 - i/32 (exact in fp32),
 *    i.e. every factor k/32 from 32/32 down to 1/32;
 *    candidate i spans [lo, hi] = [fp32(p_i * min), fp32(p_i * max)] (both
 *    bounds move toward zero; a zero bound is +0.0).  Candidate 0 is the plain
 *    min-max grid, so the search never does worse than round-to-nearest;
 *  - each candidate's fp16 scale/bias and codes are those of the plain
 *    quantizer for [lo, hi]; values outside the range clamp to code 0 or qmax
 *    (the clipping);
 *  - its error is the sum of squared errors e = fp32(w - fp32(q*scale16 + bias16))
 *    over the group, in fp32: e*e rounded, summed from zero in element order
 *    within each run of 32 elements, and the runs' sums added pairwise ((r0 + r1) + (r2 + r3) for 128);
 *  - the candidate of least error wins; equal errors keep the smaller i (the
 *    wider range). */
#define MSE_CANDIDATES 32
#define MSE_STEP_DENOM 32

static float run_error(const float *v, float sf, float bf, uint32_t qmax)
{
    float acc = 0.0f;
    for (int j = 0; j < 32; j++) {
        uint32_t q = grid_code(v[j], sf, bf, qmax);
        float deq = (float)((double)q * (double)sf + (double)bf); /* exact, rounded once */
        float e = v[j] - deq;
        float e2 = e * e;
        acc = acc + e2;
    }
    return acc;
}

static float group_error(const float *v, int G, float sf, float bf, uint32_t qmax)
{
    if (G == 32) return run_error(v, sf, bf, qmax);
    if (G == 64) return run_error(v, sf, bf, qmax) + run_error(v + 32, sf, bf, qmax);
    float a = run_error(v, sf, bf, qmax) + run_error(v + 32, sf, bf, qmax);
    float b = run_error(v + 64, sf, bf, qmax) + run_error(v + 96, sf, bf, qmax);
    return a + b;
}

int oracle_quantize_mse(const float *w, int64_t N, int64_t K, int G, int bits,
                        uint32_t *packed, uint16_t *scales, uint16_t *biases)
{
    if (!w || !packed || !scales || !biases || bad_shape(N, K, G, bits)) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits), Gn = K / G;
    const uint32_t qmax = (1u << bits) - 1u;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        const float *wr = w + n * K;
        uint32_t *pr = packed + n * P;
        for (int64_t j = 0; j < P; j++) pr[j] = 0u;
        for (int64_t g = 0; g < Gn; g++) {
            const float *v = wr + g * G;
            float mn, mx;
            group_min_max(v, G, &mn, &mx);
            uint16_t best_s = 0, best_b = 0;
            float best_err = 0.0f;
            for (int i = 0; i < MSE_CANDIDATES; i++) {
                float p = 1.0f - (float)i / (float)MSE_STEP_DENOM;   /* exact */
                float lo = p * mn, hi = p * mx;                        /* fp32 products */
                if (lo == 0.0f) lo = 0.0f;
                if (hi == 0.0f) hi = 0.0f;
                uint16_t s16, b16;
                grid_params(lo, hi, qmax, &s16, &b16);
                float err = group_error(v, G, (float)f16_value(s16), (float)f16_value(b16), qmax);
                if (i == 0 || err < best_err) {
                    best_err = err;
                    best_s = s16;
                    best_b = b16;
                }
            }
            scales[n * Gn + g] = best_s;
            biases[n * Gn + g] = best_b;
            float sf = (float)f16_value(best_s), bf = (float)f16_value(best_b);
            for (int64_t i = 0; i < G; i++)
                put_code(pr, g * G + i, bits, grid_code(v[i], sf, bf, qmax));
        }
    }
    return ORACLE_OK;
}

/* Codes as bytes [N, K], read back bit by bit from the packed bitstream. */
int oracle_unpack_codes(const uint32_t *packed, int64_t N, int64_t K, int bits, uint8_t *codes)
{
    if (!packed || !codes || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8) || (K * bits) % 32 != 0) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits);
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) codes[n * K + k] = (uint8_t)get_code(packed + n * P, k, bits);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Dequantize                                                               */
/* ------------------------------------------------------------------------ */

/* Exact q*scale + bias (fits in fp64: q has <= 8 bits, scale and bias are fp16). */
static double exact_value(const uint32_t *prow, const uint16_t *srow, const uint16_t *brow,
                          int64_t k, int G, int bits)
{
    uint32_t q = get_code(prow, k, bits);
    return (double)q * f16_value(srow[k / G]) + f16_value(brow[k / G]);
}

int oracle_dequantize_f32(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                          int64_t N, int64_t K, int G, int bits, float *out)
{
    if (!packed || !scales || !biases || !out || bad_shape(N, K, G, bits)) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits), Gn = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            out[n * K + k] = (float)exact_value(packed + n * P, scales + n * Gn, biases + n * Gn, k, G, bits);
    return ORACLE_OK;
}

int oracle_dequantize_bf16(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                           int64_t N, int64_t K, int G, int bits, uint16_t *out)
{
    if (!packed || !scales || !biases || !out || bad_shape(N, K, G, bits)) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits), Gn = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            float v = (float)exact_value(packed + n * P, scales + n * Gn, biases + n * Gn, k, G, bits);
            out[n * K + k] = bf16_bits_from_double((double)v);
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Quantized matmul reference: y = x @ dequant(W)^T in fp64                  */
/* ------------------------------------------------------------------------ */

/* y[i][j] for the requested rows m_idx[i] of x and rows n_idx[j] of W
 * (output columns); the full product is m_idx = 0..M-1, n_idx = 0..N-1. */
int oracle_matmul_sampled(const uint16_t *x_bf16, int64_t M, int64_t K,
                          const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                          int64_t N, int G, int bits,
                          const int64_t *m_idx, int64_t nm, const int64_t *n_idx, int64_t nn,
                          double *y)
{
    if (!x_bf16 || !packed || !scales || !biases || !m_idx || !n_idx || !y) return ORACLE_BAD_ARG;
    if (M <= 0 || bad_shape(N, K, G, bits) || nm < 0 || nn < 0) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < nm; i++) if (m_idx[i] < 0 || m_idx[i] >= M) return ORACLE_BAD_ARG;
    for (int64_t j = 0; j < nn; j++) if (n_idx[j] < 0 || n_idx[j] >= N) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits), Gn = K / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t j = 0; j < nn; j++) {
        const int64_t n = n_idx[j];
        const uint32_t *prow = packed + n * P;
        const uint16_t *srow = scales + n * Gn, *brow = biases + n * Gn;
        for (int64_t i = 0; i < nm; i++) {
            const uint16_t *xr = x_bf16 + m_idx[i] * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_value(xr[k]) * exact_value(prow, srow, brow, k, G, bits);
            y[i * nn + j] = acc;
        }
    }
    return ORACLE_OK;
}

/* Full product y[M][N]. */
int oracle_matmul(const uint16_t *x_bf16, int64_t M, int64_t K,
                  const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                  int64_t N, int G, int bits, double *y)
{
    if (!x_bf16 || !packed || !scales || !biases || !y) return ORACLE_BAD_ARG;
    if (M <= 0 || bad_shape(N, K, G, bits)) return ORACLE_BAD_ARG;
    const int64_t P = row_words(K, bits), Gn = K / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; n++) {
        const uint32_t *prow = packed + n * P;
        const uint16_t *srow = scales + n * Gn, *brow = biases + n * Gn;
        for (int64_t m = 0; m < M; m++) {
            const uint16_t *xr = x_bf16 + m * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_value(xr[k]) * exact_value(prow, srow, brow, k, G, bits);
            y[m * N + n] = acc;
        }
    }
    return ORACLE_OK;
}

/* Number of threads the parallel loops above use. */
/* ------------------------------------------------------------------------ */
/* mxfp4: block-scaled fp4 (E2M1 elements, one E8M0 exponent per 32)         */
/* ------------------------------------------------------------------------ */

/* "metalworking — MLX Quantization" (the paragraph on the newer modes) and
 * "Quantizing a Model for MLX", section "Modes, bits and mixed recipes": mxfp4
 * is a block-scaled float mode with groups of 32 and 4-bit elements, storing an
 * exponent per group instead of a scale and a bias.  The pages do not spell out
 * the encodings; the readings follow the OCP Microscaling (MX) v1.0 formats that
 * the name refers to, restated here:
 *  - element code c (4 bits): sign = bit 3, exponent e = bits 2..1, mantissa
 *    m = bit 0; magnitude m/2 for e = 0, else 2^(e-1) * (1 + m/2), i.e. the
 *    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7;
 *  - scale byte s: X = 2^(s - 127) (s = 255 is NaN and never produced);
 *  - quantize a group of 32 along K: amax = max |w|; shared exponent
 *    floor(log2 amax) - 2 (2 = the largest E2M1 exponent), clamped to
 *    [-127, 127]; s = shared + 127; an all-zero group gets s = 0;
 *  - each element: the E2M1 magnitude nearest to |w| / X, ties to the even code
 *    (mantissa bit 0), values above 6 saturating to 6; the sign bit is set only
 *    for negative values whose magnitude code is not 0 (zero is +0);
 *  - codes pack 8 to a uint32, LSB first (code k at bits 4k..4k+3 of the row);
 *  - dequantized value X * e2m1(c), exact in fp32 and bf16. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static double e2m1_value(uint32_t c)
{
    double v = E2M1_MAG[c & 7u];
    return (c & 8u) ? -v : v;
}

static double e8m0_value(uint8_t s) { return ldexp(1.0, (int)s - 127); }

/* Nearest E2M1 magnitude code to t >= 0 (nearer wins; on a tie the even code,
 * mantissa bit 0, wins). */
static uint32_t e2m1_nearest(double t)
{
    uint32_t best = 0;
    double best_d = fabs(t - E2M1_MAG[0]);
    for (uint32_t c = 1; c < 8; c++) {
        const double d = fabs(t - E2M1_MAG[c]);
        if (d < best_d || (d == best_d && (c & 1u) == 0u && (best & 1u) == 1u)) {
            best = c;
            best_d = d;
        }
    }
    return best;
}

static int bad_mx_shape(int64_t N, int64_t K) { return N <= 0 || K <= 0 || K % 32 != 0; }

int oracle_mxfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales)
{
    if (!w || !packed || !scales || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        const float *wr = w + n * K;
        uint32_t *pr = packed + n * P;
        for (int64_t j = 0; j < P; j++) pr[j] = 0u;
        for (int64_t g = 0; g < Gn; g++) {
            double amax = 0.0;
            for (int i = 0; i < 32; i++) {
                double a = fabs((double)wr[g * 32 + i]);
                if (a > amax) amax = a;
            }
            int shared = -127;
            if (amax > 0.0) {
                int ex;
                frexp(amax, &ex);           /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
                shared = (ex - 1) - 2;
                if (shared < -127) shared = -127;
                if (shared > 127) shared = 127;
            }
            scales[n * Gn + g] = (uint8_t)(shared + 127);
            for (int i = 0; i < 32; i++) {
                const double v = (double)wr[g * 32 + i];
                const double t = fabs(v) * ldexp(1.0, -shared);   /* exact */
                uint32_t best = e2m1_nearest(t);
                if (v < 0.0 && best != 0u) best |= 8u;
                put_code(pr, g * 32 + i, 4, best);
            }
        }
    }
    return ORACLE_OK;
}

static double mx_value(const uint32_t *prow, const uint8_t *srow, int64_t k)
{
    return e8m0_value(srow[k / 32]) * e2m1_value(get_code(prow, k, 4));
}

int oracle_mxfp4_dequantize_f32(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, float *out)
{
    if (!packed || !scales || !out || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            out[n * K + k] = (float)mx_value(packed + n * P, scales + n * Gn, k);
    return ORACLE_OK;
}

int oracle_mxfp4_matmul(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                        const uint8_t *scales, int64_t N, double *y)
{
    if (!x_bf16 || !packed || !scales || !y || M <= 0 || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; n++)
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_value(x_bf16[m * K + k]) * mx_value(packed + n * P, scales + n * Gn, k);
            y[m * N + n] = acc;
        }
    return ORACLE_OK;
}

int oracle_mxfp4_matmul_sampled(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                                const uint8_t *scales, int64_t N, const int64_t *m_idx, int64_t nm,
                                const int64_t *n_idx, int64_t nn, double *y)
{
    if (!x_bf16 || !packed || !scales || !m_idx || !n_idx || !y || M <= 0 || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < nm; i++) if (m_idx[i] < 0 || m_idx[i] >= M) return ORACLE_BAD_ARG;
    for (int64_t j = 0; j < nn; j++) if (n_idx[j] < 0 || n_idx[j] >= N) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t j = 0; j < nn; j++)
        for (int64_t i = 0; i < nm; i++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_value(x_bf16[m_idx[i] * K + k]) * mx_value(packed + n_idx[j] * P, scales + n_idx[j] * Gn, k);
            y[i * nn + j] = acc;
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* nvfp4: E2M1 elements, one E4M3 scale per 16, one fp32 scale per tensor     */
/* ------------------------------------------------------------------------ */

/* "ExecuTorch MLX backend — Quantization" (NVFP4 weight-only config, group
 * size 16) and "Quantizing a Model for MLX", section "Modes, bits and mixed
 * recipes" (nvfp4: groups of 16, 4 bits).  The pages give no encodings; the
 * readings follow NVIDIA's NVFP4 format, restated here:
 *  - elements: E2M1 codes as in mxfp4 (packed 8 per uint32, LSB first);
 *  - block scale: one E4M3 byte per 16 weights along K (sign 0, exponent bits
 *    6..3 with bias 7, mantissa bits 2..0; subnormals m * 2^-9; largest 448);
 *  - tensor scale: one fp32 value g = fp32(amax / 2688) (2688 = 6 * 448, the
 *    largest E2M1 value times the largest E4M3 value); g = 1 for an all-zero
 *    tensor;
 *  - block scale byte: E4M3 nearest to fp32(amax_block / fp32(6 * g)), ties to
 *    even, saturating at 448 (with this g no block goes past 448 beyond
 *    rounding: the clamp is defensive);
 *  - element: E2M1 nearest to fp32(|w| / fp32(scale * g)), ties to the even
 *    code, saturating at 6, sign only on a non-zero magnitude; a zero block
 *    scale gives code 0;
 *  - value: fp32(fp32(e2m1 * scale) * g) (the first product is exact). */

static uint8_t e4m3_bits_from_double(double v)   /* v >= 0, finite */
{
    double r = round_to_format(v, 3, -6);
    if (r > 448.0) r = 448.0;                     /* saturate */
    if (r == 0.0) return 0;
    int ex;
    frexp(r, &ex);
    int e = ex - 1;
    if (e < -6) return (uint8_t)ldexp(r, 9);      /* subnormal: m * 2^-9 */
    uint8_t mant = (uint8_t)(ldexp(r, 3 - e) - 8.0);
    return (uint8_t)(((e + 7) << 3) | mant);
}

static double e4m3_value(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp(8.0 + m, e - 10);
}

float oracle_nvfp4_tensor_scale(const float *w, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
    }
    if (!(amax > 0.0f)) return 1.0f;
    /* fp32 division; a tensor so small that amax / 2688 falls below the smallest
     * normal fp32 (2^-126) takes g = 2^-126, so g is never zero or subnormal and
     * every finite input quantizes (the pages are silent here: reading) */
    const float g = amax / 2688.0f;
    return g < 0x1p-126f ? 0x1p-126f : g;
}

int oracle_nvfp4_quantize(const float *w, int64_t N, int64_t K, float g, uint32_t *packed, uint8_t *scales)
{
    if (!w || !packed || !scales || N <= 0 || K <= 0 || K % 16 != 0 || !(g > 0.0f)) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 16;
    const float six_g = 6.0f * g;                 /* fp32 product */
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        const float *wr = w + n * K;
        uint32_t *pr = packed + n * P;
        for (int64_t j = 0; j < P; j++) pr[j] = 0u;
        for (int64_t b = 0; b < Gn; b++) {
            float amax = 0.0f;
            for (int i = 0; i < 16; i++) {
                float a = fabsf(wr[b * 16 + i]);
                if (a > amax) amax = a;
            }
            const float s32 = amax / six_g;       /* fp32 division */
            const uint8_t sb = e4m3_bits_from_double((double)s32);
            scales[n * Gn + b] = sb;
            const float denom = (float)e4m3_value(sb) * g;   /* fp32 product */
            for (int i = 0; i < 16; i++) {
                const float v = wr[b * 16 + i];
                uint32_t c = 0;
                if (sb != 0) {
                    const float t = fabsf(v) / denom;        /* fp32 division */
                    c = e2m1_nearest((double)t);
                    if (v < 0.0f && c != 0u) c |= 8u;
                }
                put_code(pr, b * 16 + i, 4, c);
            }
        }
    }
    return ORACLE_OK;
}

static double nv_value(const uint32_t *prow, const uint8_t *srow, float g, int64_t k)
{
    const float vs = (float)(e2m1_value(get_code(prow, k, 4)) * e4m3_value(srow[k / 16]));   /* exact */
    return (double)(vs * g);                                                                /* fp32 product */
}

int oracle_nvfp4_dequantize_f32(const uint32_t *packed, const uint8_t *scales, float g, int64_t N, int64_t K, float *out)
{
    if (!packed || !scales || !out || N <= 0 || K <= 0 || K % 16 != 0) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) out[n * K + k] = (float)nv_value(packed + n * P, scales + n * Gn, g, k);
    return ORACLE_OK;
}

/* y = x @ W^T with W's values e2m1 * scale * g taken exactly (fp64), summed in fp64. */
int oracle_nvfp4_matmul(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                        float g, int64_t N, double *y)
{
    if (!x_bf16 || !packed || !scales || !y || M <= 0 || N <= 0 || K <= 0 || K % 16 != 0) return ORACLE_BAD_ARG;
    const int64_t P = K / 8, Gn = K / 16;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; n++)
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_value(x_bf16[m * K + k]) * e2m1_value(get_code(packed + n * P, k, 4)) *
                       e4m3_value(scales[n * Gn + k / 16]);
            y[m * N + n] = acc * (double)g;
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* mxfp8: E4M3 elements, one E8M0 exponent per 32                             */
/* ------------------------------------------------------------------------ */

/* "metalworking — MLX Quantization" (the newer modes: mxfp8 with groups of 32)
 * and "Quantizing a Model for MLX", section "Modes, bits and mixed recipes"
 * (mxfp8: groups of 32, 8 bits, an exponent per group).  Encodings as read from
 * the OCP Microscaling v1.0 MXFP8 (E4M3) format:
 *  - code byte: sign bit 7, then the E4M3 magnitude (exponent bits 6..3 with
 *    bias 7, mantissa bits 2..0, subnormals m * 2^-9, largest 448); packed 4
 *    per uint32, LSB first (as 8-bit affine codes);
 *  - scale byte s: X = 2^(s - 127), as for mxfp4;
 *  - quantize a group of 32: shared exponent floor(log2 amax) - 8 (8 = the
 *    largest E4M3 exponent), clamped to [-127, 127]; an all-zero group gets
 *    s = 0; each element the E4M3 magnitude nearest to |w| / X (exact in fp64),
 *    ties to even, saturating at 448; sign only on a non-zero magnitude;
 *  - value X * e4m3(code), exact in fp64 (rounded once to fp32 / bf16). */
static double e4m3_signed_value(uint32_t c)
{
    double v = e4m3_value((uint8_t)(c & 0x7Fu));
    return (c & 0x80u) ? -v : v;
}

int oracle_mxfp8_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales)
{
    if (!w || !packed || !scales || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    const int64_t P = K / 4, Gn = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        const float *wr = w + n * K;
        uint32_t *pr = packed + n * P;
        for (int64_t j = 0; j < P; j++) pr[j] = 0u;
        for (int64_t g = 0; g < Gn; g++) {
            double amax = 0.0;
            for (int i = 0; i < 32; i++) {
                double a = fabs((double)wr[g * 32 + i]);
                if (a > amax) amax = a;
            }
            int shared = -127;
            if (amax > 0.0) {
                int ex;
                frexp(amax, &ex);           /* floor(log2 amax) = ex - 1 */
                shared = (ex - 1) - 8;
                if (shared < -127) shared = -127;
                if (shared > 127) shared = 127;
            }
            scales[n * Gn + g] = (uint8_t)(shared + 127);
            for (int i = 0; i < 32; i++) {
                const double v = (double)wr[g * 32 + i];
                uint32_t c = e4m3_bits_from_double(fabs(v) * ldexp(1.0, -shared));   /* exact product */
                if (v < 0.0 && c != 0u) c |= 0x80u;
                put_code(pr, g * 32 + i, 8, c);
            }
        }
    }
    return ORACLE_OK;
}

static double mx8_value(const uint32_t *prow, const uint8_t *srow, int64_t k)
{
    return e8m0_value(srow[k / 32]) * e4m3_signed_value(get_code(prow, k, 8));
}

int oracle_mxfp8_dequantize_f32(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K, float *out)
{
    if (!packed || !scales || !out || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    const int64_t P = K / 4, Gn = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) out[n * K + k] = (float)mx8_value(packed + n * P, scales + n * Gn, k);
    return ORACLE_OK;
}

int oracle_mxfp8_matmul(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                        const uint8_t *scales, int64_t N, double *y)
{
    if (!x_bf16 || !packed || !scales || !y || M <= 0 || bad_mx_shape(N, K)) return ORACLE_BAD_ARG;
    const int64_t P = K / 4, Gn = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; n++)
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_value(x_bf16[m * K + k]) * mx8_value(packed + n * P, scales + n * Gn, k);
            y[m * N + n] = acc;
        }
    return ORACLE_OK;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
