/*
 * CPU oracle for the NVFP4 linear layer.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the bench's CPU-baseline leg may
 * load this file's library.  Nothing on the product path (the C-ABI library
 * and its kernels) includes, links or calls it, and it shares no code, table
 * or constant with that path.
 *
 * What it follows.  The pages (imp home page, "How does it work?": weights are
 * kept as NVFP4 and multiplied in that format; Ignis README, "The decode round":
 * decode linears stream packed weights at the card's bandwidth; imp v0.20.0
 * release notes, "Highlights": a first-party NVFP4 quantizer) only name the
 * format.  Its definition is the public NVFP4 / OCP-microscaling one:
 *   - E2M1 element codes: 1 sign, 2 exponent (bias 1), 1 mantissa bit;
 *   - one E4M3 (FN variant: bias 7, no infinity, NaN = S.1111.111) scale per
 *     16 consecutive elements along the reduction axis;
 *   - one fp32 per-tensor scale gs = amax_tensor / (448 * 6).
 *
 * Readings where the definition leaves a step open (each one is listed with
 * its reason in the design notes of the repository):
 *   R1  encoders pick the representable value nearest to the input; a tie goes
 *       to the even code (mantissa LSB 0); magnitudes above the largest finite
 *       value saturate to it; the sign is kept, so a negative input that rounds
 *       to zero gives negative zero (E2M1 code 8).
 *   R2  quantizer arithmetic is IEEE binary32, round-to-nearest-even, in this
 *       exact order:  gs = amax / 2688.0f  (gs = 1.0f for an all-zero tensor);
 *       denom = gs * 6.0f;  s = enc_e4m3(amax_block / denom);
 *       r = E4M3(s) * gs;  code = enc_e2m1(x / r).
 *   R3  a block whose r is zero (its scale rounded to zero) stores +0 codes.
 *   R4  codes are packed two per byte, element 2j in the low nibble.
 *   R5  everything after decoding (dot products, scaling) runs in fp64; the
 *       per-element products x * E2M1 * E4M3 are exact there.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -fopenmp -ffp-contract=off
 * (no -ffast-math): fp32 expressions below must round exactly once each.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Code tables, built from the bit-field definitions of the formats.   */
/* ------------------------------------------------------------------ */

static double g_e2m1[16];
static double g_e4m3[256];
static int g_ready = 0;

static void build_tables(void)
{
    if (g_ready) return;
    /* E2M1: bits s e1 e0 m.  e == 0: (-1)^s * m * 0.5 (subnormal);
       otherwise (-1)^s * (1 + m/2) * 2^(e-1).                          */
    for (int c = 0; c < 16; ++c) {
        int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
        double mag = (e == 0) ? m * 0.5 : (1.0 + m / 2.0) * ldexp(1.0, e - 1);
        g_e2m1[c] = s ? -mag : mag;
    }
    /* E4M3 (FN): bits s eeee mmm, bias 7.  e == 0: (m/8) * 2^-6;
       S.1111.111 is NaN; there is no infinity.                         */
    for (int c = 0; c < 256; ++c) {
        int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
        double mag;
        if (e == 15 && m == 7) mag = NAN;
        else if (e == 0) mag = (m / 8.0) * ldexp(1.0, -6);
        else mag = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
        g_e4m3[c] = s ? -mag : mag;
    }
    g_ready = 1;
}

double nvo_e2m1_value(int code) { build_tables(); return g_e2m1[code & 15]; }
double nvo_e4m3_value(int code) { build_tables(); return g_e4m3[code & 255]; }

/* Nearest representable magnitude among codes [0, ncodes) of a table that is
   ascending in its first ncodes entries; ties go to the even code.  Inputs at
   or above the largest entry saturate to it.  Below it, |a - table[c]| is
   exact in double for every entry that can be nearest (a has 24 significant
   bits, the entries at most 4, and their exponents are close), so the tie
   test compares exact distances; entries whose distance rounds are far from
   a and can neither win nor tie.                                            */
static int nearest_code(double a, const double* table, int ncodes)
{
    if (a >= table[ncodes - 1]) return ncodes - 1;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < ncodes; ++c) {
        double d = fabs(a - table[c]);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* R1 for E2M1: nearest of {0, .5, 1, 1.5, 2, 3, 4, 6}, tie -> even code,
   saturate at 6, sign bit kept.  Input must be finite.                    */
int nvo_e2m1_encode(float f)
{
    build_tables();
    int sign = signbit(f) ? 8 : 0;
    return sign | nearest_code(fabs((double)f), g_e2m1, 8);
}

/* R1 for E4M3: nearest of the 127 finite non-negative codes (0x00..0x7E),
   tie -> even code, saturate at 448, sign bit kept.  Input must be finite.  */
int nvo_e4m3_encode(float f)
{
    build_tables();
    int sign = signbit(f) ? 0x80 : 0;
    return sign | nearest_code(fabs((double)f), g_e4m3, 127);
}

/* Per-tensor scale (R2): gs = amax / 2688.0f, or 1.0f for an all-zero tensor. */
float nvo_global_scale(const float* x, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) return 1.0f;
    volatile float q = amax / 2688.0f; /* one binary32 division */
    return q;
}

/* Quantize x[rows, cols] (cols % 16 == 0) with per-tensor scale gs (R2-R4).
   codes: rows * cols/2 bytes, row-major; scales: rows * cols/16 bytes,
   row-major (one E4M3 byte per 16-element block along cols).              */
void nvo_quantize(const float* x, int64_t rows, int64_t cols, float gs,
                  uint8_t* codes, uint8_t* scales)
{
    build_tables();
    const int64_t nb = cols / 16;
    volatile float denom_v = gs * 6.0f;
    const float denom = denom_v;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + r * cols + b * 16;
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax_b) amax_b = a;
            }
            volatile float ratio = amax_b / denom;
            int s = nvo_e4m3_encode(ratio);
            float sd = (float)g_e4m3[s];
            volatile float rr = sd * gs;
            const float rsc = rr;
            scales[r * nb + b] = (uint8_t)s;
            uint8_t* cb = codes + r * (cols / 2) + b * 8;
            for (int j = 0; j < 8; ++j) {
                int lo = 0, hi = 0;
                if (rsc != 0.0f) {
                    volatile float q0 = xb[2 * j] / rsc;
                    volatile float q1 = xb[2 * j + 1] / rsc;
                    lo = nvo_e2m1_encode(q0);
                    hi = nvo_e2m1_encode(q1);
                }
                cb[j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* w[r, c] = E2M1(code) * E4M3(scale) * gs, in fp64 (exact up to the final
   multiply by gs, which rounds once).                                       */
void nvo_dequantize(const uint8_t* codes, const uint8_t* scales, float gs,
                    int64_t rows, int64_t cols, double* out)
{
    build_tables();
    const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 15);
            double v = g_e2m1[code] * g_e4m3[scales[r * nb + c / 16]];
            out[r * cols + c] = v * (double)gs;
        }
    }
}

/* Decode one quantized row into v[k] = E2M1 * E4M3 (exact, without gs). */
static void decode_row(const uint8_t* codes, const uint8_t* scales, int64_t K,
                       double* v)
{
    for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = codes[k / 2];
        int code = (k & 1) ? (byte >> 4) : (byte & 15);
        v[k] = g_e2m1[code] * g_e4m3[scales[k / 16]];
    }
}

/* W4A16 linear (R5):  y[m, n] = gs_w * sum_k x[m, k] * E2M1(c[n, k]) * E4M3(s[n, k/16]).
   x holds the bf16 activations widened to fp32 (exact); weights are [N, K]
   with row-major codes/scales as written by nvo_quantize.  absdot[m, n] =
   gs_w * sum_k |x * E2M1 * E4M3| feeds the error bound.  absdot may be NULL. */
void nvo_linear_w4a16(const float* x, int64_t M, int64_t K,
                      const uint8_t* codes, const uint8_t* scales, float gs,
                      int64_t N, double* y, double* absdot)
{
    build_tables();
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            decode_row(codes + n * (K / 2), scales + n * (K / 16), K, w);
            for (int64_t m = 0; m < M; ++m) {
                const float* xm = x + m * K;
                double s = 0.0, a = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double p = (double)xm[k] * w[k];
                    s += p;
                    a += fabs(p);
                }
                y[m * N + n] = s * (double)gs;
                if (absdot) absdot[m * N + n] = a * (double)gs;
            }
        }
        free(w);
    }
}

/* W4A4 linear (R5): both operands quantized;
   y[m, n] = gs_x * gs_w * sum_k E2M1(cx) E4M3(sx) E2M1(cw) E4M3(sw).       */
void nvo_linear_w4a4(const uint8_t* xc, const uint8_t* xs, float gsx,
                     int64_t M, int64_t K,
                     const uint8_t* wc, const uint8_t* ws, float gsw,
                     int64_t N, double* y, double* absdot)
{
    build_tables();
    double* xd = (double*)malloc(sizeof(double) * (size_t)(M * K));
    for (int64_t m = 0; m < M; ++m)
        decode_row(xc + m * (K / 2), xs + m * (K / 16), K, xd + m * K);
    const double g = (double)gsx * (double)gsw;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            decode_row(wc + n * (K / 2), ws + n * (K / 16), K, w);
            for (int64_t m = 0; m < M; ++m) {
                const double* xm = xd + m * K;
                double s = 0.0, a = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double p = xm[k] * w[k];
                    s += p;
                    a += fabs(p);
                }
                y[m * N + n] = s * g;
                if (absdot) absdot[m * N + n] = a * g;
            }
        }
        free(w);
    }
    free(xd);
}

int nvo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
