/*
 * oracle.c -- plain, slow, double-precision CPU oracle for the weight-only
 * quantized projection GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; neither includes the other.
 *
 * Sources (the pages the method is described on):
 *   [Q4]  "RT-J -- int4 (Q4-style, mixed-precision) quantized checkpoints",
 *         section "Quantization format": uint4 codes in groups of 32 along the
 *         input dimension, two codes per byte with the low nibble holding the
 *         even index, one fp16 (scale, min) pair per group, and
 *         W[o,i] ~= nibble * scale + min; group ranges picked by a min-MSE clip
 *         search over a shrink grid running from 1.0 down to 0.8.
 *   [Q8]  "RT-J -- int8 (Q8_0-style) quantized checkpoints", section
 *         "Quantization format": int8 codes with one symmetric fp32 scale per
 *         output row, W[o,i] ~= q[o,i] * scale[o], scale[o] = max|W[o,:]|/127.
 *   [F8]  "RT-J -- FP8 E4M3 checkpoints", section "FP8 Format": each 2-D
 *         weight matrix holds float8_e4m3fn values as they are (no scale).
 *   [GEMM] Both cards, opening paragraph: the engine dequantizes inside the
 *         GEMM; the projection computes Y = X * W^T with W indexed [out, in].
 *
 * Readings where the pages are silent (each one is listed with its reason in
 * the design notes): the shrink grid has n_grid points
 * s_j = 1 - 0.2*j/(n_grid-1) (21 by default), shrinking multiplies both range
 * ends by s_j, the MSE is taken with the fp16-rounded (scale, min) that
 * dequantization will use, codes round half-to-even and clamp to [0,15], ties
 * between grid points keep the smallest j, a group whose fp16 scale is zero
 * stores all-zero codes, the companion tensor is [N, K/32, 2] with scale
 * first, the int8 codes round half-to-even and clamp to [-127, 127], and an
 * FP8 weight is the nearest E4M3 value (ties to the even code) with magnitudes
 * above 464, which would round past the largest finite value 448, out of range.
 *
 * Every function below states the step of the pages it follows.  All
 * arithmetic on weights is in IEEE double; dequantized values are exact in
 * double (a 4-bit code times an fp16 scale plus an fp16 min, or an 8-bit code
 * times an fp32 scale), so the GEMM reference differs from the exact product
 * only by the double-precision summation.
 *
 * Compile with -O2 -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

/* ---------------------------------------------------------------------------
 * fp16 encode / decode.  The pages store (scale, min) as IEEE binary16
 * ([Q4]).  Encoding rounds a double straight to binary16 (one rounding),
 * nearest-even, with subnormals; values at or above 65520 in magnitude become
 * infinity.
 * ------------------------------------------------------------------------- */
uint16_t oracle_f16_from_double(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)0x7E00u;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;               /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14;         /* binary16 subnormal quantum is 2^-24 */
    double quantum = ldexp(1.0, E - 10);
    double q = a / quantum;       /* exact: division by a power of two */
    double r = nearbyint(q);      /* default rounding mode: nearest-even */
    uint32_t n = (uint32_t)r;
    if (E == -14 && n < 1024u) return (uint16_t)(sign | n);  /* subnormal */
    if (n >= 2048u) { n >>= 1; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint32_t)((E + 15) << 10) | (n - 1024u));
}

double oracle_f16_to_double(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0)       v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else              v = ldexp((double)(m + 1024), e - 25);
    return s ? -v : v;
}

/* ---------------------------------------------------------------------------
 * Nibble packing ([Q4]): byte j of a row holds code 2j in its low nibble and
 * code 2j+1 in its high nibble.
 * ------------------------------------------------------------------------- */
void oracle_pack_nibbles(const uint8_t *codes, int64_t n_codes, uint8_t *bytes)
{
    for (int64_t j = 0; j < n_codes / 2; ++j)
        bytes[j] = (uint8_t)((codes[2 * j] & 0x0F) | ((codes[2 * j + 1] & 0x0F) << 4));
}

void oracle_unpack_nibbles(const uint8_t *bytes, int64_t n_codes, uint8_t *codes)
{
    for (int64_t j = 0; j < n_codes / 2; ++j) {
        codes[2 * j] = bytes[j] & 0x0F;
        codes[2 * j + 1] = (bytes[j] >> 4) & 0x0F;
    }
}

/* ---------------------------------------------------------------------------
 * One shrink-grid factor ([Q4] "shrink grid 1.0 -> 0.8"): n_grid evenly
 * spaced points from 1.0 down to 0.8; a one-point grid is {1.0}.
 * ------------------------------------------------------------------------- */
double oracle_shrink_factor(int j, int n_grid)
{
    if (n_grid <= 1) return 1.0;
    return 1.0 - (0.2 * (double)j) / (double)(n_grid - 1);
}

/* Candidate j for one group of 32 values: the fp16 (scale, min) pair for the
 * shrunk range [s*lo, s*hi], the codes it yields, and the squared error of
 * the reconstruction with those fp16 values.  Returns the error. */
double oracle_q4_candidate(const float *w, double lo, double hi, double s,
                           uint16_t *scale16, uint16_t *min16, uint8_t *codes)
{
    double lo_j = s * lo;
    double hi_j = s * hi;
    uint16_t sc_bits = oracle_f16_from_double((hi_j - lo_j) / 15.0);
    uint16_t mn_bits = oracle_f16_from_double(lo_j);
    double sc = oracle_f16_to_double(sc_bits);
    double mn = oracle_f16_to_double(mn_bits);
    double err = 0.0;
    for (int i = 0; i < 32; ++i) {
        int q = 0;
        if (sc != 0.0) {
            double t = nearbyint(((double)w[i] - mn) / sc);
            q = t < 0.0 ? 0 : (t > 15.0 ? 15 : (int)t);
        }
        codes[i] = (uint8_t)q;
        double d = (double)w[i] - ((double)q * sc + mn);
        err += d * d;
    }
    *scale16 = sc_bits;
    *min16 = mn_bits;
    return err;
}

/* ---------------------------------------------------------------------------
 * q4 g32 quantizer ([Q4] "Quantization format"): for every row o and group g
 * of 32 consecutive inputs, take the group's min and max, try every shrink
 * factor, keep the (scale, min) of least squared error (first one on ties),
 * and pack the codes.  W is fp32 [N, K]; Wq is [N, K/2]; scale_min is fp16
 * bits [N, K/32, 2] (scale first).  jstar, when not NULL, receives the chosen
 * grid index per group [N, K/32].  Returns 0, or -1 on a bad argument or a
 * weight that is not finite or exceeds the binary16 range.
 * ------------------------------------------------------------------------- */
int oracle_quant_q4_g32(const float *W, int64_t N, int64_t K, int n_grid,
                        uint8_t *Wq, uint16_t *scale_min, int32_t *jstar)
{
    if (N < 0 || K < 0 || K % 32 != 0 || n_grid < 1) return -1;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i]) || fabs((double)W[i]) > 65504.0) return -1;
    const int64_t G = K / 32;
    for (int64_t o = 0; o < N; ++o) {
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + o * K + g * 32;
            double lo = w[0], hi = w[0];
            for (int i = 1; i < 32; ++i) {
                if (w[i] < lo) lo = w[i];
                if (w[i] > hi) hi = w[i];
            }
            double best = INFINITY;
            int best_j = 0;
            uint16_t best_sc = 0, best_mn = 0;
            uint8_t best_codes[32] = {0};
            for (int j = 0; j < n_grid; ++j) {
                uint16_t sc, mn;
                uint8_t codes[32];
                double err = oracle_q4_candidate(w, lo, hi, oracle_shrink_factor(j, n_grid),
                                                 &sc, &mn, codes);
                if (err < best) {
                    best = err;
                    best_j = j;
                    best_sc = sc;
                    best_mn = mn;
                    for (int i = 0; i < 32; ++i) best_codes[i] = codes[i];
                }
            }
            oracle_pack_nibbles(best_codes, 32, Wq + o * (K / 2) + g * 16);
            scale_min[(o * G + g) * 2 + 0] = best_sc;
            scale_min[(o * G + g) * 2 + 1] = best_mn;
            if (jstar) jstar[o * G + g] = best_j;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * q8 per-row quantizer ([Q8] "Quantization format"): scale[o] is the fp32
 * quotient max|W[o,:]| / 127, and each code is w / scale rounded half-to-even
 * and clamped to [-127, 127].  A zero row gets scale 0 and zero codes.
 * ------------------------------------------------------------------------- */
int oracle_quant_q8_row(const float *W, int64_t N, int64_t K, int8_t *Wq, float *scale)
{
    if (N < 0 || K < 0) return -1;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i])) return -1;
    for (int64_t o = 0; o < N; ++o) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(W[o * K + k]);
            if (a > amax) amax = a;
        }
        volatile float sc = amax / 127.0f;   /* one fp32 division */
        scale[o] = sc;
        for (int64_t k = 0; k < K; ++k) {
            int q = 0;
            if (sc != 0.0f) {
                double t = nearbyint((double)W[o * K + k] / (double)sc);
                q = t < -127.0 ? -127 : (t > 127.0 ? 127 : (int)t);
            }
            Wq[o * K + k] = (int8_t)q;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Dequantization, exact in double.
 *   q4 ([Q4]): W[o,k] = nibble(o,k) * scale[o, k/32] + min[o, k/32].
 *   q8 ([Q8]): W[o,k] = q[o,k] * scale[o].
 * ------------------------------------------------------------------------- */
void oracle_dequant_q4(const uint8_t *Wq, const uint16_t *scale_min, int64_t N, int64_t K,
                       double *W)
{
    const int64_t G = K / 32;
    for (int64_t o = 0; o < N; ++o) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = Wq[o * (K / 2) + k / 2];
            int nib = (k % 2 == 0) ? (b & 0x0F) : ((b >> 4) & 0x0F);
            double sc = oracle_f16_to_double(scale_min[(o * G + k / 32) * 2 + 0]);
            double mn = oracle_f16_to_double(scale_min[(o * G + k / 32) * 2 + 1]);
            W[o * K + k] = (double)nib * sc + mn;
        }
    }
}

void oracle_dequant_q8(const int8_t *Wq, const float *scale, int64_t N, int64_t K, double *W)
{
    for (int64_t o = 0; o < N; ++o)
        for (int64_t k = 0; k < K; ++k)
            W[o * K + k] = (double)Wq[o * K + k] * (double)scale[o];
}

/* ---------------------------------------------------------------------------
 * FP8 E4M3 ([F8]).  float8_e4m3fn is the finite-only 8-bit E4M3 format: one
 * sign bit, four exponent bits with bias 7, three mantissa bits.  Exponent
 * field e = 0 holds the subnormals m * 2^-9; e = 1..15 hold (1 + m/8) *
 * 2^(e-7), except that S.1111.111 is NaN; there is no infinity, and the
 * largest finite magnitude is 1.75 * 2^8 = 448.
 * ------------------------------------------------------------------------- */
double oracle_e4m3_to_double(uint8_t b)
{
    const int sign = (b >> 7) & 1, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = (double)m * ldexp(1.0, -9);
    else
        v = (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
    return sign ? -v : v;
}

/* The nearest finite E4M3 value to x, by search over the 127 non-negative
 * finite codes; of two equally near codes the even one (mantissa bit 0
 * clear).  Returns -1 for NaN and for |x| > 464 (half way between 448 and the
 * next step 480, which the format does not have); 0 otherwise. */
int oracle_e4m3_from_double(double x, uint8_t *out)
{
    if (isnan(x) || fabs(x) > 464.0) return -1;
    const double a = fabs(x);
    int best = 0;
    double best_d = a;                       /* distance to code 0 (zero) */
    for (int c = 1; c <= 0x7E; ++c) {
        const double d = fabs(a - oracle_e4m3_to_double((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    *out = (uint8_t)(best | (signbit(x) ? 0x80 : 0));
    return 0;
}

/* [F8]: each weight kept as its E4M3 rounding.  Returns -1 (and
 * leaves the rest of `out` unspecified) at the first weight out of range. */
int oracle_quant_e4m3(const float *W, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        if (oracle_e4m3_from_double((double)W[i], &out[i]) != 0) return -1;
    return 0;
}

void oracle_dequant_e4m3(const uint8_t *Wq, int64_t N, int64_t K, double *W)
{
    for (int64_t i = 0; i < N * K; ++i) W[i] = oracle_e4m3_to_double(Wq[i]);
}

/* ---------------------------------------------------------------------------
 * The projection ([GEMM]): Y[m,o] = sum_k X[m,k] * W[o,k], summed over k in
 * ascending order in double.  `rows` (may be NULL for all rows 0..M-1) lists
 * which rows of X to compute; Y is [n_rows, N].  wrow is caller scratch of K
 * doubles holding one dequantized weight row at a time.
 * ------------------------------------------------------------------------- */
static void gemm_rows(const float *X, int64_t K, const double *wrow, int64_t o, int64_t N,
                      const int64_t *rows, int64_t n_rows, double *Y)
{
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t m = rows ? rows[r] : r;
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += (double)X[m * K + k] * wrow[k];
        Y[r * N + o] = acc;
    }
}

int oracle_gemm_q4(const float *X, const uint8_t *Wq, const uint16_t *scale_min,
                   int64_t M, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows,
                   double *Y, double *wrow)
{
    if (K % 32 != 0) return -1;
    if (!rows) n_rows = M;
    for (int64_t o = 0; o < N; ++o) {
        oracle_dequant_q4(Wq + o * (K / 2), scale_min + o * (K / 32) * 2, 1, K, wrow);
        gemm_rows(X, K, wrow, o, N, rows, n_rows, Y);
    }
    return 0;
}

int oracle_gemm_q8(const float *X, const int8_t *Wq, const float *scale,
                   int64_t M, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows,
                   double *Y, double *wrow)
{
    if (!rows) n_rows = M;
    for (int64_t o = 0; o < N; ++o) {
        oracle_dequant_q8(Wq + o * K, scale + o, 1, K, wrow);
        gemm_rows(X, K, wrow, o, N, rows, n_rows, Y);
    }
    return 0;
}

int oracle_gemm_e4m3(const float *X, const uint8_t *Wq, int64_t M, int64_t N, int64_t K,
                     const int64_t *rows, int64_t n_rows, double *Y, double *wrow)
{
    if (!rows) n_rows = M;
    for (int64_t o = 0; o < N; ++o) {
        oracle_dequant_e4m3(Wq + o * K, 1, K, wrow);
        gemm_rows(X, K, wrow, o, N, rows, n_rows, Y);
    }
    return 0;
}
