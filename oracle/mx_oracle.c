/*
 * mx_oracle.c -- plain, slow, obviously-correct CPU oracle for the MX
 * block-scaled matrix multiply C = A * B^T (NT layout).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it follows:
 *  - The operation and its contract come from the 5ulink.com page
 *    "PyTorch 接上 FlyDSL" (support-matrix table, row "MXFP 缩放 GEMM":
 *    A row-major, B column-major, K a multiple of 128; and the note under the
 *    table: one E8M0 scale per 32 values ("BlockWise1x32"), FP32
 *    accumulation, FP16/BF16 output).  The devotd.net page, section 2, names
 *    the MXFP8 / MXFP4 NT suites.
 *  - The pages name the element formats but do not define them; the bit
 *    encodings below are the public OCP Microscaling (MX) v1.0 definitions
 *    (E4M3 "fn" variant with max 448 and S.1111.111 = NaN, E2M1 with
 *    magnitudes {0,0.5,1,1.5,2,3,4,6}, E8M0 value 2^(e-127), 0xFF = NaN).
 *  - The quantisation rule (scale exponent = floor(log2(block amax)) - emax,
 *    emax = 8 for E4M3 and 2 for E2M1; elements round-to-nearest-even with
 *    saturation) is the OCP MX conversion recipe.
 *
 * Arithmetic: every decoded value, every product and every block sum is
 * exact in binary64; block contributions are summed in FP64 and the result
 * is rounded to BF16 once, directly from FP64 (no FP32 intermediate).
 *
 * Readings where the sources are silent (each also listed in the design
 * notes of the repository):
 *  - all-zero block: scale byte 0x00, elements keep the sign of each zero;
 *  - a block holding a NaN or an infinity: scale byte 0xFF, all element
 *    codes 0;
 *  - a negative value that rounds to zero keeps its sign (0x80 / nibble 0x8).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define MXO_FMT_MXFP8 0
#define MXO_FMT_MXFP4 1

/* ---------------------------------------------------------------- decoders */

/* E4M3 (OCP "fn"): sign bit 7, exponent bits 6..3 (bias 7), mantissa 2..0.
 * Exponent field 0 is subnormal: m/8 * 2^-6.  0x7F and 0xFF are NaN; there is
 * no infinity.                                                              */
double mxo_decode_e4m3(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
 * Exponent field 0 is subnormal: m * 0.5.  No NaN, no infinity.            */
double mxo_decode_e2m1(uint8_t nibble)
{
    int s = (nibble >> 3) & 1;
    int e = (nibble >> 1) & 0x3;
    int m = nibble & 0x1;
    double v;
    if (e == 0)
        v = 0.5 * (double)m;
    else
        v = ldexp(1.0 + (double)m / 2.0, e - 1);
    return s ? -v : v;
}

/* E8M0 scale: unsigned exponent, value 2^(b-127); 0xFF is NaN.             */
double mxo_decode_e8m0(uint8_t b)
{
    if (b == 0xFF)
        return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* Element k of row `row` of an operand stored NT-style: MXFP8 rows hold K
 * bytes; MXFP4 rows hold K/2 bytes, element 2j in the low nibble of byte j
 * and element 2j+1 in the high nibble.                                      */
static double element(int fmt, const uint8_t *rowp, int64_t k)
{
    if (fmt == MXO_FMT_MXFP8)
        return mxo_decode_e4m3(rowp[k]);
    uint8_t byte = rowp[k / 2];
    uint8_t nib = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return mxo_decode_e2m1(nib);
}

/* ---------------------------------------------------------------- encoders */

/* Round a finite, non-negative value to the E4M3 grid, ties to even, and
 * saturate at 448.  Returns the 7-bit magnitude code.                      */
static uint8_t e4m3_magnitude(double v)
{
    if (v >= 448.0)
        return 0x7E;                        /* saturate to the max finite */
    if (v < ldexp(1.0, -6)) {               /* subnormal binade: step 2^-9 */
        double q = nearbyint(v / ldexp(1.0, -9));      /* 0..8, RNE      */
        return (uint8_t)q;                  /* q == 8 is 2^-6, code 0x08   */
    }
    int ex;
    frexp(v, &ex);                          /* v = f * 2^ex, f in [0.5,1)  */
    int e = ex - 1;                         /* floor(log2 v)               */
    double q = nearbyint((ldexp(v, -e) - 1.0) * 8.0);  /* mantissa, RNE   */
    if (q == 8.0) {
        q = 0.0;
        e += 1;
    }
    int code = ((e + 7) << 3) | (int)q;
    if (code > 0x7E)
        code = 0x7E;
    return (uint8_t)code;
}

uint8_t mxo_encode_e4m3(double v)
{
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    return sign | e4m3_magnitude(fabs(v));
}

/* Round a finite, non-negative value to the E2M1 grid {0,.5,1,1.5,2,3,4,6},
 * ties to even, saturating at 6.  Returns the 3-bit magnitude code.        */
static uint8_t e2m1_magnitude(double v)
{
    if (v >= 6.0)
        return 0x7;
    if (v < 1.0) {                          /* subnormal binade: step 0.5  */
        double q = nearbyint(v / 0.5);      /* 0, 1 or 2                   */
        return (uint8_t)q;                  /* q == 2 is 1.0, code 0b010   */
    }
    int ex;
    frexp(v, &ex);
    int e = ex - 1;                         /* 0, 1 or 2                   */
    double q = nearbyint((ldexp(v, -e) - 1.0) * 2.0);
    if (q == 2.0) {
        q = 0.0;
        e += 1;
    }
    int code = ((e + 1) << 1) | (int)q;
    if (code > 0x7)
        code = 0x7;
    return (uint8_t)code;
}

uint8_t mxo_encode_e2m1(double v)
{
    if (isnan(v))
        return 0x0;                         /* E2M1 has no NaN code        */
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    return sign | e2m1_magnitude(fabs(v));
}

/* floor(log2 |x|) of a non-zero finite FP32 value, read from its exponent
 * bits (subnormals included), never from a rounded log2.                   */
static int floor_log2_f32(float x)
{
    int ex;
    frexp((double)fabsf(x), &ex);           /* exact: FP32 -> FP64         */
    return ex - 1;
}

/* OCP MX quantisation of one operand, rows R, length K (K % 32 == 0).
 * X: FP32 [R][K].  Q: MXFP8 -> [R][K] bytes, MXFP4 -> [R][K/2] bytes
 * (element 2j low nibble).  S: E8M0 [R][K/32].
 * Per 32-block: amax = max |x|; scale exponent s = floor(log2 amax) - emax
 * clamped to [-127, 127]; element = RNE(x / 2^s) saturated.               */
void mxo_quantize(int fmt, int64_t R, int64_t K, const float *X,
                  uint8_t *Q, uint8_t *S)
{
    const int emax = (fmt == MXO_FMT_MXFP8) ? 8 : 2;
    const int64_t nblk = K / 32;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t j = 0; j < nblk; ++j) {
            const float *xb = X + r * K + j * 32;
            float amax = 0.0f;
            int nonfinite = 0;
            for (int t = 0; t < 32; ++t) {
                if (!isfinite(xb[t]))
                    nonfinite = 1;
                else if (fabsf(xb[t]) > amax)
                    amax = fabsf(xb[t]);
            }
            int s;
            uint8_t sbyte;
            if (nonfinite) {
                sbyte = 0xFF;
                s = 0;
            } else if (amax == 0.0f) {
                s = -127;
                sbyte = 0x00;
            } else {
                s = floor_log2_f32(amax) - emax;
                if (s < -127) s = -127;
                if (s > 127) s = 127;
                sbyte = (uint8_t)(s + 127);
            }
            S[r * nblk + j] = sbyte;
            for (int t = 0; t < 32; ++t) {
                int64_t k = j * 32 + t;
                double q = nonfinite ? 0.0 : ldexp((double)xb[t], -s);
                if (fmt == MXO_FMT_MXFP8) {
                    Q[r * K + k] = nonfinite ? 0x00 : mxo_encode_e4m3(q);
                } else {
                    uint8_t nib = nonfinite ? 0x0 : mxo_encode_e2m1(q);
                    uint8_t *bp = Q + r * (K / 2) + k / 2;
                    if (k % 2 == 0)
                        *bp = (uint8_t)((*bp & 0xF0) | nib);
                    else
                        *bp = (uint8_t)((*bp & 0x0F) | (nib << 4));
                }
            }
        }
    }
}

/* ------------------------------------------------------------ BF16 rounding */

/* Round a binary64 value to bfloat16 (8 significant bits, exponent range of
 * binary32), round-to-nearest-even, directly from FP64.  Overflow gives
 * +-Inf, NaN gives the quiet NaN 0x7FC0 (sign kept).                       */
uint16_t mxo_bf16_rne(double x)
{
    if (isnan(x))
        return signbit(x) ? 0xFFC0 : 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    if (isinf(a))
        return sign | 0x7F80;
    if (a == 0.0)
        return sign;
    int ex;
    frexp(a, &ex);
    int e = ex - 1;                          /* floor(log2 a)               */
    if (e < -126)
        e = -126;                            /* subnormal spacing 2^-133    */
    double ulp = ldexp(1.0, e - 7);
    double q = nearbyint(a / ulp);           /* exact division, RNE         */
    double r = q * ulp;
    const double bf16_max = ldexp(255.0, 120);   /* (2 - 2^-7) * 2^127     */
    if (r > bf16_max)
        return sign | 0x7F80;
    float f = (float)r;                      /* exact: r is a bf16 value    */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | ((bits >> 16) & 0x7FFF));
}

/* ------------------------------------------------------------------- GEMM */

/* One output element: the FP64 sum over the K/32 blocks of
 * 2^(SA-127) * 2^(SB-127) * sum_t a_t * b_t, plus the magnitude sum
 * sum_k |a_k * b_k| of the dequantised products (the tolerance's scale).   */
static void one_element(int fmt, int64_t K,
                        const uint8_t *arow, const uint8_t *sarow,
                        const uint8_t *brow, const uint8_t *sbrow,
                        double *value, double *abssum)
{
    const int64_t nblk = K / 32;
    double acc = 0.0, mag = 0.0;
    for (int64_t j = 0; j < nblk; ++j) {
        double scale = mxo_decode_e8m0(sarow[j]) * mxo_decode_e8m0(sbrow[j]);
        double blk = 0.0, blkmag = 0.0;
        for (int t = 0; t < 32; ++t) {
            int64_t k = j * 32 + t;
            double p = element(fmt, arow, k) * element(fmt, brow, k);
            blk += p;
            blkmag += fabs(p);
        }
        acc += scale * blk;
        mag += fabs(scale) * blkmag;
    }
    *value = acc;
    *abssum = mag;
}

static int64_t row_bytes(int fmt, int64_t K)
{
    return fmt == MXO_FMT_MXFP8 ? K : K / 2;
}

/* Full product.  A: [M][row_bytes], SA: [M][K/32], B: [N][row_bytes],
 * SB: [N][K/32], C: BF16 bits [M][N].  `exact` and `abssum` may be NULL;
 * when given they receive the unrounded FP64 value and sum |a*b| per
 * element, [M][N].                                                         */
void mxo_gemm(int fmt, int64_t M, int64_t N, int64_t K,
              const uint8_t *A, const uint8_t *SA,
              const uint8_t *B, const uint8_t *SB,
              uint16_t *C, double *exact, double *abssum)
{
    const int64_t rb = row_bytes(fmt, K), nblk = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double v, mag;
            one_element(fmt, K, A + m * rb, SA + m * nblk,
                        B + n * rb, SB + n * nblk, &v, &mag);
            C[m * N + n] = mxo_bf16_rne(v);
            if (exact) exact[m * N + n] = v;
            if (abssum) abssum[m * N + n] = mag;
        }
    }
}

/* Selected elements only: (im[i], in[i]) for i < npts.  Same outputs as
 * mxo_gemm, one entry per point.                                           */
void mxo_gemm_points(int fmt, int64_t M, int64_t N, int64_t K,
                     const uint8_t *A, const uint8_t *SA,
                     const uint8_t *B, const uint8_t *SB,
                     int64_t npts, const int64_t *im, const int64_t *in,
                     uint16_t *C, double *exact, double *abssum)
{
    const int64_t rb = row_bytes(fmt, K), nblk = K / 32;
    (void)M;
    (void)N;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < npts; ++i) {
        double v, mag;
        one_element(fmt, K, A + im[i] * rb, SA + im[i] * nblk,
                    B + in[i] * rb, SB + in[i] * nblk, &v, &mag);
        C[i] = mxo_bf16_rne(v);
        if (exact) exact[i] = v;
        if (abssum) abssum[i] = mag;
    }
}

/* --------------------------------------------------------- dense BF16 GEMM */

/* A BF16 value from its bit pattern: the upper half of a binary32, widened
 * exactly to binary64.                                                     */
double mxo_decode_bf16(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* C = A * B^T for dense BF16 operands (the dense-GEMM comparison suite of
 * the 5ulink.com page, table 内核级成绩): A [M][K], B [N][K] BF16 bits, C
 * BF16 bits [M][N].  Every product of two BF16 values is exact in binary64;
 * the products are summed in FP64 in k order and the sum is rounded to BF16
 * once.  `exact` / `abssum` as in mxo_gemm (may be NULL).                   */
void mxo_gemm_bf16(int64_t M, int64_t N, int64_t K,
                   const uint16_t *A, const uint16_t *B,
                   uint16_t *C, double *exact, double *abssum)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = mxo_decode_bf16(A[m * K + k]) * mxo_decode_bf16(B[n * K + k]);
                acc += p;
                mag += fabs(p);
            }
            C[m * N + n] = mxo_bf16_rne(acc);
            if (exact) exact[m * N + n] = acc;
            if (abssum) abssum[m * N + n] = mag;
        }
    }
}

/* ------------------------------------------------------- fused epilogue */

/* The activations of the fused epilogue, in binary64, from their
 * definitions: ReLU max(x, 0) (NaN stays NaN), SiLU x * sigmoid(x) =
 * x / (1 + e^-x), GELU x * Phi(x) with the standard normal CDF
 * Phi(x) = erfc(-x / sqrt(2)) / 2.                                          */
double mxo_activation(int act, double x)
{
    switch (act) {
    case 1:
        return x < 0.0 ? 0.0 : x;
    case 2:
        return x / (1.0 + exp(-x));
    case 3:
        return 0.5 * x * erfc(-x / sqrt(2.0));
    default:
        return x;
    }
}

/* Epilogue fusion (the roadmap's "GEMM 尾部融合" on the 5ulink.com page,
 * section 怎么用起来): from the unrounded product `exact` [M][N] (binary64,
 * as mxo_gemm returns it), out = act(exact + bias[n]) + residual[m][n] in
 * binary64, rounded to BF16 once.  bias: BF16 bits [N] or NULL; residual:
 * BF16 bits [M][N] or NULL.  `pre` (may be NULL) receives exact + bias.    */
void mxo_epilogue(int64_t M, int64_t N, const double *exact,
                  const uint16_t *bias, int act, const uint16_t *residual,
                  uint16_t *C, double *pre)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double v = exact[m * N + n];
            if (bias)
                v += mxo_decode_bf16(bias[n]);
            if (pre)
                pre[m * N + n] = v;
            v = mxo_activation(act, v);
            if (residual)
                v += mxo_decode_bf16(residual[m * N + n]);
            C[m * N + n] = mxo_bf16_rne(v);
        }
    }
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP).        */
int mxo_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
