/*
 * mxref.c -- fp64 CPU oracle for the block-scaled projection GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline / reference leg load this file's library.  It shares no code,
 * header, table or constant generator with the CUDA library, and it is never
 * a fallback for it.
 *
 * What it computes (one function per step of the path):
 *
 *   decoders    e4m3fn, e2m1 and E8M0 from their bit fields (closed forms).
 *               The pages name these only as dtypes: "e4m3 weights with
 *               uint8 E8M0 scales (32 x 32 blocks)" and fp4x2 weights with
 *               1 x 32 scales (vLLM DeepSeek-V4 mono runner page,
 *               AttnWeights / MonoLayerWeights layouts).
 *   quant       activations bf16 -> e4m3 with a per-(row, 32-wide K block)
 *               E8M0 scale 2^ceil(log2(amax/448)), or with a per-token fp32
 *               scale amax/448 (sly-radiance README, RadianceLMHeadFp8 row:
 *               "per-token fp8 activation"); weights with 32 x 32 E8M0 blocks,
 *               e2m1 with 1 x 32 E8M0 blocks, or a per-output-channel fp32
 *               scale amax/448 (same README row: "fp8 per output channel").
 *   gemm        y[m, n] = x[m, :] . W[n, :]^T (cortiq-engine dit.rs,
 *               Proj::matmat "y[b, rows] = x[b, cols] . W^T"), each 32-wide K
 *               block scaled by 2^(ea-127) 2^(eb-127), summed in fp64.
 *   epilogues   +bias (dit.rs `linear`: y = x.W^T + b); bias then GELU-tanh
 *               0.5 v (1 + tanh(0.7978845608 (v + 0.044715 v^3))) (vit.rs
 *               vt_bias_act, act == 2: bias added first, then the activation);
 *               SwiGLU silu(g) * u with silu(v) = v / (1 + e^-v) (dit.rs
 *               `silu` and the FFN's silu(g) * u) on a fused [gate; up] N.
 *   tolerance   T[m, n] = sum_k |a_k b_k| of the scaled operands, the term of
 *               the acceptance bound |y_gpu - y| <= 2^-8 |y| + 1e-5 T.
 *   producers   the steps that hand the next GEMM its MX operand directly
 *   of codes    (sly-radiance README, radiance_fused_norm.py row: the fused
 *               add_rms_quant and silu_mul_quant ops return (q_fp8, scale)
 *               for the W4A8 linear; check_fused_norm.py row: their numerics
 *               are compared with the unfused chain).  Each is read as that
 *               unfused chain: bf16 rounding wherever the chain stores bf16,
 *               then the activation quantisation above.  residual add:
 *               bf16(x + r); RMSNorm with a plain weight (cortiq-engine
 *               dit.rs rms_norm: x * rsqrt(mean x^2 + eps) * w), in fp64,
 *               rounded once to bf16.
 *
 * Readings where the pages are silent: the E8M0 exponent is the smallest
 * integer k with amax <= 448 * 2^k (computed by exact comparisons, no log2),
 * biased and clamped to [0, 254]; an all-zero block gets code 0; rounding to
 * e4m3 / e2m1 is round-to-nearest-even, saturating to the largest finite
 * value, and keeps the sign of zero; the per-token scale of an all-zero row is
 * 1.0f; fp32 divisions are IEEE round-to-nearest; gate rows come first in the
 * fused gate|up weight.
 *
 * Threading: OpenMP over output elements; every y[m, n] is summed serially in
 * fixed k order, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ---- formats ---------------------------------------------------------- */
/* A_E2M1_1X32: e2m1 activation codes packed two per byte [M, K/2] (low nibble
 * = even k) with E8M0 scales [M, K/32] -- the W4A4 operand of the MXFP4 GEMM
 * (sly-radiance README, the native MXFP4 W4A4 gemm_afp4wfp4 path); its
 * quantiser is the 1 x 32 e2m1 rule of mxr_quant_w_e2m1_1x32 applied to rows
 * of activations. */
enum { A_E8M0_1X32 = 0, A_F32_ROW = 1, A_E2M1_1X32 = 3 };
enum { B_E4M3_32X32 = 0, B_E2M1_1X32 = 1, B_E4M3_F32_ROW = 2 };
enum { EPI_NONE = 0, EPI_BIAS = 1, EPI_BIAS_GELU_TANH = 2, EPI_SWIGLU = 3 };

/* ---- decoders (closed forms) ----------------------------------------- */

/* e4m3fn: sign 1, exponent 4 (bias 7), mantissa 3; E=0 subnormal
 * 2^-6 * m/8; S.1111.111 is NaN; no infinities; largest finite 448. */
EXPORT double mxr_e4m3_value(unsigned c)
{
    unsigned s = (c >> 7) & 1u, E = (c >> 3) & 15u, m = c & 7u;
    double v;
    if (E == 15u && m == 7u)
        return NAN;
    if (E == 0u)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, (int)E - 7);
    return s ? -v : v;
}

/* e2m1: sign 1, exponent 2 (bias 1), mantissa 1; E=0 subnormal m * 0.5. */
EXPORT double mxr_e2m1_value(unsigned nib)
{
    unsigned s = (nib >> 3) & 1u, E = (nib >> 1) & 3u, m = nib & 1u;
    double v = (E == 0u) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)E - 1);
    return s ? -v : v;
}

/* E8M0: 2^(e-127); e = 255 is NaN. */
EXPORT double mxr_e8m0_value(unsigned e)
{
    return (e == 255u) ? NAN : ldexp(1.0, (int)e - 127);
}

static double bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---- rounding to the code grids --------------------------------------- */

/* Round-to-nearest-even onto a sorted table of non-negative code values
 * tab[0..n-1] (code i has value tab[i]); ties go to the even code; values
 * beyond the last entry saturate to it. */
static unsigned rne_table(double a, const double *tab, unsigned n)
{
    unsigned lo = 0, hi = n - 1;
    if (a >= tab[n - 1])
        return n - 1;
    /* find lo with tab[lo] <= a < tab[lo+1] */
    while (hi - lo > 1) {
        unsigned mid = (lo + hi) / 2;
        if (tab[mid] <= a) lo = mid; else hi = mid;
    }
    {
        double dlo = a - tab[lo], dhi = tab[lo + 1] - a;
        if (dlo < dhi) return lo;
        if (dhi < dlo) return lo + 1;
        return (lo % 2u == 0u) ? lo : lo + 1;
    }
}

static double E4M3_TAB[127]; /* codes 0x00..0x7E */
static double E2M1_TAB[8];   /* codes 0..7 */
static int tabs_ready = 0;

static void init_tabs(void)
{
    unsigned i;
    if (tabs_ready) return;
    for (i = 0; i < 127; ++i) E4M3_TAB[i] = mxr_e4m3_value(i);
    for (i = 0; i < 8; ++i) E2M1_TAB[i] = mxr_e2m1_value(i);
    tabs_ready = 1;
}

/* filled once when the library is loaded, before any OpenMP region */
__attribute__((constructor)) static void init_tabs_at_load(void) { init_tabs(); }

/* RNE to e4m3fn, saturating at 448, sign of zero kept. */
EXPORT unsigned mxr_rne_e4m3(double v)
{
    unsigned c;
    init_tabs();
    c = rne_table(fabs(v), E4M3_TAB, 127);
    return signbit(v) ? (c | 0x80u) : c;
}

/* RNE to e2m1, saturating at 6, sign of zero kept. */
EXPORT unsigned mxr_rne_e2m1(double v)
{
    unsigned c;
    init_tabs();
    c = rne_table(fabs(v), E2M1_TAB, 8);
    return signbit(v) ? (c | 0x8u) : c;
}

/* Biased E8M0 exponent of a block: smallest integer k with
 * amax <= fmax * 2^k, biased by 127 and clamped to [0, 254]; amax = 0 -> 0. */
EXPORT unsigned mxr_e8m0_for_amax(double amax, double fmax)
{
    int k;
    if (!(amax > 0.0))
        return 0u;
    k = (int)floor(log2(amax / fmax)); /* a guess, corrected exactly below */
    while (amax > ldexp(fmax, k)) ++k;
    while (amax <= ldexp(fmax, k - 1)) --k;
    k += 127;
    if (k < 0) k = 0;
    if (k > 254) k = 254;
    return (unsigned)k;
}

/* ---- activation quantisation ----------------------------------------- */

/* bf16 [M, K] -> e4m3 codes [M, K] + E8M0 scales [M, K/32]. */
EXPORT void mxr_quant_act_e8m0(const uint16_t *x, int M, int K, uint8_t *codes, uint8_t *scales)
{
    int m;
    const int KB = K / 32;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int b, k;
        for (b = 0; b < KB; ++b) {
            double amax = 0.0, inv;
            unsigned e;
            for (k = 0; k < 32; ++k) {
                double a = fabs(bf16_to_double(x[(size_t)m * K + b * 32 + k]));
                if (a > amax) amax = a;
            }
            e = mxr_e8m0_for_amax(amax, 448.0);
            scales[(size_t)m * KB + b] = (uint8_t)e;
            inv = ldexp(1.0, 127 - (int)e); /* exact power of two */
            for (k = 0; k < 32; ++k) {
                size_t i = (size_t)m * K + b * 32 + k;
                codes[i] = (uint8_t)mxr_rne_e4m3(bf16_to_double(x[i]) * inv);
            }
        }
    }
}

/* bf16 [R, K] -> e4m3 codes [R, K] + fp32 scale per row s = fl(amax / 448),
 * code = RNE_e4m3(fl(x / s)); an all-zero row has s = 1.  Used for the
 * per-token activation scale and the per-output-channel weight scale. */
EXPORT void mxr_quant_f32_row(const uint16_t *x, int R, int K, uint8_t *codes, float *s_out)
{
    int r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < R; ++r) {
        volatile float amax = 0.0f, s;
        int k;
        for (k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(x[(size_t)r * K + k]));
            if (a > amax) amax = a;
        }
        s = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        s_out[r] = s;
        for (k = 0; k < K; ++k) {
            volatile float q = bf16_to_float(x[(size_t)r * K + k]) / s;
            codes[(size_t)r * K + k] = (uint8_t)mxr_rne_e4m3((double)q);
        }
    }
}

/* ---- bf16 rounding and the producers of MX codes ---------------------- */

/* Round-to-nearest-even of a double onto the bf16 grid (8 significant bits,
 * fp32's exponent range, subnormals down to 2^-133), in one step (no detour
 * through fp32); the sign of zero is kept, a NaN gives the quiet NaN 0x7FC0
 * and magnitudes that round to 2^128 or more give infinity. */
EXPORT unsigned mxr_bf16_rne(double v)
{
    double a = fabs(v), val;
    int ex, E;
    float f;
    uint32_t u;
    unsigned sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return 0x7FC0u;
    if (a == 0.0)
        return sign;
    (void)frexp(a, &ex); /* a = f 2^ex, f in [0.5, 1): a's binary exponent is ex - 1 */
    E = ex - 1;
    if (E < -126)
        E = -126;                                /* subnormal range: quantum 2^-133 */
    val = ldexp(nearbyint(ldexp(a, 7 - E)), E - 7); /* quantum 2^(E-7); ties to even */
    if (val >= ldexp(1.0, 128))
        return sign | 0x7F80u;
    f = (float)val; /* exact: at most 9 significant bits inside fp32's range */
    memcpy(&u, &f, 4);
    return sign | (u >> 16);
}

/* fp64 [n] -> bf16 bits [n], each rounded by mxr_bf16_rne. */
EXPORT void mxr_round_bf16(const double *v, size_t n, uint16_t *out)
{
    size_t i;
    for (i = 0; i < n; ++i) out[i] = (uint16_t)mxr_bf16_rne(v[i]);
}

/* Residual add of two bf16 tensors: bf16(x + r); the sum of two bf16 values
 * is exact in double, so this is a single rounding. */
EXPORT void mxr_add_bf16(const uint16_t *x, const uint16_t *r, size_t n, uint16_t *out)
{
    size_t i;
    for (i = 0; i < n; ++i) out[i] = (uint16_t)mxr_bf16_rne(bf16_to_double(x[i]) + bf16_to_double(r[i]));
}

/* RMSNorm of each row of v [M, K] with a plain per-column weight w [K] (both
 * bf16): y = v * (1 / sqrt(mean_k v^2 + eps)) * w, in fp64 with the squares
 * summed in k order, rounded once to bf16. */
EXPORT void mxr_rmsnorm_bf16(const uint16_t *v, const uint16_t *w, int M, int K, double eps, uint16_t *y)
{
    int m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        double ss = 0.0, inv;
        int k;
        for (k = 0; k < K; ++k) {
            double a = bf16_to_double(v[(size_t)m * K + k]);
            ss += a * a;
        }
        inv = 1.0 / sqrt(ss / (double)K + eps);
        for (k = 0; k < K; ++k) {
            size_t i = (size_t)m * K + k;
            y[i] = (uint16_t)mxr_bf16_rne(bf16_to_double(v[i]) * inv * bf16_to_double(w[k]));
        }
    }
}

/* ---- weight quantisation (test-data preparation) ---------------------- */

/* bf16 W [N, K] -> e4m3 codes [N, K] + E8M0 scales [N/32, K/32] over 32 x 32
 * blocks (N % 32 == 0, K % 32 == 0). */
EXPORT void mxr_quant_w_e4m3_32x32(const uint16_t *w, int N, int K, uint8_t *codes, uint8_t *scales)
{
    int nb;
    const int NB = N / 32, KB = K / 32;
#pragma omp parallel for schedule(static)
    for (nb = 0; nb < NB; ++nb) {
        int b, r, k;
        for (b = 0; b < KB; ++b) {
            double amax = 0.0, inv;
            unsigned e;
            for (r = 0; r < 32; ++r)
                for (k = 0; k < 32; ++k) {
                    double a = fabs(bf16_to_double(w[(size_t)(nb * 32 + r) * K + b * 32 + k]));
                    if (a > amax) amax = a;
                }
            e = mxr_e8m0_for_amax(amax, 448.0);
            scales[(size_t)nb * KB + b] = (uint8_t)e;
            inv = ldexp(1.0, 127 - (int)e);
            for (r = 0; r < 32; ++r)
                for (k = 0; k < 32; ++k) {
                    size_t i = (size_t)(nb * 32 + r) * K + b * 32 + k;
                    codes[i] = (uint8_t)mxr_rne_e4m3(bf16_to_double(w[i]) * inv);
                }
        }
    }
}

/* bf16 W [N, K] -> e2m1 codes packed two per byte [N, K/2] (low nibble =
 * even k) + E8M0 scales [N, K/32]; exponent = smallest k with amax <= 6 * 2^k. */
EXPORT void mxr_quant_w_e2m1_1x32(const uint16_t *w, int N, int K, uint8_t *packed, uint8_t *scales)
{
    int n;
    const int KB = K / 32;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        int b, k;
        for (b = 0; b < KB; ++b) {
            double amax = 0.0, inv;
            unsigned e;
            for (k = 0; k < 32; ++k) {
                double a = fabs(bf16_to_double(w[(size_t)n * K + b * 32 + k]));
                if (a > amax) amax = a;
            }
            e = mxr_e8m0_for_amax(amax, 6.0);
            scales[(size_t)n * KB + b] = (uint8_t)e;
            inv = ldexp(1.0, 127 - (int)e);
            for (k = 0; k < 32; k += 2) {
                size_t i = (size_t)n * K + b * 32 + k;
                unsigned lo = mxr_rne_e2m1(bf16_to_double(w[i]) * inv);
                unsigned hi = mxr_rne_e2m1(bf16_to_double(w[i + 1]) * inv);
                packed[i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* ---- the GEMM --------------------------------------------------------- */

static double dec_b(const uint8_t *b, int b_fmt, size_t row, int K, int k)
{
    if (b_fmt == B_E2M1_1X32) {
        uint8_t byte = b[row * (size_t)(K / 2) + (size_t)(k / 2)];
        return mxr_e2m1_value((k & 1) ? (byte >> 4) : (byte & 15u));
    }
    return mxr_e4m3_value(b[row * (size_t)K + (size_t)k]);
}

static double dec_a(const uint8_t *a, int a_fmt, size_t row, int K, int k)
{
    if (a_fmt == A_E2M1_1X32) {
        uint8_t byte = a[row * (size_t)(K / 2) + (size_t)(k / 2)];
        return mxr_e2m1_value((k & 1) ? (byte >> 4) : (byte & 15u));
    }
    return mxr_e4m3_value(a[row * (size_t)K + (size_t)k]);
}

/* Pre-activation accumulator and its |a||b| sum for one (m, n). */
static void dot_one(const uint8_t *a, const void *sa, int a_fmt,
                    const uint8_t *b, const void *sb, int b_fmt,
                    int m, int n, int K, double *acc_out, double *abs_out)
{
    const int KB = K / 32;
    double acc = 0.0, aabs = 0.0;
    int kb, k;
    if (a_fmt == A_F32_ROW) {
        const double s = (double)((const float *)sa)[m] * (double)((const float *)sb)[n];
        double blk = 0.0, blkabs = 0.0;
        for (k = 0; k < K; ++k) {
            double p = mxr_e4m3_value(a[(size_t)m * K + k]) * dec_b(b, b_fmt, (size_t)n, K, k);
            blk += p;
            blkabs += fabs(p);
        }
        acc = s * blk;
        aabs = fabs(s) * blkabs;
    } else {
        const uint8_t *sa8 = (const uint8_t *)sa, *sb8 = (const uint8_t *)sb;
        for (kb = 0; kb < KB; ++kb) {
            double blk = 0.0, blkabs = 0.0, s;
            unsigned eb = (b_fmt == B_E4M3_32X32) ? sb8[(size_t)(n / 32) * KB + kb]
                                                  : sb8[(size_t)n * KB + kb];
            s = mxr_e8m0_value(sa8[(size_t)m * KB + kb]) * mxr_e8m0_value(eb);
            for (k = kb * 32; k < kb * 32 + 32; ++k) {
                double p = dec_a(a, a_fmt, (size_t)m, K, k) * dec_b(b, b_fmt, (size_t)n, K, k);
                blk += p;
                blkabs += fabs(p);
            }
            acc += s * blk;
            aabs += s * blkabs;
        }
    }
    *acc_out = acc;
    *abs_out = aabs;
}

static double gelu_tanh(double v)
{
    const double c = sqrt(2.0 / M_PI); /* 0.7978845608... */
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* d/dv silu(v) = sigma(v) (1 + v (1 - sigma(v))), sigma(v) = 1 / (1 + e^-v):
 * the product rule on v * sigma(v) with sigma' = sigma (1 - sigma).  Used to
 * carry the gate's error term through the SwiGLU epilogue. */
static double silu_grad(double v)
{
    const double sig = 1.0 / (1.0 + exp(-v));
    return sig * (1.0 + v * (1.0 - sig));
}

/* y = epilogue(x . W^T) in fp64 for all m < M and output columns n < Nout
 * (Nout = N/2 for SwiGLU, else N).  y and tol are [M, Nout] row-major;
 * tol gets the T term (for SwiGLU the propagated
 * |silu'(g)| T_g |u| + |silu(g)| T_u); either may be NULL.  acc_out, if not
 * NULL, gets the raw pre-epilogue accumulators [M, N]. */
EXPORT void mxr_gemm(const uint8_t *a, const void *sa, int a_fmt,
                     const uint8_t *b, const void *sb, int b_fmt,
                     const float *bias, int epi, int M, int N, int K,
                     double *y, double *tol, double *acc_out)
{
    const int Nout = (epi == EPI_SWIGLU) ? N / 2 : N;
    long long i;
    if (acc_out) {
#pragma omp parallel for schedule(static)
        for (i = 0; i < (long long)M * N; ++i) {
            double acc, aabs;
            dot_one(a, sa, a_fmt, b, sb, b_fmt, (int)(i / N), (int)(i % N), K, &acc, &aabs);
            acc_out[i] = acc;
        }
    }
    /* every output element is independent and summed serially in fixed k
     * order, so the split of elements over threads does not change results */
#pragma omp parallel for schedule(static)
    for (i = 0; i < (long long)M * Nout; ++i) {
        const int m = (int)(i / Nout), n = (int)(i % Nout);
        double acc, aabs, out, t;
        dot_one(a, sa, a_fmt, b, sb, b_fmt, m, n, K, &acc, &aabs);
        if (epi == EPI_SWIGLU) {
            double g = acc + (bias ? (double)bias[n] : 0.0);
            double u_acc, u_abs, u, sg, dsg;
            dot_one(a, sa, a_fmt, b, sb, b_fmt, m, n + Nout, K, &u_acc, &u_abs);
            u = u_acc + (bias ? (double)bias[n + Nout] : 0.0);
            sg = silu(g);
            dsg = silu_grad(g);
            out = sg * u;
            /* first-order propagation of |d acc_g| <= T_g and |d acc_u| <= T_u
             * through y = silu(g) u */
            t = fabs(dsg) * aabs * fabs(u) + fabs(sg) * u_abs;
        } else {
            double v = acc;
            if (epi == EPI_BIAS || epi == EPI_BIAS_GELU_TANH)
                v += (double)bias[n];
            out = (epi == EPI_BIAS_GELU_TANH) ? gelu_tanh(v) : v;
            t = aabs;
        }
        if (y) y[i] = out;
        if (tol) tol[i] = t;
    }
}

/* Exposed for the epilogue pins. */
EXPORT double mxr_gelu_tanh(double v) { return gelu_tanh(v); }
EXPORT double mxr_silu(double v) { return silu(v); }
EXPORT double mxr_silu_grad(double v) { return silu_grad(v); }
