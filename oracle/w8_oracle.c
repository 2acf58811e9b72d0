/*
 * w8_oracle.c -- plain, slow, single-threaded CPU oracle for the 8-bit quantized
 * linear layer (dynamic activation quantizers, fused rms_norm / silu_and_mul
 * producers, and the scaled GEMM in FP8-dynamic, W8A8-INT8 and Block-FP8 form).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path loads this library.  Only
 * the test suite, the package's smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or constant generator with the CUDA
 * path; every constant below is written out here from the definition it names.
 *
 * Sources.  The pages that describe the method are:
 *   [FP8]  "PyTorch integra Helion en vLLM para acelerar inferencia FP8"
 *          (noticias.mechatronicstore.cl), sections "Patron de fusion del forward
 *          pass" and "Kernels Helion implementados";
 *   [LIN]  "Helion DSL added to vLLM to autotune linear inference backends"
 *          (signaltitans.com), section "Unified GEMM Architecture";
 *   [IT]   "Helion nel backend vLLM: un solo GEMM, tuning per forma e guadagni
 *          fino al 10%" (ai-radar.it), second and third paragraphs.
 * The pages name the operations (dynamic per-token fp8 quant, per-token-group fp8
 * quant, rms_norm + fp8 quant, silu_and_mul + fp8 quant, fused_qk_norm_rope, scaled_mm
 * for FP8 Dynamic / W8A8 INT8 / Block FP8, Split-K, Swap-AB) but print no formula.  Each function
 * below states the plain definition it implements; where the pages are silent the
 * comment says which reading is taken.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 * (-ffp-contract=off keeps every a*b+c below as two rounded operations unless the
 * code calls fmaf explicitly).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Number formats                                                             */
/* ------------------------------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32: widening is a 16-bit shift. */
float orc_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to the nearest bf16 (8 significant bits, binary32 exponent range),
 * ties to even, in ONE rounding (no detour through float, which would round twice).
 * Overflow goes to +-inf, as IEEE round-to-nearest does. */
uint16_t orc_bf16_from_double(double v)
{
    if (isnan(v)) return 0x7FC0;
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        /* spacing of bf16 values near a: 2^(e-7) in binade [2^e, 2^(e+1)),
         * 2^-133 below the smallest normal 2^-126 */
        double step = (a < ldexp(1.0, -126)) ? ldexp(1.0, -133) : ldexp(1.0, ilogb(a) - 7);
        r = nearbyint(a / step) * step;            /* default mode: ties to even */
        if (r >= ldexp(1.0, 128)) r = INFINITY;    /* past the largest finite bf16 */
    }
    float f = (float)r;                            /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    return neg ? (uint16_t)(b | 0x8000) : b;
}

/* e4m3 "fn" (OCP 8-bit floating point, E4M3): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; no infinities; 0x7F / 0xFF are NaN; the largest finite magnitude is
 * 1.75 * 2^8 = 448 (code 0x7E); subnormals are m * 2^-9 for m = 1..7. */
double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 0x7;
    if (e == 0xF && m == 0x7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    return s ? -mag : mag;
}

/* fp32 -> e4m3 with round-to-nearest-even and saturation to +-448 ("satfinite").
 * NaN -> 0x7F.  The sign of a result that rounds to zero is kept (0x80 = -0). */
uint8_t orc_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* grid spacing: 2^-9 among subnormals (a < 2^-6), 2^(e-3) in binade [2^e, 2^(e+1)) */
    double step = (a < ldexp(1.0, -6)) ? ldexp(1.0, -9) : ldexp(1.0, ilogb(a) - 3);
    double r = nearbyint(a / step) * step;         /* ties to even mantissa */
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6))                        /* subnormal: exponent field 0 */
        return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9)));
    int er = ilogb(r);                             /* r may have carried into the next binade */
    int mant = (int)(r / ldexp(1.0, er - 3)) - 8;  /* 0..7 */
    return (uint8_t)(sign | (uint8_t)(((er + 7) << 3) | mant));
}

/* fp32 -> symmetric int8: round to nearest, ties to even, clamp to [-127, 127]
 * (symmetric W8A8: -128 is never produced).  NaN -> 0. */
int8_t orc_int8_encode(float v)
{
    if (isnan(v)) return 0;
    double r = nearbyint((double)v);
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int8_t)r;
}

/* ------------------------------------------------------------------------- */
/* Scales                                                                     */
/* ------------------------------------------------------------------------- */

#define ORC_Q_FP8 0
#define ORC_Q_INT8 1

/* Dynamic scale from the largest magnitude: s = amax / Q (Q = 448 for e4m3, 127 for
 * int8), an IEEE fp32 division.  Reading for an all-zero group: s = 1 (any positive
 * scale decodes the zero codes to zero; the plain formula would give 0/0).
 * UE8M0 ("power-of-two") scales: s = 2^ceil(log2(amax/Q)), the smallest power of two
 * not below the fp32 quotient, so that no element saturates; the exponent is clamped
 * to the UE8M0 range [-127, 127]. */
float orc_scale(float amax, float qmax, int ue8m0)
{
    if (!(amax > 0.0f)) return 1.0f;
    float r = amax / qmax;
    if (!ue8m0) return r;
    int e;
    float f = frexpf(r, &e);                       /* r = f * 2^e, f in [0.5, 1) */
    int p = (f == 0.5f) ? e - 1 : e;               /* smallest 2^p >= r */
    if (p < -127) p = -127;
    if (p > 127) p = 127;
    return ldexpf(1.0f, p);
}

static void orc_encode_row(int qfmt, const float* v, int n, float s, uint8_t* q)
{
    for (int k = 0; k < n; ++k) {
        float t = v[k] / s;                        /* true division, not v * (1/s) */
        q[k] = (qfmt == ORC_Q_FP8) ? orc_e4m3_encode(t) : (uint8_t)orc_int8_encode(t);
    }
}

/* ------------------------------------------------------------------------- */
/* Activation quantizers                                                      */
/* ------------------------------------------------------------------------- */

/* Dynamic per-token quantization ([FP8] "Kernels Helion implementados":
 * dynamic_per_token_scaled_fp8_quant; the int8 form is the W8A8 INT8 activation side
 * of [LIN] "Unified GEMM Architecture") and per-token-group quantization
 * (per_token_group_fp8_quant, 1x128 groups along K, the activation side of Block FP8).
 *   group == 0: one scale per row m over all K columns -> scale[m]
 *   group >  0: one scale per (m, g) over columns [g*group, (g+1)*group)
 *               -> scale[m * (K/group) + g]; K must be a multiple of group.
 * x is bf16 bits, row stride ldx elements; q is row-major [M, K] (1 byte each). */
int orc_quant_rows(int qfmt, const uint16_t* x, int M, int K, int ldx,
                   uint8_t* q, float* scale, int group, int ue8m0)
{
    if (group < 0 || (group > 0 && K % group != 0)) return -1;
    int gsz = group ? group : K;
    int ng = K / gsz;
    float qmax = (qfmt == ORC_Q_FP8) ? 448.0f : 127.0f;
    float* v = (float*)malloc(sizeof(float) * (size_t)gsz);
    if (!v) return -2;
    for (int m = 0; m < M; ++m) {
        for (int g = 0; g < ng; ++g) {
            float amax = 0.0f;
            for (int k = 0; k < gsz; ++k) {
                v[k] = orc_bf16_to_float(x[(size_t)m * ldx + (size_t)g * gsz + k]);
                amax = fmaxf(amax, fabsf(v[k]));
            }
            float s = orc_scale(amax, qmax, ue8m0);
            scale[(size_t)m * ng + g] = s;
            orc_encode_row(qfmt, v, gsz, s, q + (size_t)m * K + (size_t)g * gsz);
        }
    }
    free(v);
    return 0;
}

/* Block-FP8 weight quantization: one scale per 128x128 block of W[N, K] (row-major,
 * K contiguous): scale[(n/128) * ceil(K/128) + k/128] = amax(block) / 448 (or its UE8M0
 * power of two).  Blocks at a ragged edge cover the rows/columns that exist. */
int orc_quant_weight_block(const uint16_t* w, int N, int K, uint8_t* q, float* scale, int ue8m0)
{
    int nbn = (N + 127) / 128, nbk = (K + 127) / 128;
    for (int bn = 0; bn < nbn; ++bn) {
        for (int bk = 0; bk < nbk; ++bk) {
            int n_end = (bn + 1) * 128 < N ? (bn + 1) * 128 : N;
            int k_end = (bk + 1) * 128 < K ? (bk + 1) * 128 : K;
            float amax = 0.0f;
            for (int n = bn * 128; n < n_end; ++n)
                for (int k = bk * 128; k < k_end; ++k)
                    amax = fmaxf(amax, fabsf(orc_bf16_to_float(w[(size_t)n * K + k])));
            float s = orc_scale(amax, 448.0f, ue8m0);
            scale[(size_t)bn * nbk + bk] = s;
            for (int n = bn * 128; n < n_end; ++n)
                for (int k = bk * 128; k < k_end; ++k)
                    q[(size_t)n * K + k] = orc_e4m3_encode(orc_bf16_to_float(w[(size_t)n * K + k]) / s);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Fused producers                                                            */
/* ------------------------------------------------------------------------- */

/* Sum of squares of n bf16 values, exactly, then rounded once to fp32 (round to
 * nearest, ties to even).  The pages fix no summation order, so the sum is taken as
 * the mathematical one: its fp32 rounding is then a function of the values alone.
 *
 * Each finite bf16 is q * 2^e with an integer q < 256 (8 significant bits) and
 * e >= -133, so each square is q^2 * 2^(2e), an integer q^2 < 2^16 times a power of two
 * no smaller than 2^-266.  The sum is accumulated as an exact integer count of units
 * of 2^-266 in a 576-bit number (18 words of 32 bits; the largest square of a finite
 * bf16 needs bit 506 and a sum of up to 2^31 of them at most 31 bits more), then
 * rounded to fp32 by inspecting its bits.  Any NaN input gives NaN, any infinity +inf. */
#define ORC_SQ_WORDS 18
float orc_sumsq_f32(const uint16_t* x, int n)
{
    uint32_t acc[ORC_SQ_WORDS];
    memset(acc, 0, sizeof acc);
    int has_nan = 0, has_inf = 0;
    for (int k = 0; k < n; ++k) {
        const unsigned E = (x[k] >> 7) & 0xFFu, m = x[k] & 0x7Fu;
        if (E == 0xFFu) {
            if (m) has_nan = 1; else has_inf = 1;
            continue;
        }
        const uint64_t q = (E == 0) ? m : (128u + m);         /* |x| = q * 2^e */
        const int e = (E == 0) ? -133 : (int)E - 134;
        const int shift = 2 * e + 266;                        /* x^2 = q^2 * 2^shift units */
        int w = shift / 32;
        uint64_t add = (q * q) << (shift % 32);               /* < 2^48: two words */
        while (add != 0 && w < ORC_SQ_WORDS) {
            const uint64_t t = (uint64_t)acc[w] + (add & 0xFFFFFFFFu);
            acc[w] = (uint32_t)t;
            add = (add >> 32) + (t >> 32);
            ++w;
        }
    }
    if (has_nan) return NAN;
    if (has_inf) return INFINITY;
    /* highest set bit p: the sum lies in [2^(p-266), 2^(p-265)) */
    int p = -1;
    for (int w = ORC_SQ_WORDS - 1; w >= 0 && p < 0; --w)
        for (int b = 31; b >= 0; --b)
            if ((acc[w] >> b) & 1u) { p = 32 * w + b; break; }
    if (p < 0) return 0.0f;
    /* fp32 keeps 24 bits from p down, and nothing below 2^-149 (bit 117 here) */
    int lsb = p - 23;
    if (lsb < 117) lsb = 117;
#define ORC_SQ_BIT(i) ((acc[(i) / 32] >> ((i) % 32)) & 1u)
    uint32_t mant = 0;
    for (int i = p; i >= lsb; --i) mant = (mant << 1) | ORC_SQ_BIT(i);
    const unsigned half = ORC_SQ_BIT(lsb - 1);
    unsigned sticky = 0;
    for (int i = lsb - 2; i >= 0 && !sticky; --i) sticky = ORC_SQ_BIT(i);
#undef ORC_SQ_BIT
    if (half && (sticky || (mant & 1u))) ++mant;             /* ties to even */
    return ldexpf((float)mant, lsb - 266);                   /* exact, or +inf past FLT_MAX */
}

/* RMS normalization in fp32 ([FP8] "Patron de fusion del forward pass":
 * post-attention rms_norm fused with the per-token fp8 quant):
 *   ss   = sum_k x_k^2, the exact sum rounded once to fp32 (orc_sumsq_f32);
 *   mean = ss / H;  r = 1 / sqrt(mean + eps)    (fp32, each step correctly rounded);
 *   y_k  = (x_k * r) * gamma_k                  (fp32, in this order).
 * y stays fp32 (the point of the fusion: no bf16 round trip before the quant). */
void orc_rmsnorm_f32(const uint16_t* x, const uint16_t* gamma, float eps,
                     int M, int H, int ldx, float* y)
{
    for (int m = 0; m < M; ++m) {
        const uint16_t* xr = x + (size_t)m * ldx;
        float ss = orc_sumsq_f32(xr, H);
        float mean = ss / (float)H;
        float r = 1.0f / sqrtf(mean + eps);
        for (int k = 0; k < H; ++k)
            y[(size_t)m * H + k] = (orc_bf16_to_float(xr[k]) * r) * orc_bf16_to_float(gamma[k]);
    }
}

/* rms_norm followed by dynamic per-token fp8 quant of the fp32 result. */
int orc_rmsnorm_quant(const uint16_t* x, const uint16_t* gamma, float eps,
                      int M, int H, int ldx, uint8_t* q, float* scale)
{
    float* y = (float*)malloc(sizeof(float) * (size_t)M * H);
    if (!y) return -2;
    orc_rmsnorm_f32(x, gamma, eps, M, H, ldx, y);
    for (int m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int k = 0; k < H; ++k) amax = fmaxf(amax, fabsf(y[(size_t)m * H + k]));
        float s = orc_scale(amax, 448.0f, 0);
        scale[m] = s;
        orc_encode_row(ORC_Q_FP8, y + (size_t)m * H, H, s, q + (size_t)m * H);
    }
    free(y);
    return 0;
}

/* fp8 quantization of fp32 rows v[M, K] (row-major): one scale per row (group == 0) or
 * per 1x`group` block of a row (scale[m * (K/group) + g]), fp32 or UE8M0 scales. */
static int orc_quant_f32_rows(const float* v, int M, int K, int group, int ue8m0, uint8_t* q, float* scale)
{
    if (group < 0 || (group > 0 && K % group != 0)) return -1;
    int gsz = group ? group : K;
    int ng = K / gsz;
    for (int m = 0; m < M; ++m) {
        for (int g = 0; g < ng; ++g) {
            const float* row = v + (size_t)m * K + (size_t)g * gsz;
            float amax = 0.0f;
            for (int k = 0; k < gsz; ++k) amax = fmaxf(amax, fabsf(row[k]));
            float s = orc_scale(amax, 448.0f, ue8m0);
            scale[(size_t)m * ng + g] = s;
            orc_encode_row(ORC_Q_FP8, row, gsz, s, q + (size_t)m * K + (size_t)g * gsz);
        }
    }
    return 0;
}

/* rms_norm followed by 1x`group` fp8 quantization of the fp32 result ([FP8] "Kernels
 * Helion implementados": rms_norm_per_block_quant; the Block-FP8 activation side). */
int orc_rmsnorm_quant_group(const uint16_t* x, const uint16_t* gamma, float eps, int M, int H, int ldx,
                            int group, int ue8m0, uint8_t* q, float* scale)
{
    float* y = (float*)malloc(sizeof(float) * (size_t)M * H);
    if (!y) return -2;
    orc_rmsnorm_f32(x, gamma, eps, M, H, ldx, y);
    int rc = orc_quant_f32_rows(y, M, H, group, ue8m0, q, scale);
    free(y);
    return rc;
}

/* exp(x) in fp32, written for this project so that the CPU and GPU sides can agree to
 * the bit (neither may call a vendor exp).  Method: Cody & Waite argument reduction
 * (W. J. Cody, W. Waite, "Software Manual for the Elementary Functions", 1980):
 *   n = rint(x * log2(e)),  r = (x - n*ln2_hi) - n*ln2_lo  with |r| <~ ln2/2,
 * then exp(r) by its Taylor series to degree 7 in Horner form (truncation error
 * below r^8/8! ~ 5e-9 relative), then the exact scaling by 2^n, done as two
 * multiplications by powers of two so each factor stays a normal number.
 * Every multiply-add in the reduction and the polynomial is an explicit fmaf. */
float orc_exp_f32(float x)
{
    if (isnan(x)) return x;
    if (x > 100.0f) return INFINITY;   /* e^100 > FLT_MAX */
    if (x < -150.0f) return 0.0f;      /* e^-150 < half the smallest subnormal */
    const float log2e  = 0x1.715476p+0f;   /* log2(e) rounded to fp32 */
    const float ln2_hi = 0x1.62e400p-1f;   /* 0.693145751953125: leading bits of ln 2 */
    const float ln2_lo = 0x1.7f7d1cp-20f;  /* ln 2 - ln2_hi, rounded to fp32 */
    float n = nearbyintf(x * log2e);
    float r = fmaf(-n, ln2_hi, x);
    r = fmaf(-n, ln2_lo, r);
    /* 1/k! for k = 7..2, each rounded to fp32 */
    float p = 0x1.a01a02p-13f;             /* 1/5040 */
    p = fmaf(p, r, 0x1.6c16c2p-10f);       /* 1/720 */
    p = fmaf(p, r, 0x1.111112p-7f);        /* 1/120 */
    p = fmaf(p, r, 0x1.555556p-5f);        /* 1/24 */
    p = fmaf(p, r, 0x1.555556p-3f);        /* 1/6 */
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;                       /* in [-217, 145] given the range checks */
    int n1 = ni / 2, n2 = ni - n1;         /* each in [-109, 73]: 2^n1, 2^n2 are normal */
    return (p * ldexpf(1.0f, n1)) * ldexpf(1.0f, n2);
}

/* silu_and_mul in fp32 ([FP8] "Kernels Helion implementados":
 * silu_and_mul_dynamic_per_token_quant).  Input row m of X[M, 2I] holds the gate in
 * columns [0, I) and the up projection in [I, 2I) (reading: the pages do not fix the
 * order; gate-first is the common layout of a merged gate_up projection).
 *   h = (g / (1 + exp(-g))) * u, every step an fp32 operation in this order. */
void orc_silu_mul_f32(const uint16_t* xgu, int M, int I, int ld, float* h)
{
    for (int m = 0; m < M; ++m) {
        const uint16_t* row = xgu + (size_t)m * ld;
        for (int k = 0; k < I; ++k) {
            float g = orc_bf16_to_float(row[k]);
            float u = orc_bf16_to_float(row[I + k]);
            float den = 1.0f + orc_exp_f32(-g);
            float sg = g / den;
            h[(size_t)m * I + k] = sg * u;
        }
    }
}

/* silu_and_mul followed by 1x`group` fp8 quantization of the fp32 result ([FP8]
 * "Kernels Helion implementados": silu_and_mul_per_block_quant). */
int orc_silu_mul_quant_group(const uint16_t* xgu, int M, int I, int ld, int group, int ue8m0, uint8_t* q,
                             float* scale)
{
    float* h = (float*)malloc(sizeof(float) * (size_t)M * I);
    if (!h) return -2;
    orc_silu_mul_f32(xgu, M, I, ld, h);
    int rc = orc_quant_f32_rows(h, M, I, group, ue8m0, q, scale);
    free(h);
    return rc;
}

/* silu_and_mul followed by dynamic per-token fp8 quant of the fp32 result. */
int orc_silu_mul_quant(const uint16_t* xgu, int M, int I, int ld, uint8_t* q, float* scale)
{
    float* h = (float*)malloc(sizeof(float) * (size_t)M * I);
    if (!h) return -2;
    orc_silu_mul_f32(xgu, M, I, ld, h);
    for (int m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int k = 0; k < I; ++k) amax = fmaxf(amax, fabsf(h[(size_t)m * I + k]));
        float s = orc_scale(amax, 448.0f, 0);
        scale[m] = s;
        orc_encode_row(ORC_Q_FP8, h + (size_t)m * I, I, s, q + (size_t)m * I);
    }
    free(h);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Scaled GEMM                                                                */
/* ------------------------------------------------------------------------- */

#define ORC_FMT_FP8_DYN 0
#define ORC_FMT_INT8 1
#define ORC_FMT_BLOCK_FP8 2

/* Decoded value of one stored 8-bit operand. */
static double orc_operand(int fmt, uint8_t c)
{
    return (fmt == ORC_FMT_INT8) ? (double)(int8_t)c : orc_e4m3_decode(c);
}

/* Scaled 8-bit GEMM, naive triple loop ([LIN] "Unified GEMM Architecture": FP8
 * Dynamic, W8A8 INT8 and Block FP8 formats; [FP8] "Kernels Helion implementados":
 * scaled_mm and scaled_mm_blockwise).  A is Aq[M, K], W is Wq[N, K] (both K contiguous),
 * out[m, n] for n in [n_lo, n_hi) is written to out[m * (n_hi - n_lo) + (n - n_lo)].
 *   FP8_DYN : ref = (sum_k a*w) * sA[m] * sW[n]
 *   INT8    : acc = sum_k a*w as an exact integer; ref = acc * sA[m] * sW[n]
 *   BLOCK   : ref = sum_kb sA[m, kb] * sW[n/128, kb] * (sum_{k in kb} a*w), with
 *             sA[M, ceil(K/128)] and sW[ceil(N/128), ceil(K/128)] row-major.
 * Sums of products of decoded e4m3 (or int8) values are exact in fp64 at these sizes.
 * out_bf16 = ref rounded once to bf16; ref_f64 (optional) = ref; acc_i64 (optional,
 * INT8 only) = the integer dot products. */
void orc_gemm(int fmt, const uint8_t* Aq, const float* sA, const uint8_t* Wq, const float* sW,
              int M, int N, int K, int n_lo, int n_hi,
              uint16_t* out_bf16, double* ref_f64, int64_t* acc_i64)
{
    (void)N;
    int w = n_hi - n_lo;
    int nbk = (K + 127) / 128;
    for (int m = 0; m < M; ++m) {
        for (int n = n_lo; n < n_hi; ++n) {
            const uint8_t* a = Aq + (size_t)m * K;
            const uint8_t* b = Wq + (size_t)n * K;
            double ref;
            if (fmt == ORC_FMT_BLOCK_FP8) {
                ref = 0.0;
                for (int kb = 0; kb < nbk; ++kb) {
                    double part = 0.0;
                    int k_end = (kb + 1) * 128 < K ? (kb + 1) * 128 : K;
                    for (int k = kb * 128; k < k_end; ++k)
                        part += orc_e4m3_decode(a[k]) * orc_e4m3_decode(b[k]);
                    ref += (double)sA[(size_t)m * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + kb] * part;
                }
            } else if (fmt == ORC_FMT_INT8) {
                int64_t acc = 0;
                for (int k = 0; k < K; ++k) acc += (int64_t)(int8_t)a[k] * (int64_t)(int8_t)b[k];
                if (acc_i64) acc_i64[(size_t)m * w + (n - n_lo)] = acc;
                ref = (double)acc * (double)sA[m] * (double)sW[n];
            } else {
                double acc = 0.0;
                for (int k = 0; k < K; ++k) acc += orc_e4m3_decode(a[k]) * orc_e4m3_decode(b[k]);
                ref = acc * (double)sA[m] * (double)sW[n];
            }
            if (ref_f64) ref_f64[(size_t)m * w + (n - n_lo)] = ref;
            if (out_bf16) out_bf16[(size_t)m * w + (n - n_lo)] = orc_bf16_from_double(ref);
        }
    }
}

/* Unscaled dot products for a list of (m, n) pairs: dot[i] = sum_k a[m_i, k] * w[n_i, k]
 * (for spot checks of large problems one output at a time). */
void orc_gemm_points(int fmt, const uint8_t* Aq, const float* sA, const uint8_t* Wq, const float* sW,
                     int M, int N, int K, int npts, const int* pm, const int* pn, double* ref_f64)
{
    (void)M; (void)N;
    int nbk = (K + 127) / 128;
    for (int i = 0; i < npts; ++i) {
        int m = pm[i], n = pn[i];
        const uint8_t* a = Aq + (size_t)m * K;
        const uint8_t* b = Wq + (size_t)n * K;
        double ref = 0.0;
        if (fmt == ORC_FMT_BLOCK_FP8) {
            for (int kb = 0; kb < nbk; ++kb) {
                double part = 0.0;
                int k_end = (kb + 1) * 128 < K ? (kb + 1) * 128 : K;
                for (int k = kb * 128; k < k_end; ++k)
                    part += orc_e4m3_decode(a[k]) * orc_e4m3_decode(b[k]);
                ref += (double)sA[(size_t)m * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + kb] * part;
            }
        } else {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += orc_operand(fmt, a[k]) * orc_operand(fmt, b[k]);
            ref = acc * (double)sA[m] * (double)sW[n];
        }
        ref_f64[i] = ref;
    }
}

/* Swap-AB formulation ([IT], second paragraph: A@B rewritten as (B^T @ A^T)^T): the
 * transposed product outT[n, m] = sum_k W[n, k] * A[m, k] is formed with W as the left
 * operand (loop over weight rows outermost), scaled, and transposed on the way out.
 * Unscaled-then-scaled exactly as orc_gemm; written as its own loop nest so that the
 * identity can be checked.  ref_f64 is [M, N]. */
void orc_gemm_swap_ab(int fmt, const uint8_t* Aq, const float* sA, const uint8_t* Wq, const float* sW,
                      int M, int N, int K, double* ref_f64)
{
    int nbk = (K + 127) / 128;
    double* outT = (double*)malloc(sizeof(double) * (size_t)N * M);
    if (!outT) return;
    for (int n = 0; n < N; ++n) {              /* rows of the left operand W */
        for (int m = 0; m < M; ++m) {          /* columns: rows of A */
            double v = 0.0;
            if (fmt == ORC_FMT_BLOCK_FP8) {
                for (int kb = 0; kb < nbk; ++kb) {
                    double part = 0.0;
                    int k_end = (kb + 1) * 128 < K ? (kb + 1) * 128 : K;
                    for (int k = kb * 128; k < k_end; ++k)
                        part += orc_e4m3_decode(Wq[(size_t)n * K + k]) * orc_e4m3_decode(Aq[(size_t)m * K + k]);
                    v += (double)sA[(size_t)m * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + kb] * part;
                }
            } else {
                for (int k = 0; k < K; ++k)
                    v += orc_operand(fmt, Wq[(size_t)n * K + k]) * orc_operand(fmt, Aq[(size_t)m * K + k]);
                v = v * (double)sA[m] * (double)sW[n];   /* same scale order as the plain form */
            }
            outT[(size_t)n * M + m] = v;
        }
    }
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) ref_f64[(size_t)m * N + n] = outT[(size_t)n * M + m];
    free(outT);
}

/* Split-K formulation ([IT], second and third paragraphs: K divided among thread
 * blocks, split_k a power of two up to 256): the K range is cut into S contiguous
 * chunks of ceil(K/S) columns (the last may be shorter or empty), each chunk's partial
 * sum is formed on its own, and the partials are added in chunk order before scaling.
 * For Block FP8 the chunk boundaries fall on 128-column blocks (S <= number of blocks)
 * and each partial already carries its block scales.  ref_f64 is [M, N]. */
int orc_gemm_split_k(int fmt, const uint8_t* Aq, const float* sA, const uint8_t* Wq, const float* sW,
                     int M, int N, int K, int S, double* ref_f64)
{
    if (S < 1) return -1;
    int nbk = (K + 127) / 128;
    int blockwise = (fmt == ORC_FMT_BLOCK_FP8);
    int units = blockwise ? nbk : K;               /* what a chunk is made of */
    if (S > units) return -1;
    int per = (units + S - 1) / S;
    double* part = (double*)malloc(sizeof(double) * (size_t)S);
    if (!part) return -2;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            for (int s = 0; s < S; ++s) {
                int u0 = s * per, u1 = (s + 1) * per < units ? (s + 1) * per : units;
                double p = 0.0;
                for (int u = u0; u < u1; ++u) {
                    if (blockwise) {
                        double blk = 0.0;
                        int k_end = (u + 1) * 128 < K ? (u + 1) * 128 : K;
                        for (int k = u * 128; k < k_end; ++k)
                            blk += orc_e4m3_decode(Aq[(size_t)m * K + k]) * orc_e4m3_decode(Wq[(size_t)n * K + k]);
                        p += (double)sA[(size_t)m * nbk + u] * (double)sW[(size_t)(n / 128) * nbk + u] * blk;
                    } else {
                        p += orc_operand(fmt, Aq[(size_t)m * K + u]) * orc_operand(fmt, Wq[(size_t)n * K + u]);
                    }
                }
                part[s] = p;
            }
            double v = 0.0;
            for (int s = 0; s < S; ++s) v += part[s];
            if (!blockwise) v = v * (double)sA[m] * (double)sW[n];
            ref_f64[(size_t)m * N + n] = v;
        }
    }
    free(part);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* fused_qk_norm_rope                                                         */

/* Per-head rms_norm of the query and key heads, then rotary position embedding ([FP8]
 * "Kernels Helion implementados": fused_qk_norm_rope -- named there, no formula).
 * Reading, for the merged projection qkv[T, (Hq + 2*Hkv) * D] (bf16, row-major: the Hq
 * query heads, then the Hkv key heads, then the Hkv value heads, D values each):
 *   for every token t and every query or key head (x = that head's D values):
 *     y = rms_norm of x with the head-dimension weight (q_weight for query heads,
 *         k_weight for key heads): the exact sum of squares rounded once to fp32, then
 *         mean = ss / D, r = 1 / sqrt(mean + eps), y_k = (x_k * r) * w_k in fp32;
 *     with p = positions[t], c_i = cos_sin[p * D + i] and s_i = cos_sin[p * D + D/2 + i]
 *     (i < D/2), each pair (y_i, y_{i+D/2}) is rotated by the angle whose cosine and
 *     sine these are (the rotate-halves pairing):
 *       o_i       = y_i * c_i - y_{i+D/2} * s_i
 *       o_{i+D/2} = y_{i+D/2} * c_i + y_i * s_i      (fp32: two products, then the sum)
 *     and each o is rounded once to bf16;
 *   the value heads are copied unchanged.
 * The cos / sin table (fp32 [max_pos, D]) is an input: the caller computes it once from
 * the rotary base, so nothing here evaluates a transcendental function.
 * Returns 0, or -1 for a bad size or a position outside [0, max_pos). */
int orc_qk_norm_rope(const uint16_t* qkv, uint16_t* out, int T, int Hq, int Hkv, int D, const uint16_t* q_weight,
                     const uint16_t* k_weight, const float* cos_sin, int max_pos, const int64_t* positions, float eps)
{
    if (T < 0 || Hq < 0 || Hkv < 0 || D <= 0 || D % 2 != 0) return -1;
    const int H = Hq + 2 * Hkv;
    const int half = D / 2;
    float* y = (float*)malloc(sizeof(float) * (size_t)D);
    if (!y) return -2;
    for (int t = 0; t < T; ++t) {
        const int64_t p = positions[t];
        if (p < 0 || p >= max_pos) { free(y); return -1; }
        const float* cs = cos_sin + (size_t)p * D;
        for (int h = 0; h < H; ++h) {
            const uint16_t* x = qkv + ((size_t)t * H + h) * D;
            uint16_t* o = out + ((size_t)t * H + h) * D;
            if (h >= Hq + Hkv) {
                for (int k = 0; k < D; ++k) o[k] = x[k];
                continue;
            }
            const uint16_t* w = (h < Hq) ? q_weight : k_weight;
            float ss = orc_sumsq_f32(x, D);
            float mean = ss / (float)D;
            float r = 1.0f / sqrtf(mean + eps);
            for (int k = 0; k < D; ++k) y[k] = (orc_bf16_to_float(x[k]) * r) * orc_bf16_to_float(w[k]);
            for (int i = 0; i < half; ++i) {
                const float c = cs[i], sn = cs[half + i];
                const float lo = y[i] * c - y[half + i] * sn;
                const float hi = y[half + i] * c + y[i] * sn;
                o[i] = orc_bf16_from_double((double)lo);
                o[half + i] = orc_bf16_from_double((double)hi);
            }
        }
    }
    free(y);
    return 0;
}
