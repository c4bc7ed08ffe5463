/*
 * w4ref.c -- CPU oracle for per-group INT4 round-to-nearest weight quantization
 * and the W4A16 linear layer.  TEST INFRASTRUCTURE ONLY: only the test suite,
 * the smoke check and the CPU-baseline leg of the benchmark may load it.  It
 * shares no code, header, table or helper with the CUDA library and it is
 * never part of the product path.
 *
 * Plain, slow, scalar C.  Every step follows the method as the source pages
 * state it, in their order:
 *
 *   [LQ]  "LLM quantization methods: principles and implementation"
 *         (zhiyuanblog.org/blog/llm-quantization)
 *         §2.2 integer quantization maths: symmetric  s = max|x| / (2^(b-1)-1),
 *              x_q = clamp(round(x/s), -qmax, qmax), x ~ x_q * s;
 *              asymmetric s = (max-min)/(2^b-1), zero_point = clamp(round(-min/s), 0, 2^b-1),
 *              x_q = clamp(round(x/s + zero_point), 0, 2^b-1), x ~ (x_q - zero_point) * s.
 *         §2.3 per-group granularity: W is (out_features, in_features), the in
 *              dimension is cut into groups of g (e.g. 128) with one scale each,
 *              and in_features must be a multiple of g.
 *         §4.2 AWQ: W is multiplied column-wise by a per-input-channel factor s
 *              before the per-group quantizer runs; s = (a/w)^alpha from the
 *              mean magnitudes of activations and weights, alpha grid-searched
 *              to minimise the layer's output error.
 *         §4.3 SmoothQuant: s = max|X_j|^a / max|W_j|^(1-a), W*s and X/s both
 *              quantized to INT8 per tensor (W8A8).
 *         §4.6 FP8 E4M3: scale = max|x| / 448, cast.
 *   [PTQ] "PTQ weight quantization: from GPTQ to AWQ" (jonathanding.github.io),
 *         section "Round-to-Nearest": every weight is rounded on its own to the
 *         nearest level; section "AWQ": XW = (X diag(s)^-1)(diag(s) W).
 *   [MF]  "Quantization method families" (inference-learning-path.pages.dev),
 *         §2 mental model: W4A16 keeps activations in 16-bit floats and
 *         dequantizes the weights before the matmul.
 *
 * Readings where the pages leave a step open (each one is also listed in the
 * design notes of the repository):
 *   - all scale / zero-point / division arithmetic is IEEE fp32 with
 *     round-to-nearest-even; "round" is round-half-to-even (torch.round);
 *   - the asymmetric path uses the code form of §2.2 (integer zero point),
 *     rounding after the fp32 add: u = rne(fl(fl(w/s) + zp));
 *   - symmetric codes q in [-7, 7] are stored as u = q + 8 with zero = 8.0f,
 *     so both forms dequantize as (u - zero) * scale;
 *   - a group whose scale comes out 0 (all-zero symmetric group, constant
 *     asymmetric group) stores scale 0, zero 8 (sym) or 0 (asym) and u = zero,
 *     so it dequantizes to 0;
 *   - nibble layout (ours; the pages give only "0.5 byte per parameter"):
 *     packed is [N][K/2] bytes; the 8 codes of k = 8j..8j+7 of a row form the
 *     little-endian 32-bit word j, whose nibble i (bits 4i..4i+3) holds
 *     k = 8j + SIGMA[i] with SIGMA = {0,2,4,6,1,3,5,7};
 *   - scales and zeros are fp32 [N][K/group].
 *
 * Compiled with -O2 -ffp-contract=off -fno-fast-math so that every float
 * operation below is one correctly rounded IEEE binary32 operation.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define W4REF_OK 0
#define W4REF_EINVAL 1
#define W4REF_ENONFINITE 5

#define DT_F16 0
#define DT_BF16 1

/* Position of k-within-word for nibble i of a packed 32-bit word. */
static const int SIGMA[8] = {0, 2, 4, 6, 1, 3, 5, 7};

/* ---- 16-bit float decoding, from the IEEE 754 binary16 and bfloat16 definitions ---- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double w4ref_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double w4ref_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double decode16(uint16_t h, int dtype)
{
    return dtype == DT_BF16 ? w4ref_bf16_to_f64(h) : w4ref_f16_to_f64(h);
}

/* Round-to-nearest, ties to even (torch.round), in the current FE_TONEAREST mode. */
static float rne(float x) { return nearbyintf(x); }

static float clampf(float v, float lo, float hi)
{
    if (v < lo) return lo;
    if (v > hi) return hi;
    return v;
}

/* ---- quantize ------------------------------------------------------------------ */

/*
 * Quantize W [N][K] (fp16 or bf16 bit patterns, row-major, out x in) group by
 * group along K.  col_scale (nullable, [K] fp32) is the AWQ per-input-channel
 * factor folded in first: w = fl32(w * col_scale[k]).
 * Outputs: packed [N][K/2], scales [N][K/group], zeros [N][K/group].
 * group must divide K, be a multiple of 8 and be at most 4096.
 * Returns W4REF_EINVAL on a bad shape, W4REF_ENONFINITE if a folded weight,
 * a group range or a scale is not finite (that group's outputs are not written).
 */
int w4ref_quantize(const uint16_t *W, int dtype, long K, long N, long group, int sym,
                   const float *col_scale, uint8_t *packed, float *scales, float *zeros)
{
    if (K <= 0 || N <= 0 || group <= 0 || group > 4096 || group % 8 != 0 || K % group != 0)
        return W4REF_EINVAL;
    if (dtype != DT_F16 && dtype != DT_BF16) return W4REF_EINVAL;
    fesetround(FE_TONEAREST);
    const long G = K / group;
    int status = W4REF_OK;

#pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        float w[4096];
        uint8_t u[4096];
        for (long g = 0; g < G; ++g) {
            const long k0 = g * group;
            /* step 1: load, optional AWQ fold (one fp32 multiply) */
            int bad = 0;
            for (long i = 0; i < group; ++i) {
                float v = (float)decode16(W[n * K + k0 + i], dtype);
                if (col_scale) v = v * col_scale[k0 + i];
                if (!isfinite(v)) bad = 1;
                w[i] = v;
            }
            float s, z;
            if (sym) {
                /* step 2: amax = max |w|; step 3: s = amax / qmax, qmax = 2^(4-1)-1 = 7 */
                float amax = 0.0f;
                for (long i = 0; i < group; ++i) {
                    float a = fabsf(w[i]);
                    if (a > amax) amax = a;
                }
                s = amax / 7.0f;
                z = 8.0f;
                if (!isfinite(s)) bad = 1;
                if (!bad) {
                    for (long i = 0; i < group; ++i) {
                        if (s == 0.0f) { u[i] = 8; continue; }
                        /* step 4: q = clamp(round(w / s), -7, 7); stored as q + 8 */
                        float q = clampf(rne(w[i] / s), -7.0f, 7.0f);
                        u[i] = (uint8_t)((int)q + 8);
                    }
                }
            } else {
                /* step 2: min and max of the group; step 3: s = (max - min) / (2^4 - 1) */
                float mn = w[0], mx = w[0];
                for (long i = 1; i < group; ++i) {
                    if (w[i] < mn) mn = w[i];
                    if (w[i] > mx) mx = w[i];
                }
                float range = mx - mn;
                s = range / 15.0f;
                if (!isfinite(range) || !isfinite(s)) bad = 1;
                if (!bad) {
                    if (s == 0.0f) {
                        z = 0.0f;
                        for (long i = 0; i < group; ++i) u[i] = 0;
                    } else {
                        /* zero_point = clamp(round(-min / s), 0, 15) */
                        float negmn = -mn;
                        z = clampf(rne(negmn / s), 0.0f, 15.0f);
                        /* the zero point is an integer in [0, 15]; store 0 as +0.0 */
                        z = z + 0.0f;
                        for (long i = 0; i < group; ++i) {
                            /* step 4: u = clamp(round(w / s + zero_point), 0, 15) */
                            float t = w[i] / s;
                            float y = t + z;
                            float q = clampf(rne(y), 0.0f, 15.0f);
                            u[i] = (uint8_t)(int)q;
                        }
                    }
                } else {
                    z = 0.0f;
                }
            }
            if (bad) {
#pragma omp atomic write
                status = W4REF_ENONFINITE;
                continue;
            }
            scales[n * G + g] = s;
            zeros[n * G + g] = z;
            /* step 5: pack 8 codes per 32-bit little-endian word */
            for (long j = 0; j < group / 8; ++j) {
                uint32_t word = 0;
                for (int i = 0; i < 8; ++i) word |= (uint32_t)(u[j * 8 + SIGMA[i]] & 0xF) << (4 * i);
                uint8_t *dst = packed + n * (K / 2) + (k0 + j * 8) / 2;
                for (int b = 0; b < 4; ++b) dst[b] = (uint8_t)(word >> (8 * b));
            }
        }
    }
    return status;
}

/* ---- unpack / dequantize ----------------------------------------------------------- */

/* Code u of (n, k) from packed [N][K/2]: the inverse of the packing above. */
int w4ref_code(const uint8_t *packed, long K, long n, long k)
{
    long j = k / 8, r = k % 8;
    const uint8_t *src = packed + n * (K / 2) + j * 4;
    uint32_t word = (uint32_t)src[0] | ((uint32_t)src[1] << 8) | ((uint32_t)src[2] << 16) |
                    ((uint32_t)src[3] << 24);
    for (int i = 0; i < 8; ++i)
        if (SIGMA[i] == r) return (int)((word >> (4 * i)) & 0xF);
    return -1;
}

/*
 * What [N][K] (fp64) = (u - zero) * scale, computed exactly in fp64.
 * zeros == NULL means the symmetric storage (zero = 8).
 */
int w4ref_dequant(const uint8_t *packed, const float *scales, const float *zeros, long K,
                  long N, long group, double *What)
{
    if (K <= 0 || N <= 0 || group <= 0 || K % group != 0 || K % 8 != 0) return W4REF_EINVAL;
    const long G = K / group;
#pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n)
        for (long k = 0; k < K; ++k) {
            double s = (double)scales[n * G + k / group];
            double z = zeros ? (double)zeros[n * G + k / group] : 8.0;
            What[n * K + k] = ((double)w4ref_code(packed, K, n, k) - z) * s;
        }
    return W4REF_OK;
}

/* ---- the W4A16 linear layer ------------------------------------------------------------ */

/*
 * Y[m][n] = sum_k X[m][k] * What[n][k], naive fp64 loop in k order.
 * X [M][K] holds fp16/bf16 bit patterns.  rows (nullable) selects the m to
 * compute; Y is then [nrows][N] in the order of rows.
 */
int w4ref_linear(const uint16_t *X, int dtype, long M, long K, const double *What, long N,
                 const long *rows, long nrows, double *Y)
{
    if (M <= 0 || K <= 0 || N <= 0) return W4REF_EINVAL;
    if (!rows) nrows = M;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < nrows; ++r) {
        long m = rows ? rows[r] : r;
        if (m < 0 || m >= M) continue;
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += decode16(X[m * K + k], dtype) * What[n * K + k];
            Y[r * N + n] = acc;
        }
    }
    return W4REF_OK;
}

/*
 * Same product straight from the packed weights, for one (m, n) pair at a
 * time: used where the full fp64 W-hat would not fit (sampled checks).
 */
double w4ref_linear_at(const uint16_t *X, int dtype, long K, const uint8_t *packed,
                       const float *scales, const float *zeros, long group, long m, long n)
{
    const long G = K / group;
    double acc = 0.0;
    for (long k = 0; k < K; ++k) {
        double s = (double)scales[n * G + k / group];
        double z = zeros ? (double)zeros[n * G + k / group] : 8.0;
        double w = ((double)w4ref_code(packed, K, n, k) - z) * s;
        acc += decode16(X[m * K + k], dtype) * w;
    }
    return acc;
}

/* Number of OpenMP threads the parallel loops above use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int w4ref_threads(void) { return omp_get_max_threads(); }
void w4ref_set_threads(int n) { omp_set_num_threads(n); }
#else
int w4ref_threads(void) { return 1; }
void w4ref_set_threads(int n) { (void)n; }
#endif

/* ---- AWQ per-input-channel scale search ------------------------------------------------ */

/*
 * Nearest binary16 (dtype F16) or bfloat16 (dtype BF16) value to v, ties to
 * even, returned as a double; from the formats' definitions: p significant
 * bits (11 / 8), smallest normal exponent emin (-14 / -126), below which the
 * spacing stays 2^(emin - p + 1) (subnormals), and largest finite value
 * (65504 / (2 - 2^-7) * 2^127).  A magnitude that rounds above it is +-inf.
 */
double w4ref_round16(double v, int dtype)
{
    if (v == 0.0 || isnan(v) || isinf(v)) return v;
    const int p = dtype == DT_BF16 ? 8 : 11;
    const int emin = dtype == DT_BF16 ? -126 : -14;
    const double maxv = dtype == DT_BF16 ? ldexp(255.0, 120) : 65504.0;
    int e;
    frexp(v, &e); /* |v| = f * 2^e with f in [0.5, 1): the leading bit is worth 2^(e-1) */
    int lead = e - 1;
    if (lead < emin) lead = emin;
    const int q = lead - (p - 1); /* exponent of one unit in the last place */
    const double r = ldexp(nearbyint(ldexp(v, -q)), q);
    if (fabs(r) > maxv) return copysign(INFINITY, v);
    return r;
}

/*
 * AWQ scale search for one linear layer.
 *   [LQ] §4.2: find the per-input-channel factor s that minimises
 *        || Q(W * s) (X / s) - W X ||; its code form takes, per input
 *        channel j, the activation importance a_j = mean_i |X_ij| and the
 *        weight magnitude w_j = mean_n |W_nj|, forms s_j = (a_j / w_j)^alpha,
 *        scales the columns of W by s before the per-group quantizer, and at
 *        inference divides the activations by s; alpha in [0, 1] is picked by
 *        a grid search.
 *   [PTQ] section "AWQ": the same identity XW = (X diag(s)^-1)(diag(s) W).
 *
 * Inputs: W [N][K] and the calibration activations X [Mc][K], both 16-bit
 * bit patterns of `dtype`; alphas [n_alpha].
 * Outputs: err [n_alpha]; s_all (nullable) [n_alpha][K] fp32; *best.
 *
 * Readings where the pages leave a step open:
 *   - a_j and w_j are fp64 sums in index order, divided by the count in
 *     fp64 and rounded once to fp32;
 *   - s_j = fl32(pow(a_j / w_j, alpha)) with the ratio and pow in fp64, and
 *     s_j = 1 for a channel whose a_j or w_j is 0 (no evidence either way);
 *   - Q is the per-group RTN quantizer above with col_scale = s (the fold is
 *     one fp32 multiply per weight);
 *   - the scaled activations are those the W4A16 layer would be fed:
 *     fl16(fl32(x) / s_j), an fp32 division rounded once to `dtype`;
 *   - the quantized layer's output is that of the W4A16 layer: the exact
 *     product rounded once to `dtype`; the reference W X is the exact fp64
 *     product of the unquantized 16-bit operands;
 *   - the norm is the Frobenius norm, and err holds its square
 *     sum_{i,n} (Yq - Yref)^2 (same argmin);
 *   - best is the first index of the smallest err; a NaN err is never best,
 *     and *best = -1 when every err is NaN.
 * Returns W4REF_EINVAL on a bad shape, or the quantizer's status.
 */
int w4ref_awq_search(const uint16_t *W, const uint16_t *X, int dtype, long Mc, long K, long N,
                     long group, int sym, const float *alphas, long n_alpha, double *err,
                     float *s_all, long *best)
{
    if (Mc <= 0 || K <= 0 || N <= 0 || n_alpha <= 0) return W4REF_EINVAL;
    if (group <= 0 || group > 4096 || group % 8 != 0 || K % group != 0) return W4REF_EINVAL;
    if (dtype != DT_F16 && dtype != DT_BF16) return W4REF_EINVAL;
    fesetround(FE_TONEAREST);
    const long G = K / group;
    int status = W4REF_OK;
    float *a = malloc(sizeof(float) * K);
    float *wm = malloc(sizeof(float) * K);
    float *s = malloc(sizeof(float) * K);
    double *Yref = malloc(sizeof(double) * Mc * N);
    double *D = malloc(sizeof(double) * Mc * N);
    double *Xs = malloc(sizeof(double) * Mc * K);
    double *What = malloc(sizeof(double) * N * K);
    uint8_t *packed = malloc((size_t)N * K / 2);
    float *scales = malloc(sizeof(float) * N * G);
    float *zeros = malloc(sizeof(float) * N * G);
    if (!a || !wm || !s || !Yref || !D || !Xs || !What || !packed || !scales || !zeros) {
        status = W4REF_EINVAL;
        goto done;
    }

    /* importance of each input channel: mean |X_ij| over the calibration rows,
       and the weight magnitude: mean |W_nj| over the output rows */
    for (long j = 0; j < K; ++j) {
        double sa = 0.0, sw = 0.0;
        for (long i = 0; i < Mc; ++i) sa += fabs(decode16(X[i * K + j], dtype));
        for (long n = 0; n < N; ++n) sw += fabs(decode16(W[n * K + j], dtype));
        a[j] = (float)(sa / (double)Mc);
        wm[j] = (float)(sw / (double)N);
    }

    /* the unquantized layer's output W X on the calibration rows */
#pragma omp parallel for schedule(static)
    for (long i = 0; i < Mc; ++i)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k)
                acc += decode16(X[i * K + k], dtype) * decode16(W[n * K + k], dtype);
            Yref[i * N + n] = acc;
        }

    for (long t = 0; t < n_alpha; ++t) {
        const double alpha = (double)alphas[t];
        /* s_j = (a_j / w_j)^alpha */
        for (long j = 0; j < K; ++j)
            s[j] = (a[j] == 0.0f || wm[j] == 0.0f) ? 1.0f
                                                   : (float)pow((double)a[j] / (double)wm[j], alpha);
        if (s_all) memcpy(s_all + t * K, s, sizeof(float) * K);
        /* Q(W * s): fold s into the columns, then the per-group quantizer */
        int st = w4ref_quantize(W, dtype, K, N, group, sym, s, packed, scales, zeros);
        if (st != W4REF_OK) {
            status = st;
            goto done;
        }
        st = w4ref_dequant(packed, scales, sym ? NULL : zeros, K, N, group, What);
        if (st != W4REF_OK) {
            status = st;
            goto done;
        }
        /* X / s, as the 16-bit activations of the quantized layer */
        for (long i = 0; i < Mc; ++i)
            for (long k = 0; k < K; ++k) {
                float x = (float)decode16(X[i * K + k], dtype);
                Xs[i * K + k] = w4ref_round16((double)(x / s[k]), dtype);
            }
        /* || Q(W * s)(X / s) - W X ||^2: squared differences, then one sum in
           (i, n) order */
#pragma omp parallel for schedule(static)
        for (long i = 0; i < Mc; ++i)
            for (long n = 0; n < N; ++n) {
                double acc = 0.0;
                for (long k = 0; k < K; ++k) acc += Xs[i * K + k] * What[n * K + k];
                const double d = w4ref_round16(acc, dtype) - Yref[i * N + n];
                D[i * N + n] = d * d;
            }
        double e = 0.0;
        for (long i = 0; i < Mc * N; ++i) e += D[i];
        err[t] = e;
    }

    /* grid search: the first alpha with the smallest error */
    *best = -1;
    for (long t = 0; t < n_alpha; ++t)
        if (!isnan(err[t]) && (*best < 0 || err[t] < err[*best])) *best = t;

done:
    free(a);
    free(wm);
    free(s);
    free(Yref);
    free(D);
    free(Xs);
    free(What);
    free(packed);
    free(scales);
    free(zeros);
    return status;
}

/* ---- W8A8: SmoothQuant factors, per-tensor INT8 / FP8 E4M3, the 8-bit GEMM -------------- */
/*
 *   [LQ] §4.3 SmoothQuant: s_j = max|X_j|^alpha / max|W_j|^(1-alpha) (alpha = 0.5),
 *        clamped below at 1e-5; W' = W * s (columns), X' = X / s; both quantized
 *        to INT8 with the symmetric formula of §2.2 (per tensor; X dynamically).
 *   [LQ] §4.6 FP8: scale = max|x| / 448 (the largest E4M3 value), x_fp8 = cast(x / scale).
 *   [LQ] §2.2 symmetric: s = max|x| / (2^(b-1) - 1), q = clamp(round(x / s), -qmax, qmax).
 */

#define FMT_INT8 0
#define FMT_E4M3 1

/*
 * Nearest E4M3 value to v (ties to even) as a double: 4 significant bits,
 * smallest normal exponent -6 (spacing 2^-9 below it), largest finite 448;
 * magnitudes beyond 448 saturate to +-448 (no infinities in this format).
 */
double w4ref_round_e4m3(double v)
{
    if (v == 0.0 || isnan(v)) return v;
    int e;
    frexp(v, &e);
    int lead = e - 1;
    if (lead < -6) lead = -6;
    const int q = lead - 3;
    double r = ldexp(nearbyint(ldexp(v, -q)), q);
    if (fabs(r) > 448.0) r = copysign(448.0, v);
    return r;
}

/* Byte code of an E4M3 value r (exactly representable): sign, 4 exponent bits
   (bias 7; 0 = subnormal), 3 fraction bits. */
static uint8_t e4m3_code(double r)
{
    uint8_t sign = signbit(r) ? 0x80 : 0;
    double a = fabs(r);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -6) /* subnormal: a = f * 2^-9, f in 1..7 */
        return sign | (uint8_t)(int)ldexp(a, 9);
    const int frac = (int)(ldexp(a, 3 - lead)) - 8; /* a = (8 + frac) * 2^(lead-3) */
    return sign | (uint8_t)((lead + 7) << 3) | (uint8_t)frac;
}

/* Value of an E4M3 byte (0x7F / 0xFF are NaN). */
double w4ref_e4m3_to_f64(uint8_t c)
{
    const int sign = c >> 7, e = (c >> 3) & 0xF, f = c & 7;
    double v;
    if (e == 15 && f == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)f, -9);
    else
        v = ldexp((double)(8 + f), e - 10);
    return sign ? -v : v;
}

/*
 * SmoothQuant factors: a_j = max_i |X_ij|, w_j = max_n |W_nj| (exact),
 * s_j = max(fl32(fl32(a_j^alpha) / fl32(w_j^(1-alpha))), 1e-5), each power in
 * fp64 rounded once to fp32, the quotient an fp32 division.  A channel with
 * a_j == 0 or w_j == 0 keeps s_j = 1.
 */
int w4ref_smooth_scales(const uint16_t *X, const uint16_t *W, int dtype, long Mc, long K, long N,
                        double alpha, float *s)
{
    if (Mc <= 0 || K <= 0 || N <= 0) return W4REF_EINVAL;
    fesetround(FE_TONEAREST);
    for (long j = 0; j < K; ++j) {
        double a = 0.0, w = 0.0;
        for (long i = 0; i < Mc; ++i) a = fmax(a, fabs(decode16(X[i * K + j], dtype)));
        for (long n = 0; n < N; ++n) w = fmax(w, fabs(decode16(W[n * K + j], dtype)));
        if (a == 0.0 || w == 0.0) {
            s[j] = 1.0f;
            continue;
        }
        const float num = (float)pow((double)(float)a, alpha);
        const float den = (float)pow((double)(float)w, 1.0 - alpha);
        float v = num / den;
        s[j] = v < 1e-5f ? 1e-5f : v;
    }
    return W4REF_OK;
}

/*
 * Per-tensor symmetric 8-bit quantization of A [rows][K] (16-bit bits).
 * col_op: 0 none, 1 multiply column k by col[k] (the weight side, W * s),
 * 2 divide column k by col[k] (the activation side, X / s); one fp32 op.
 * fmt INT8: scale = fl32(amax / 127), q = clamp(rne(fl32(v / scale)), -127, 127);
 * fmt E4M3: scale = fl32(amax / 448), q = e4m3(fl32(v / scale)).
 * amax = 0 gives scale = 0 and every q = 0.  q is [rows][K] bytes (int8 or E4M3).
 */
int w4ref_quant8(const uint16_t *A, int dtype, long rows, long K, const float *col, int col_op,
                 int fmt, uint8_t *q, float *scale_out)
{
    if (rows <= 0 || K <= 0 || (col_op != 0 && !col) || col_op < 0 || col_op > 2) return W4REF_EINVAL;
    if (fmt != FMT_INT8 && fmt != FMT_E4M3) return W4REF_EINVAL;
    fesetround(FE_TONEAREST);
    float amax = 0.0f;
    for (long i = 0; i < rows * K; ++i) {
        float v = (float)decode16(A[i], dtype);
        if (col_op == 1) v = v * col[i % K];
        if (col_op == 2) v = v / col[i % K];
        if (!isfinite(v)) return W4REF_ENONFINITE;
        if (fabsf(v) > amax) amax = fabsf(v);
    }
    const float scale = amax / (fmt == FMT_INT8 ? 127.0f : 448.0f);
    *scale_out = scale;
    for (long i = 0; i < rows * K; ++i) {
        float v = (float)decode16(A[i], dtype);
        if (col_op == 1) v = v * col[i % K];
        if (col_op == 2) v = v / col[i % K];
        if (scale == 0.0f) {
            q[i] = 0;
            continue;
        }
        const float t = v / scale;
        if (fmt == FMT_INT8)
            q[i] = (uint8_t)(int8_t)(int)clampf(rne(t), -127.0f, 127.0f);
        else
            q[i] = e4m3_code(w4ref_round_e4m3((double)t));
    }
    return W4REF_OK;
}

/*
 * The W8A8 layer on quantized operands: Y[m][n] from Xq [M][K] and Wq [N][K].
 * INT8: the exact integer sum acc, then y = fl32(fl32(acc) * fl32(sx * sw))
 *       rounded once to the 16-bit dtype (the tensor-core path's epilogue);
 *       Y holds that 16-bit value.
 * E4M3: Y holds the exact product sum_k x_k w_k * sx * sw in fp64 (unrounded).
 * rows (nullable) selects the m to compute, as in w4ref_linear.
 */
int w4ref_gemm8(const uint8_t *Xq, const uint8_t *Wq, int fmt, long M, long K, long N, float sx,
                float sw, int dtype, const long *rows, long nrows, double *Y)
{
    if (M <= 0 || K <= 0 || N <= 0) return W4REF_EINVAL;
    if (fmt != FMT_INT8 && fmt != FMT_E4M3) return W4REF_EINVAL;
    fesetround(FE_TONEAREST);
    if (!rows) nrows = M;
    const float alpha = sx * sw;
    double e4m3[256]; /* value of every E4M3 byte, from the decoder above */
    for (int c = 0; c < 256; ++c) e4m3[c] = w4ref_e4m3_to_f64((uint8_t)c);
#pragma omp parallel for schedule(static)
    for (long r = 0; r < nrows; ++r) {
        const long m = rows ? rows[r] : r;
        if (m < 0 || m >= M) continue;
        for (long n = 0; n < N; ++n) {
            if (fmt == FMT_INT8) {
                long long acc = 0;
                for (long k = 0; k < K; ++k)
                    acc += (long long)(int8_t)Xq[m * K + k] * (long long)(int8_t)Wq[n * K + k];
                const float y = (float)acc * alpha;
                Y[r * N + n] = w4ref_round16((double)y, dtype);
            } else {
                double acc = 0.0;
                for (long k = 0; k < K; ++k)
                    acc += e4m3[Xq[m * K + k]] * e4m3[Wq[n * K + k]];
                Y[r * N + n] = acc * (double)sx * (double)sw;
            }
        }
    }
    return W4REF_OK;
}


/* ---- GPTQ: Hessian-guided column-by-column quantization ------------------------------- */
/*
 *   [LQ] §4.1 GPTQ: minimise ||WX - W^X||_F^2 with H = 2 X X^T; quantize one
 *        column at a time and push each column's error onto the columns not yet
 *        quantized through the inverse Hessian (delta_j = (w_j - q_j) / [H^-1]_jj,
 *        W[:, j+1:] -= delta_j H^-1[j, j+1:]); in practice through a Cholesky
 *        factor of H^-1, with the updates to later blocks batched.
 *   [PTQ] section "GPTQ": lazy batch updates every 128 columns.
 *   Here X is [Mc][K] (rows = calibration samples), so H = 2 X^T X is [K][K].
 *   U is the upper Cholesky factor of H^-1 (H^-1 = U^T U); its row j gives
 *   [H_F^-1]_jj and the update row of the still-unquantized set F at step j.
 */

/* Group parameters (the RTN quantizer's formulas above) of w[0..g-1]. */
static void group_params(const float *w, long g, int sym, float *s_out, float *z_out)
{
    if (sym) {
        float amax = 0.0f;
        for (long i = 0; i < g; ++i)
            if (fabsf(w[i]) > amax) amax = fabsf(w[i]);
        *s_out = amax / 7.0f;
        *z_out = 8.0f;
    } else {
        float mn = w[0], mx = w[0];
        for (long i = 1; i < g; ++i) {
            if (w[i] < mn) mn = w[i];
            if (w[i] > mx) mx = w[i];
        }
        const float s = (mx - mn) / 15.0f;
        *s_out = s;
        *z_out = s == 0.0f ? 0.0f : clampf(rne((-mn) / s), 0.0f, 15.0f) + 0.0f;
    }
}

/* Stored code u of w under (s, z): the RTN quantizer's rounding and clamp. */
static int code_of(float w, float s, float z, int sym)
{
    if (s == 0.0f) return (int)z;
    if (sym) return (int)clampf(rne(w / s), -7.0f, 7.0f) + 8;
    return (int)clampf(rne(w / s + z), 0.0f, 15.0f);
}

/*
 * The GPTQ column loop for W [N][K] (16-bit bits) given U [K][K] fp32
 * (row-major; only the upper triangle k >= j is read).  block == group:
 * each group's parameters are taken from the row's current weights when the
 * loop reaches the group (all earlier blocks' updates applied, none of its
 * own).  Every update is fp32:
 *   in the block, after column j:  w_k = fma(-err_j, U[j][k], w_k), k > j;
 *   err_j = (w_j - (u_j - z) * s) / U[j][j];
 *   after the block, for each later k: acc = fma chain over the block's j in
 *   order (acc = fma(err_j, U[j][k], acc) from 0), then w_k = w_k - acc.
 * Outputs in the w4_quantize layout: packed [N][K/2], scales and zeros [N][K/group].
 */
int w4ref_gptq_quantize(const uint16_t *W, int dtype, long K, long N, long group, int sym,
                        const float *U, uint8_t *packed, float *scales, float *zeros)
{
    if (K <= 0 || N <= 0 || group <= 0 || group > 4096 || group % 8 != 0 || K % group != 0)
        return W4REF_EINVAL;
    fesetround(FE_TONEAREST);
    const long G = K / group;
    int status = W4REF_OK;
#pragma omp parallel
    {
        float *w = malloc(sizeof(float) * K);
        float *err = malloc(sizeof(float) * group);
        uint8_t *u = malloc(K);
        if (!w || !err || !u) {
#pragma omp atomic write
            status = W4REF_EINVAL;
        }
#pragma omp for schedule(static)
        for (long n = 0; n < N; ++n) {
            if (!w || !err || !u) continue;
            for (long k = 0; k < K; ++k) w[k] = (float)decode16(W[n * K + k], dtype);
            for (long g = 0; g < G; ++g) {
                const long b0 = g * group;
                float s, z;
                group_params(w + b0, group, sym, &s, &z);
                scales[n * G + g] = s;
                zeros[n * G + g] = z;
                for (long jj = 0; jj < group; ++jj) {
                    const long j = b0 + jj;
                    const int c = code_of(w[j], s, z, sym);
                    u[j] = (uint8_t)c;
                    const float deq = (float)c - z;
                    const float e = (w[j] - deq * s) / U[j * K + j];
                    err[jj] = e;
                    for (long k = j + 1; k < b0 + group; ++k) w[k] = fmaf(-e, U[j * K + k], w[k]);
                }
                for (long k = b0 + group; k < K; ++k) {
                    float acc = 0.0f;
                    for (long jj = 0; jj < group; ++jj) acc = fmaf(err[jj], U[(b0 + jj) * K + k], acc);
                    w[k] = w[k] - acc;
                }
            }
            for (long j8 = 0; j8 < K / 8; ++j8) {
                uint32_t word = 0;
                for (int i = 0; i < 8; ++i) word |= (uint32_t)(u[j8 * 8 + SIGMA[i]] & 0xF) << (4 * i);
                uint8_t *dst = packed + n * (K / 2) + j8 * 4;
                for (int b = 0; b < 4; ++b) dst[b] = (uint8_t)(word >> (8 * b));
            }
        }
        free(w);
        free(err);
        free(u);
    }
    return status;
}

/* H = 2 X^T X in fp64 ([K][K]) from X [Mc][K] (16-bit bits). */
int w4ref_gptq_hessian(const uint16_t *X, int dtype, long Mc, long K, double *H)
{
    if (Mc <= 0 || K <= 0) return W4REF_EINVAL;
    double *Xt = malloc(sizeof(double) * Mc * K); /* X transposed, decoded: Xt[a][i] */
    if (!Xt) return W4REF_EINVAL;
    for (long i = 0; i < Mc; ++i)
        for (long a = 0; a < K; ++a) Xt[a * Mc + i] = decode16(X[i * K + a], dtype);
#pragma omp parallel for schedule(static)
    for (long a = 0; a < K; ++a)
        for (long b = 0; b < K; ++b) {
            double acc = 0.0;
            for (long i = 0; i < Mc; ++i) acc += Xt[a * Mc + i] * Xt[b * Mc + i];
            H[a * K + b] = 2.0 * acc;
        }
    free(Xt);
    return W4REF_OK;
}
