/*
 * bnbq_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE LIBRARY (see bnbq_oracle.h for the
 * source keys [BWQ], [CN-32], [CN-OPT], [PT-W3], [NF4], [ADAM], [LION], [QLORA]).
 *
 * Plain loops, single thread, no blocking beyond the method's own blocks, no fusion, no
 * vectorisation.  Built with: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math.
 */
#include "bnbq_oracle.h"

#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------
 * Codebooks.
 *
 * [BWQ] names dynamic quantization, a non-linear code meant to keep small and large
 * magnitudes alike accurate, and gives no values.  Reading taken: the dynamic tree
 * of the same paper -- a magnitude is 10^-E * f where E counts leading zero bits, one
 * indicator bit follows, and the remaining bits select one of 2^nE equal fraction bins of
 * (0.1, 1]; the bin's upper edge is used, so the largest code is exactly 1.
 * A magnitude with E leading zeros and nE fraction bits, bin k, is the rational
 *      10^-E * (1/10 + 9/10 * (k+1)/2^nE) = (2^nE + 9(k+1)) / (2^nE * 10^(E+1)).
 * ------------------------------------------------------------------------------------ */
static float dyn_magnitude(int E, int nE, int k)
{
    double num = (double)((1 << nE) + 9 * (k + 1));
    double den = (double)(1 << nE) * pow(10.0, (double)(E + 1));
    return (float)(num / den);
}

static void sort_floats(float* v, int n)
{
    /* insertion sort: plain and obviously correct for 256 entries */
    for (int i = 1; i < n; i++) {
        float x = v[i];
        int j = i - 1;
        while (j >= 0 && v[j] > x) {
            v[j + 1] = v[j];
            j--;
        }
        v[j + 1] = x;
    }
}

/* Unsigned dynamic code (second Adam state v >= 0): 8 magnitude bits, E = 0..7 leading
 * zeros, nE = 7 - E fraction bits -> 255 magnitudes in [1e-7, 1], plus the all-zero code. */
void oracle_code_dynamic_unsigned(float out[256])
{
    int c = 0;
    out[c++] = 0.0f;
    for (int E = 0; E <= 7; E++) {
        int nE = 7 - E;
        for (int k = 0; k < (1 << nE); k++) out[c++] = dyn_magnitude(E, nE, k);
    }
    sort_floats(out, 256);
}

/* Signed dynamic code (first moment m, Lion / momentum state): a sign bit and 7 magnitude
 * bits, E = 0..6, nE = 6 - E -> 127 magnitudes in [1e-6, 1].  +m, -m and one zero give 255
 * values; the 256th bit pattern (the "negative zero") is given the next tree level, +1e-7,
 * so that the table stays strictly increasing and holds -1, 0 and +1 exactly. */
void oracle_code_dynamic_signed(float out[256])
{
    int c = 0;
    out[c++] = 0.0f;
    for (int E = 0; E <= 6; E++) {
        int nE = 6 - E;
        for (int k = 0; k < (1 << nE); k++) {
            float m = dyn_magnitude(E, nE, k);
            out[c++] = m;
            out[c++] = -m;
        }
    }
    out[c++] = (float)(1.0 / 1e7);
    sort_floats(out, 256);
}

/* Standard normal CDF from the complementary error function of the C library. */
static double normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Inverse normal CDF by bisection on normal_cdf: slow, plain, accurate to the double
 * resolution of the bracket. */
static double normal_quantile(double p)
{
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 2000; it++) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (normal_cdf(mid) < p)
            lo = mid;
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* NF4 [NF4], constructed as in [QLORA] section 3: quantiles of N(0,1) -- 8 positive values at
 * probabilities evenly spaced over (1/2, 1-delta], 7 negative values at probabilities evenly
 * spaced over [delta, 1/2), and zero -- each divided by the largest magnitude so that -1, 0
 * and +1 are exact.  delta = (1/30 + 1/32)/2 (the offset of [QLORA]; not on the pages). */
void oracle_code_nf4(float out[16])
{
    const double delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
    const double scale = normal_quantile(1.0 - delta);
    int c = 0;
    for (int k = 0; k <= 6; k++) {
        double prob = delta + (0.5 - delta) * (double)k / 7.0;
        out[c++] = (float)(normal_quantile(prob) / scale);
    }
    out[c++] = 0.0f;
    for (int k = 1; k <= 8; k++) {
        double prob = 0.5 + (0.5 - delta) * (double)k / 8.0;
        out[c++] = (float)(normal_quantile(prob) / scale);
    }
    sort_floats(out, 16);
}

/* FP4 [FP4]: the 4-bit float E2M1 -- a sign bit, 2 exponent bits (bias 1) and 1 mantissa bit,
 * subnormals and no inf/NaN, so the magnitudes are 0, 0.5 (subnormal) and 2^(e-1) * (1 + f/2)
 * for e = 1..3, f = 0..1: 1, 1.5, 2, 3, 4, 6 -- divided by the largest, 6, so -1, 0 and +1 are
 * exact.  READING: E2M1 has two zeros; the codebook must be strictly increasing, so the -0
 * pattern is given the next finer subnormal magnitude, 0.25/6 (as the signed dynamic code gives
 * its -0 pattern the next tree level).  16 values, formed in double and rounded once. */
void oracle_code_fp4(float out[16])
{
    int c = 0;
    for (int sign = -1; sign <= 1; sign += 2) {
        for (int e = 0; e <= 3; e++) {
            for (int f = 0; f <= 1; f++) {
                double mag = (e == 0) ? 0.5 * (double)f : ldexp(1.0 + 0.5 * (double)f, e - 1);
                if (sign < 0 && e == 0 && f == 0) {
                    out[c++] = (float)(0.25 / 6.0); /* the -0 pattern */
                    continue;
                }
                out[c++] = (float)((double)sign * mag / 6.0);
            }
        }
    }
    sort_floats(out, 16);
}

/* Linear (uniform) code over [-1, 1], used by tests only. */
void oracle_code_linear(float out[256])
{
    for (int k = 0; k < 256; k++) out[k] = (float)(-1.0 + 2.0 * (double)k / 255.0);
}

/* ------------------------------------------------------------------------------------
 * Nearest-code rule.  The normalised value xn in [-1, 1] is given the index of the nearest
 * code; the decision is taken against the binary32 midpoints of neighbouring codes,
 *      mid_j = fl32((code_j + code_{j+1}) / 2)   (sum formed in double),
 *      q = #{ j : xn > mid_j },
 * so a value exactly on a midpoint goes to the lower code.
 * ------------------------------------------------------------------------------------ */
float oracle_code_mid(const float* code, int j)
{
    return (float)(((double)code[j] + (double)code[j + 1]) * 0.5);
}

int oracle_nearest_code(const float* code, int K, float xn)
{
    int q = 0;
    for (int j = 0; j < K - 1; j++)
        if (xn > oracle_code_mid(code, j)) q++;
    return q;
}

/* ---- bf16 ---- */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb; /* round to nearest, ties to even */
    return (uint16_t)(u >> 16);
}

static float load_value(const void* x, int dtype, int64_t i)
{
    if (dtype == OR_BF16) return oracle_bf16_to_f32(((const uint16_t*)x)[i]);
    return ((const float*)x)[i];
}

static int valid_blocksize(int B) { return B == 64 || B == 128 || B == 256 || B == 2048 || B == 4096; }

/* ------------------------------------------------------------------------------------
 * Block-wise quantization [BWQ]: the tensor is cut into blocks of B consecutive elements
 * (the last one may be shorter; blocks never cross tensors), each block is normalised by
 * its own absolute maximum and quantized on its own.
 * ------------------------------------------------------------------------------------ */
static float block_absmax(const float* v, int64_t len)
{
    float a = 0.0f;
    for (int64_t i = 0; i < len; i++) {
        float m = fabsf(v[i]);
        if (m > a) a = m;
    }
    return a;
}

static int quantize_one(const float* code, int K, float x, float absmax)
{
    float xn = (absmax == 0.0f) ? 0.0f : x / absmax;
    return oracle_nearest_code(code, K, xn);
}

int oracle_quantize_blockwise(const float* code, int K, const void* x, int x_dtype, int64_t n,
                              int B, float* absmax, uint8_t* out)
{
    if (!code || (K != 256 && K != 16) || n < 0 || !valid_blocksize(B)) return -1;
    if (n == 0) return 0;
    if (!x || !absmax || !out) return -1;
    float buf[4096];
    int64_t nb = (n + B - 1) / B;
    if (K == 16) memset(out, 0, (size_t)((n + 1) / 2));
    for (int64_t b = 0; b < nb; b++) {
        int64_t start = b * (int64_t)B;
        int64_t len = (n - start < B) ? (n - start) : B;
        for (int64_t i = 0; i < len; i++) buf[i] = load_value(x, x_dtype, start + i);
        float a = block_absmax(buf, len);
        absmax[b] = a;
        for (int64_t i = 0; i < len; i++) {
            int q = quantize_one(code, K, buf[i], a);
            int64_t e = start + i;
            if (K == 256) {
                out[e] = (uint8_t)q;
            } else if ((e & 1) == 0) {
                out[e >> 1] = (uint8_t)(out[e >> 1] | (q << 4)); /* even element: high nibble */
            } else {
                out[e >> 1] = (uint8_t)(out[e >> 1] | q);        /* odd element: low nibble */
            }
        }
    }
    return 0;
}

int oracle_dequantize_blockwise(const float* code, int K, const uint8_t* q, const float* absmax,
                                int64_t n, int B, void* y, int y_dtype)
{
    if (!code || (K != 256 && K != 16) || n < 0 || !valid_blocksize(B)) return -1;
    if (n == 0) return 0;
    if (!q || !absmax || !y) return -1;
    for (int64_t e = 0; e < n; e++) {
        int idx;
        if (K == 256)
            idx = q[e];
        else
            idx = (e & 1) ? (q[e >> 1] & 0xf) : (q[e >> 1] >> 4);
        float v = code[idx] * absmax[e / B];
        if (y_dtype == OR_BF16)
            ((uint16_t*)y)[e] = oracle_f32_to_bf16(v);
        else
            ((float*)y)[e] = v;
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Nested (double) quantization of the block scales [NEST]: the fp32 absmax array of an
 * already quantized tensor is itself quantized.  Following [QLORA] (section 3, "Double
 * Quantization"): the scales are centred by their mean (they are all >= 0, the code is
 * signed) and quantized block-wise to 8 bits in blocks of 256 with the signed dynamic code.
 * Reconstruction: a_i = code2[qabs_i] * absmax2[i / 256] + offset (two roundings).
 * READING: the mean's summation order is not given anywhere; it is fixed here as a double
 * sum over chunks of 4096 consecutive scales (each chunk summed in index order, the chunk
 * sums added in index order), divided by nb in double and rounded once to float.
 * ------------------------------------------------------------------------------------ */
float oracle_absmax_mean(const float* absmax, int64_t nb)
{
    if (nb <= 0) return 0.0f;
    double total = 0.0;
    for (int64_t c = 0; c < nb; c += ORACLE_NEST_CHUNK) {
        int64_t end = (c + ORACLE_NEST_CHUNK < nb) ? c + ORACLE_NEST_CHUNK : nb;
        double s = 0.0;
        for (int64_t i = c; i < end; i++) s += (double)absmax[i];
        total += s;
    }
    return (float)(total / (double)nb);
}

int oracle_nest_absmax(const float* absmax, int64_t nb, const float* code2, uint8_t* qabs,
                       float* absmax2, float* offset)
{
    if (nb < 0 || !code2 || !offset) return -1;
    *offset = 0.0f;
    if (nb == 0) return 0;
    if (!absmax || !qabs || !absmax2) return -1;
    float mean = oracle_absmax_mean(absmax, nb);
    float* centred = (float*)malloc((size_t)nb * sizeof(float));
    if (!centred) return -1;
    for (int64_t i = 0; i < nb; i++) centred[i] = absmax[i] - mean;
    int rc = oracle_quantize_blockwise(code2, 256, centred, OR_F32, nb, ORACLE_NEST_B, absmax2, qabs);
    free(centred);
    *offset = mean;
    return rc;
}

int oracle_unnest_absmax(const uint8_t* qabs, const float* absmax2, float offset, const float* code2,
                         int64_t nb, float* out)
{
    if (nb < 0 || !code2) return -1;
    if (nb == 0) return 0;
    if (!qabs || !absmax2 || !out) return -1;
    for (int64_t i = 0; i < nb; i++) out[i] = code2[qabs[i]] * absmax2[i / ORACLE_NEST_B] + offset;
    return 0;
}

/* ------------------------------------------------------------------------------------
 * The optimizer step [BWQ]: per block, dequantize the 8-bit state, apply the 32-bit update
 * to the fp32 parameters, take the new block absmax of each state and requantize it.
 *
 * Update rules (each binary32 operation rounded on its own, left to right):
 *   AdamW [ADAM, decoupled decay]:  m' = b1*m + (1-b1)*g ;  v' = b2*v + ((1-b2)*g)*g
 *        p = p*(1 - lr*wd) ;  p = p - (lr/bc1) * (m' / (sqrt(v')/sqrt(bc2) + eps))
 *        with bc1 = 1 - b1^t, bc2 = 1 - b2^t.
 *   Adam: as AdamW with no decoupled decay; weight decay, if any, is added to the gradient
 *        first, g = g + wd*p.
 *   Lion [LION]: c = b1*m + (1-b1)*g ; p = p*(1 - lr*wd) ; p = p - lr*sign(c) (sign(0)=0);
 *        m' = b2*m + (1-b2)*g.
 *   Momentum SGD (the "exponentially smoothed sum" of [BWQ]; dampening 0): g = g + wd*p if
 *        wd != 0 ; m' = b1*m + g ; p = p - lr*m'.
 *   RMSprop [RMSP] (one state, the running mean of squares, kept with the unsigned code; b1
 *        carries the smoothing constant alpha): g = g + wd*p if wd != 0 ;
 *        v' = b1*v + ((1-b1)*g)*g ; p = p - lr * (g / (sqrt(v') + eps)).
 * The update uses the unrounded binary32 m', v'; only the stored state is quantized.
 * ------------------------------------------------------------------------------------ */
typedef struct {
    float b1, b2, omb1, omb2, step_size, sqrt_bc2, decay, lr, eps, wd;
} derived_scalars;

static derived_scalars derive(int optim, const oracle_hparams* hp, int t)
{
    derived_scalars d;
    double b1 = hp->beta1, b2 = hp->beta2;
    d.b1 = hp->beta1;
    d.b2 = hp->beta2;
    d.omb1 = (float)(1.0 - b1);
    d.omb2 = (float)(1.0 - b2);
    d.step_size = (float)((double)hp->lr / (1.0 - pow(b1, (double)t)));
    d.sqrt_bc2 = (float)sqrt(1.0 - pow(b2, (double)t));
    d.decay = (optim == OR_ADAMW || optim == OR_LION)
                  ? (float)(1.0 - (double)hp->lr * (double)hp->weight_decay)
                  : 1.0f;
    d.lr = hp->lr;
    d.eps = hp->eps;
    d.wd = hp->weight_decay;
    return d;
}

static int n_states(int optim) { return (optim == OR_ADAMW || optim == OR_ADAM) ? 2 : 1; }

/* One element: given p, g and the dequantized (or 32-bit) state m, v, return the new p, m, v. */
static void update_element(int optim, const derived_scalars* d, float* p, float g, float* m,
                           float* v)
{
    float pv = *p;
    if (optim == OR_ADAMW || optim == OR_ADAM) {
        if (optim == OR_ADAM && d->wd != 0.0f) g = g + d->wd * pv;
        float m1 = d->b1 * (*m) + d->omb1 * g;
        float v1 = d->b2 * (*v) + (d->omb2 * g) * g;
        if (optim == OR_ADAMW) pv = pv * d->decay;
        float denom = sqrtf(v1) / d->sqrt_bc2 + d->eps;
        pv = pv - d->step_size * (m1 / denom);
        *m = m1;
        *v = v1;
    } else if (optim == OR_LION) {
        float c = d->b1 * (*m) + d->omb1 * g;
        float s = (c > 0.0f) ? 1.0f : ((c < 0.0f) ? -1.0f : 0.0f);
        pv = pv * d->decay;
        pv = pv - d->lr * s;
        *m = d->b2 * (*m) + d->omb2 * g;
    } else if (optim == OR_MOMENTUM) {
        if (d->wd != 0.0f) g = g + d->wd * pv;
        float m1 = d->b1 * (*m) + g;
        pv = pv - d->lr * m1;
        *m = m1;
    } else { /* OR_RMSPROP: the state slot m holds the mean of squares */
        if (d->wd != 0.0f) g = g + d->wd * pv;
        float v1 = d->b1 * (*m) + (d->omb1 * g) * g;
        float denom = sqrtf(v1) + d->eps;
        pv = pv - d->lr * (g / denom);
        *m = v1;
    }
    *p = pv;
}

int oracle_step_blocks(int optim, int state_bits, float* p, const void* g, int g_dtype, int64_t n,
                       void* s1, void* s2, float* absmax1, float* absmax2, const float* code1,
                       const float* code2, int B, const oracle_hparams* hp, int t, int64_t b0,
                       int64_t b1)
{
    if (optim < OR_ADAMW || optim > OR_RMSPROP || (state_bits != 8 && state_bits != 32)) return -1;
    if (n < 0 || !valid_blocksize(B) || t < 1 || !hp) return -1;
    if (n == 0) return 0;
    int ns = n_states(optim);
    if (!p || !g || !s1 || (ns == 2 && !s2)) return -1;
    if (state_bits == 8 && (!absmax1 || !code1 || (ns == 2 && (!absmax2 || !code2)))) return -1;
    int64_t nb = (n + B - 1) / B;
    if (b0 < 0) b0 = 0;
    if (b1 > nb) b1 = nb;

    derived_scalars d = derive(optim, hp, t);
    float mbuf[4096], vbuf[4096];

    for (int64_t b = b0; b < b1; b++) {
        int64_t start = b * (int64_t)B;
        int64_t len = (n - start < B) ? (n - start) : B;
        /* 1. load and dequantize the state of this block */
        for (int64_t i = 0; i < len; i++) {
            int64_t e = start + i;
            if (state_bits == 8) {
                mbuf[i] = code1[((const uint8_t*)s1)[e]] * absmax1[b];
                vbuf[i] = (ns == 2) ? code2[((const uint8_t*)s2)[e]] * absmax2[b] : 0.0f;
            } else {
                mbuf[i] = ((const float*)s1)[e];
                vbuf[i] = (ns == 2) ? ((const float*)s2)[e] : 0.0f;
            }
        }
        /* 2. the 32-bit update, element by element */
        for (int64_t i = 0; i < len; i++) {
            int64_t e = start + i;
            update_element(optim, &d, &p[e], load_value(g, g_dtype, e), &mbuf[i], &vbuf[i]);
        }
        /* 3. store the state: new block absmax, then requantize each element */
        if (state_bits == 8) {
            float a1 = block_absmax(mbuf, len);
            absmax1[b] = a1;
            for (int64_t i = 0; i < len; i++)
                ((uint8_t*)s1)[start + i] = (uint8_t)quantize_one(code1, 256, mbuf[i], a1);
            if (ns == 2) {
                float a2 = block_absmax(vbuf, len);
                absmax2[b] = a2;
                for (int64_t i = 0; i < len; i++)
                    ((uint8_t*)s2)[start + i] = (uint8_t)quantize_one(code2, 256, vbuf[i], a2);
            }
        } else {
            for (int64_t i = 0; i < len; i++) {
                ((float*)s1)[start + i] = mbuf[i];
                if (ns == 2) ((float*)s2)[start + i] = vbuf[i];
            }
        }
    }
    return 0;
}

int oracle_step_tensor(int optim, int state_bits, float* p, const void* g, int g_dtype, int64_t n,
                       void* s1, void* s2, float* absmax1, float* absmax2, const float* code1,
                       const float* code2, int B, const oracle_hparams* hp, int t)
{
    if (!valid_blocksize(B)) return -1;
    return oracle_step_blocks(optim, state_bits, p, g, g_dtype, n, s1, s2, absmax1, absmax2,
                              code1, code2, B, hp, t, 0, (n + B - 1) / B);
}
