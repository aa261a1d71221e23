/*
 * oracle.c -- plain, single-threaded CPU oracle of the loss-scaled FP32-master
 * SGD-momentum step.  TEST INFRASTRUCTURE ONLY (see oracle.h): the product
 * path never includes, links or runs it.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fPIC -shared (x86-64 SSE
 * scalar arithmetic, so every float operation below rounds once to binary32).
 */
#include "oracle.h"

#include <math.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* binary16 codec, written from the IEEE-754 definition of the formats.     */
/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits;       */
/* normal exponents [-14, 15], largest finite 65504, smallest subnormal     */
/* 2^-24 (the ranges the analysis page quotes in section 3.4, "Failure      */
/* mechanism 1").                                                           */
/* ------------------------------------------------------------------------ */

static uint32_t bits_of(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    return u;
}

static float float_of(uint32_t u)
{
    float x;
    memcpy(&x, &u, sizeof x);
    return x;
}

uint16_t orc_rne16(float x)
{
    uint32_t u = bits_of(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t exp32 = (u >> 23) & 0xffu;
    uint32_t frac32 = u & 0x7fffffu;

    if (exp32 == 0xffu) {
        if (frac32 == 0)
            return (uint16_t)(sign | 0x7c00u);                  /* +-inf */
        return (uint16_t)(sign | 0x7e00u | (frac32 >> 13));     /* quiet NaN */
    }
    if (exp32 == 0)
        return sign; /* zero or binary32 subnormal: |x| < 2^-126, far below 2^-25 */

    /* |x| = sig * 2^(e - 23) with a 24-bit integer significand. */
    int e = (int)exp32 - 127;
    uint32_t sig = frac32 | 0x800000u;

    if (e > 15)
        return (uint16_t)(sign | 0x7c00u); /* |x| >= 2^16: beyond every finite */

    /* The binary16 result is an integer multiple m of the quantum 2^(te-10),
     * where te = max(e, -14) is the exponent of the binade it lands in
     * (-14 for the subnormal range).  m = sig / 2^shift rounded to nearest,
     * ties to even. */
    int te = e > -14 ? e : -14;
    int shift = 13 + (te - e);
    if (shift > 25)
        return sign; /* e < -26: |x| < 2^-26, under half the smallest subnormal */

    uint32_t m = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (m & 1u)))
        m += 1u;

    /* Encode m * 2^(te-10).  For te > -14 (normal), m is in [1024, 2048]: the
     * exponent field is te+15 and the fraction m-1024, and m == 2048 (carry
     * out of the fraction) is the first value of the next binade.  For te ==
     * -14, m < 1024 is a subnormal fraction and m == 1024 is 2^-14, the
     * smallest normal.  Both cases are the single sum below. */
    uint32_t enc = ((uint32_t)(te + 14) << 10) + m;
    if (enc >= 0x7c00u)
        return (uint16_t)(sign | 0x7c00u); /* rounded past 65504: overflow */
    return (uint16_t)(sign | enc);
}

float orc_widen16(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t exp16 = (h >> 10) & 0x1fu;
    uint32_t frac16 = h & 0x3ffu;

    if (exp16 == 0x1fu) /* inf / NaN: keep the payload */
        return float_of(sign | 0x7f800000u | (frac16 << 13));
    if (exp16 == 0) {
        /* subnormal (or zero): frac16 * 2^-24, exact in binary32 */
        float mag = ldexpf((float)frac16, -24);
        return sign ? -mag : mag;
    }
    return float_of(sign | ((exp16 - 15u + 127u) << 23) | (frac16 << 13));
}

void orc_rne16_array(const float* x, uint16_t* out, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = orc_rne16(x[i]);
}

void orc_widen16_array(const uint16_t* h, float* out, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = orc_widen16(h[i]);
}

/* ------------------------------------------------------------------------ */
/* The step.                                                                 */
/* ------------------------------------------------------------------------ */

/* Step 5, "Gradient unscaling": g_true = g_scaled / S, taken here as the
 * binary32 product with the binary32 reciprocal 1/S (identical to a division
 * whenever S is a power of two). */
static float unscale(uint16_t g16, float inv_scale)
{
    return orc_widen16(g16) * inv_scale;
}

void orc_check(const uint16_t* const* grads, const int64_t* sizes, int32_t n,
               float inv_scale, orc_result* r)
{
    int32_t found = 0;
    uint64_t nz = 0, ns = 0, nf = 0;
    uint16_t max_mag = 0;
    double sumsq = 0.0;

    memset(r->exp_hist, 0, sizeof r->exp_hist);
    for (int32_t i = 0; i < n; ++i) {
        for (int64_t j = 0; j < sizes[i]; ++j) {
            uint16_t h = grads[i][j];
            uint16_t mag = (uint16_t)(h & 0x7fffu);
            r->exp_hist[mag >> 10] += 1;   /* binade of the scaled gradient */
            /* Step 6, "Overflow detection": any +-inf or NaN (exponent field
             * all ones) anywhere in the list. */
            if (mag >= 0x7c00u) {
                nf += 1;
                found = 1;
                continue;
            }
            if (mag == 0)
                nz += 1;
            else if (mag < 0x0400u)
                ns += 1;
            if (mag > max_mag)   /* bit patterns of magnitudes order like values */
                max_mag = mag;
            /* Global L2 norm of the unscaled gradients: every square of a
             * binary32 value is exact in binary64; the sum is binary64. */
            double x = (double)unscale(h, inv_scale);
            sumsq = sumsq + x * x;
        }
    }
    r->found_inf = found;
    r->n_zero = nz;
    r->n_subnormal = ns;
    r->n_nonfinite = nf;
    r->sumsq = sumsq;
    r->max_mag16 = max_mag;
    r->max_abs = unscale(max_mag, inv_scale);
}

void orc_clip_coef(orc_result* r, float clip)
{
    r->clipped = 0;
    r->clip_coef = 1.0f;
    if (r->found_inf) {
        r->norm = INFINITY;
        return;
    }
    r->norm = sqrt(r->sumsq);
    /* "Summary of Design Choices": clipping acts on the unscaled gradients,
     * so the threshold means what it means in FP32 training.  Global L2:
     * scale every gradient by clip/norm when the norm exceeds clip. */
    if (clip > 0.0f && r->norm > (double)clip) {
        r->clipped = 1;
        r->clip_coef = (float)((double)clip / r->norm);
    }
}

uint64_t orc_update(int64_t count, const uint16_t* g16, float* w, float* v,
                    uint16_t* w16, float inv_scale, int32_t clipped, float coef,
                    float lr, float momentum, float weight_decay, float eps,
                    uint32_t flags)
{
    uint64_t stale = 0;
    for (int64_t j = 0; j < count; ++j) {
        float g = unscale(g16[j], inv_scale);          /* Step 5 */
        if (clipped)
            g = g * coef;                              /* global-L2 clip */

        /* Without a master copy the FP16 weight itself is the operand. */
        float w_old = (flags & ORC_NO_MASTER) ? orc_widen16(w16[j]) : w[j];

        float t = weight_decay * w_old;                /* g_eff = g + lambda*w */
        float d = g + t;
        float vn, step;
        if (flags & ORC_ADAGRAD) {
            /* Adagrad: the state is the running sum of squared gradients,
             * h = h + d^2, and the step is d / (sqrt(h) + eps). */
            float sq = d * d;
            vn = v[j] + sq;
            float den = sqrtf(vn) + eps;
            step = d / den;
        } else {
            float u = momentum * v[j];                 /* v_t = mu*v_{t-1} + g */
            vn = u + d;
            step = vn;
            if (flags & ORC_NESTEROV) {
                /* Nesterov momentum: step along d + mu * v_t */
                float m2 = momentum * vn;
                step = d + m2;
            }
        }
        float s = lr * step;                           /* w = w - eta*v_t      */
        float wn = w_old - s;

        v[j] = vn;
        uint16_t h_new = orc_rne16(wn);                /* Step 1: FP16 copy    */
        if (!(flags & ORC_NO_MASTER)) {
            if (wn != w_old && h_new == orc_rne16(w_old))
                stale += 1;
            w[j] = wn;
        }
        w16[j] = h_new;
    }
    return stale;
}

float orc_scaler_next(const orc_scaler_cfg* cfg, int32_t found_inf, float max_abs,
                      float scale, int32_t* clean_run)
{
    /* Method 3 of "Choosing the Loss Scaling Factor" and the tutorial's
     * dynamic rule: on overflow skip and multiply S by beta; after N
     * consecutive clean steps multiply S by alpha.  N = 0 keeps S constant
     * except for the backoff. */
    if (found_inf) {
        float s = scale * cfg->backoff;
        *clean_run = 0;
        return s < cfg->min_scale ? cfg->min_scale : s;
    }
    *clean_run += 1;
    if (cfg->mode == ORC_SCALER_DIRECT) {
        /* Method 2 with this step's own statistics standing in for those of
         * an FP32 run; no information (all gradients zero) keeps S. */
        float s = orc_direct_scale(max_abs, cfg->direct_margin, cfg->min_scale, cfg->max_scale);
        return s > 0.0f ? s : scale;
    }
    if (cfg->growth_interval > 0 && *clean_run >= cfg->growth_interval) {
        float s = scale * cfg->growth;
        *clean_run = 0;
        return s > cfg->max_scale ? cfg->max_scale : s;
    }
    return scale;
}

float orc_direct_scale(float max_abs, float margin, float min_scale, float max_scale)
{
    if (!(max_abs > 0.0f))
        return 0.0f;
    /* 65504 is the largest binary16 value; the margin leaves headroom for
     * the next step's gradients to be larger than this one's. */
    float s = (float)(65504.0 / ((double)margin * (double)max_abs));
    if (s < min_scale)
        s = min_scale;
    if (s > max_scale)
        s = max_scale;
    return s;
}

void orc_step(const uint16_t* const* grads, float* const* master,
              float* const* momentum, uint16_t* const* w16, const int64_t* sizes,
              int32_t n, float scale, float lr, float momentum_coef,
              float weight_decay, float clip, float eps, const orc_scaler_cfg* cfg,
              int32_t* clean_run, uint32_t flags, orc_result* r)
{
    float inv_scale = 1.0f / scale;

    memset(r, 0, sizeof *r);
    orc_check(grads, sizes, n, inv_scale, r);
    orc_clip_coef(r, clip);

    /* Step 6: on overflow the update is skipped and the weights, the
     * momentum and the FP16 copy are left exactly as they were. */
    if (!r->found_inf) {
        for (int32_t i = 0; i < n; ++i)
            r->n_stale += orc_update(sizes[i], grads[i], master ? master[i] : NULL,
                                     momentum[i], w16[i], inv_scale, r->clipped,
                                     r->clip_coef, lr, momentum_coef,
                                     weight_decay, eps, flags);
    }
    r->new_scale = orc_scaler_next(cfg, r->found_inf, r->max_abs, scale, clean_run);
    r->new_clean_run = *clean_run;
}
