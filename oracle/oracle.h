/*
 * oracle.h -- plain, single-threaded CPU oracle of the loss-scaled FP32-master
 * SGD-momentum step of mixed-precision training.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or execute this code: only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark do.  It shares no source with the CUDA
 * library (no common header, helper, table or constant) and it is written to
 * be read against the pages, not to be fast.
 *
 * Sources (page title, then the section it follows):
 *   [A] "Mixed Precision Training" -- paper-graph-ui.vercel.app analysis,
 *       section 3.4 "Detailed, Sentence-Based Technical Breakdown":
 *         "FP32 Master Copy of Weights"                   (A1, A2)
 *         "Loss Scaling" -- the unscaling step and
 *                           "Overflow detection and handling" (A4, A5, A6)
 *         "The Integrated Training Procedure (Figure 1)",
 *                           Steps 1, 5, 6, 7               (A2, A4-A6, A9)
 *         "A subtle interaction: weight decay"             (A8)
 *         "Choosing the Loss Scaling Factor", Method 3     (A13)
 *         "Summary of Design Choices"                      (clip after unscale)
 *   [T] "Mixed Precision Training" -- azimuth.plus tutorial, section
 *       "Loss scaling: why gradients vanish in FP16" (dynamic scaling rule)
 *   [R] "Mixed-precision training ..." -- worldresearchstate.com record,
 *       "Scientific scope" (gradients unscaled before updates or clipping)
 *
 * Arithmetic: IEEE-754 binary32 with round-to-nearest-even for every
 * separately written operation (built with -ffp-contract=off, no fast-math,
 * x86-64 SSE scalar arithmetic), binary64 for the sum of squares and the
 * norm, and this file's own binary16 codec.
 *
 * Every function here is pinned by a CPU test to facts fixed outside the
 * oracle (IEEE-754, library conversions, closed forms, the pages' worked
 * numbers); none is marked "parity unpinned".
 */
#ifndef LSF32_ORACLE_H
#define LSF32_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- binary16 codec (IEEE-754 definition) ------------------------------ */

/* binary32 -> binary16, round to nearest, ties to even; |x| >= 65520 -> inf;
 * NaN stays NaN (quiet bit set, top payload bits kept). */
uint16_t orc_rne16(float x);
/* binary16 -> binary32, exact for every one of the 2^16 patterns. */
float orc_widen16(uint16_t h);
void orc_rne16_array(const float* x, uint16_t* out, size_t n);
void orc_widen16_array(const uint16_t* h, float* out, size_t n);

/* ---- step ---------------------------------------------------------------- */

typedef struct {
    float backoff;           /* beta, applied on overflow (e.g. 0.5)          */
    float growth;            /* alpha, applied after N clean steps (e.g. 2)   */
    int32_t growth_interval; /* N; 0 = never grow (constant S)               */
    float min_scale;         /* floor on S after a backoff                    */
    float max_scale;         /* ceiling on S after a growth                   */
    int32_t mode;            /* ORC_SCALER_DYNAMIC or ORC_SCALER_DIRECT       */
    float direct_margin;     /* direct mode: S = 65504 / (margin * max|g|)    */
} orc_scaler_cfg;

#define ORC_SCALER_DYNAMIC 0 /* Method 3: backoff on overflow, growth after N */
#define ORC_SCALER_DIRECT 1  /* Method 2 from each step's own max|g|; backoff
                                on overflow                                   */

typedef struct {
    int32_t found_inf;   /* any +-inf/NaN anywhere in the list                */
    int32_t clipped;     /* 1 when clip > 0 and norm > clip                   */
    double sumsq;        /* sum of squares of the unscaled gradients          */
    double norm;         /* sqrt(sumsq); +inf when found_inf                  */
    float clip_coef;     /* clip / norm when clipped, else 1                  */
    uint64_t n_zero;     /* gradients equal to +-0                            */
    uint64_t n_subnormal;/* 0 < |g16| < 2^-14                                 */
    uint64_t n_nonfinite;/* +-inf or NaN                                      */
    uint64_t n_stale;    /* master moved but its FP16 copy did not            */
    float new_scale;     /* S for the next step                               */
    int32_t new_clean_run;
    /* gradient statistics of pass 1 (the same read): */
    uint16_t max_mag16;  /* largest |g16| bit pattern among finite gradients  */
    float max_abs;       /* its unscaled value, fp32(max|g16|) * (1/S)        */
    uint64_t exp_hist[32];/* count of gradients per binary16 exponent field  */
} orc_result;

/* Ablation mode of the test suite: update the FP16 weights directly, with no
 * FP32 master copy (the configuration the pages compare against). */
#define ORC_NO_MASTER 1u

/* Optimizer of the update (default: SGD with momentum, Step 7 of "The
 * Integrated Training Procedure (Figure 1)").  The pages' speech models used
 * Nesterov SGD and the bigLSTM Adagrad (section 5 of the analysis, model
 * descriptions); neither formula is printed there, so these are the standard
 * forms, each operation rounded to binary32:
 *   Nesterov: v = mu*v + d;  w = w - eta*(d + mu*v)
 *   Adagrad:  h = h + d*d;   w = w - eta*d/(sqrt(h) + eps)   (h in the
 *             momentum array, h0 = 0) */
#define ORC_NESTEROV 2u
#define ORC_ADAGRAD 4u

/* Pass 1 (Steps 5-6): overflow check, range counts and the sum of squares of
 * fp32(g16) * inv_scale over every tensor of the list, in list order. */
void orc_check(const uint16_t* const* grads, const int64_t* sizes, int32_t n,
               float inv_scale, orc_result* r);

/* norm = sqrt(sumsq); clip coefficient of the global-L2 clip. */
void orc_clip_coef(orc_result* r, float clip);

/* Pass 2 (Step 7) over one tensor (or any gathered set of elements): unscale,
 * clip, weight decay, momentum, master update, FP16 copy.  Returns the number
 * of "stale" elements (master moved, FP16 copy did not). */
uint64_t orc_update(int64_t count, const uint16_t* g16, float* w, float* v,
                    uint16_t* w16, float inv_scale, int32_t clipped, float coef,
                    float lr, float momentum, float weight_decay, float eps,
                    uint32_t flags);

/* Loss-scale state machine; returns the next S and updates *clean_run.
 * max_abs (the step's largest unscaled finite |g|) is used by direct mode. */
float orc_scaler_next(const orc_scaler_cfg* cfg, int32_t found_inf, float max_abs,
                      float scale, int32_t* clean_run);

/* Direct choice of S from gradient statistics ("Choosing the Loss Scaling
 * Factor", Method 2): S = 65504 / (margin * max|g|), in binary64, rounded to
 * binary32 and clamped to [min_scale, max_scale]; max_abs == 0 gives 0 (no
 * information: the caller keeps its S). */
float orc_direct_scale(float max_abs, float margin, float min_scale, float max_scale);

/* One whole step over a list of n tensors.  master/momentum/w16 are updated in
 * place unless the step overflows; r receives every output scalar. */
void orc_step(const uint16_t* const* grads, float* const* master,
              float* const* momentum, uint16_t* const* w16, const int64_t* sizes,
              int32_t n, float scale, float lr, float momentum_coef,
              float weight_decay, float clip, float eps, const orc_scaler_cfg* cfg,
              int32_t* clean_run, uint32_t flags, orc_result* r);

#ifdef __cplusplus
}
#endif
#endif
