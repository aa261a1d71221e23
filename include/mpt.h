/*
 * mpt.h -- libmpt: the loss-scaled FP32-master SGD-momentum optimizer step of
 * mixed-precision training, on one NVIDIA B200 (sm_100a).
 *
 * What one step computes (Micikevicius et al., "Mixed Precision Training",
 * as explained by the paper-graph-ui.vercel.app analysis, section 3.4,
 * "The Integrated Training Procedure (Figure 1)", Steps 5-7, and the
 * azimuth.plus tutorial, "Loss scaling: why gradients vanish in FP16"):
 *
 *   given FP16 weight gradients g16 of a list of tensors, computed from a loss
 *   multiplied by S, and per-parameter FP32 state (master w, momentum v):
 *     1. found_inf = any g16 is +-inf or NaN, over the whole list   (Step 6)
 *     2. g   = fp32(g16) * (1/S)                                     (Step 5)
 *     3. norm = sqrt(sum g^2) over the whole list (binary64);
 *        if clip > 0 and norm > clip: g = g * (clip / norm)  (global-L2 clip,
 *        after unscaling: "Summary of Design Choices")
 *     4. if found_inf: leave w, v and the FP16 copy untouched, S = S*beta
 *                                                   (Step 6, Method 3)
 *        else, per element, every operation rounded to binary32:
 *          d = g + lambda*w        ("A subtle interaction: weight decay")
 *          v = mu*v + d            (Step 7)
 *          w = w - eta*v           (Step 7)
 *          w16 = round_to_nearest_even_fp16(w)   (Step 1 of the next pass)
 *     5. after N consecutive clean steps, S = S*alpha (dynamic scaling,
 *        "Choosing the Loss Scaling Factor", Method 3)
 *
 * Conventions for every call:
 *   - Every function returns an int status: MPT_OK (0) or a negative
 *     MPT_ERR_* code.  No call aborts, throws, traps or prints.
 *   - A handle is used by one host thread at a time.
 *   - "device pointer" means memory of the CUDA device that is current when
 *     mpt_create is called; every later call must run with that device current.
 *   - cuda_stream arguments are cudaStream_t values passed as void*; NULL is
 *     the legacy default stream.
 *   - After MPT_ERR_CUDA the handle is broken: every later call except
 *     mpt_stats, mpt_error_string and mpt_destroy returns MPT_ERR_BROKEN.
 */
#ifndef LIBMPT_MPT_H
#define LIBMPT_MPT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define MPT_OK 0
#define MPT_ERR_INVALID_ARG (-1)  /* null or odd pointer, n <= 0, size <= 0,
                                     S not finite or <= 0, lr / momentum /
                                     weight decay / clip not finite          */
#define MPT_ERR_WORKSPACE (-2)    /* workspace too small, not 256-B aligned,
                                     or not device memory of this device    */
#define MPT_ERR_CUDA (-3)         /* a CUDA runtime call failed             */
#define MPT_ERR_DEVICE_CHECK (-4) /* checked mode found a work-table entry out
                                     of bounds; that entry was not touched   */
#define MPT_ERR_BROKEN (-5)       /* the handle saw MPT_ERR_CUDA earlier     */
#define MPT_ERR_TOO_LARGE (-6)    /* input longer than MPT_NOALLOC_MAX_ELEMS
                                     (mpt_check_flat_noalloc only)           */

/* ---- configuration ------------------------------------------------------ */
#define MPT_FLAG_CHECKED 0x1u     /* kernels validate every work-table entry
                                     against the tensor sizes and arenas     */
#define MPT_FLAG_COUNT_STALE 0x2u /* count elements whose master moved but
                                     whose FP16 copy did not                 */
#define MPT_FLAG_GRAD_STATS 0x4u  /* the check pass also finds the largest
                                     |g16| and counts the gradients per
                                     binary16 exponent field (see
                                     mpt_grad_histogram); implied by
                                     MPT_SCALER_DIRECT                      */

/* Loss-scale modes ("Choosing the Loss Scaling Factor").  Both skip the
 * update and multiply S by backoff on overflow.
 *   DYNAMIC (Method 3): after growth_interval consecutive clean steps,
 *     multiply S by growth.
 *   DIRECT (Method 2): after every clean step set S = 65504 / (margin *
 *     max|g|), max|g| being that step's largest unscaled finite gradient
 *     (binary64, rounded to binary32, clamped to [min_scale, max_scale]);
 *     a step whose gradients are all zero keeps S. */
#define MPT_SCALER_DYNAMIC 0
#define MPT_SCALER_DIRECT 1

/* Update rule of the FP32 master (every operation rounded to binary32; d is
 * the unscaled, clipped gradient plus weight decay, d = g + lambda*w):
 *   MOMENTUM (default; Step 7): v = mu*v + d;  w = w - eta*v
 *   NESTEROV (the pages' speech models): v = mu*v + d;  w = w - eta*(d + mu*v)
 *   ADAGRAD (the pages' bigLSTM): v = v + d*d;  w = w - eta*d/(sqrt(v) + eps)
 *     -- the momentum arena holds the running sum of squares (zero at
 *     creation) and the momentum argument of the step is ignored. */
#define MPT_OPT_MOMENTUM 0
#define MPT_OPT_NESTEROV 1
#define MPT_OPT_ADAGRAD 2

typedef struct {
    float backoff;            /* beta: S multiplier on overflow (default 0.5)      */
    float growth;             /* alpha: S multiplier after N clean steps (2.0)     */
    int32_t growth_interval;  /* N; 0 = constant S (an overflow still backs off) */
    float min_scale;          /* lower bound of S after a backoff (2^-24)          */
    float max_scale;          /* upper bound of S after a growth (2^24)            */
    uint32_t flags;           /* MPT_FLAG_* (default 0)                            */
    int32_t check_chunk_elems;  /* elements per work bin (one CTA) of the check
                                   pass: a multiple of 2048 in [2048, 2^20];
                                   0 = default: 65536, halved down to 2048
                                   while the list gives fewer than 592 bins */
    int32_t scaler_mode;      /* MPT_SCALER_DYNAMIC (default) or _DIRECT           */
    float direct_margin;      /* direct mode: margin > 0 (default 2: one bit of
                                 headroom, as the pages suggest)                   */
    int32_t optimizer;        /* MPT_OPT_MOMENTUM (default), _NESTEROV, _ADAGRAD   */
    float eps;                /* Adagrad denominator term (default 1e-10)          */
    int32_t update_chunk_elems; /* the same for the update pass; 0 = default
                                   (4096)                                         */
} mpt_config;

/* ---- results ------------------------------------------------------------ */
typedef struct {
    int32_t found_inf;     /* 1: some gradient was +-inf/NaN; the update was
                              skipped and the state is bitwise unchanged        */
    int32_t clipped;       /* 1: clip > 0 and grad_norm > clip                  */
    float new_scale;       /* S to use for the next step                        */
    int32_t clean_run;     /* consecutive clean steps after this one            */
    double grad_norm;      /* global L2 norm of the unscaled, unclipped
                              gradients; +inf when found_inf                    */
    float clip_coef;       /* clip / grad_norm when clipped, else 1             */
    float max_abs_grad;    /* MPT_FLAG_GRAD_STATS / direct mode, else 0: the
                              largest unscaled finite |g|, fp32(max|g16|)*(1/S) */
    uint64_t n_zero;       /* FP16 gradients equal to +-0 (counted by the check
                              pass, so overflow steps report them too)         */
    uint64_t n_subnormal;  /* FP16 gradients with 0 < |g16| < 2^-14             */
    uint64_t n_nonfinite;  /* FP16 gradients that are +-inf or NaN              */
    uint64_t n_fp16_stale; /* MPT_FLAG_COUNT_STALE only, else 0: elements whose
                              master changed while the rounded copy did not     */
} mpt_step_result;

typedef struct {
    uint64_t steps;           /* steps completed on the device                  */
    uint64_t skipped;         /* of which were skipped on overflow              */
    float scale;              /* current S (last new_scale, or the value set)   */
    int32_t clean_run;        /* current clean-step counter                     */
    mpt_step_result last;     /* result of the last completed step              */
    uint64_t n_fp16_stale_total; /* MPT_FLAG_COUNT_STALE: n_fp16_stale summed
                              over every step since creation, queued ones
                              included (summed on the device)                 */
    uint64_t timed_steps;     /* steps timed while mpt_set_timing was on        */
    double check_ms_total;    /* summed CUDA-event durations of the check       */
    double update_ms_total;   /* kernel and of the update kernel over them      */
} mpt_stats_t;

typedef struct mpt_handle mpt_handle;  /* opaque */

/* ---- calls -------------------------------------------------------------- */

/* Fill *cfg with the defaults listed in mpt_config.
 * Errors: MPT_ERR_INVALID_ARG (cfg NULL). */
int mpt_config_init(mpt_config* cfg);

/* Bytes of device workspace mpt_create needs for n tensors with the given
 * element counts (host array sizes[n]); cfg NULL = defaults.  The workspace
 * holds the FP32 master arena, the FP32 momentum arena and the FP16
 * working-copy arena (each tensor at a 16-element-aligned offset) plus the
 * work tables and a small control block.
 * Errors: MPT_ERR_INVALID_ARG (a pointer NULL, n <= 0, a size <= 0, bad cfg). */
int mpt_workspace_bytes(const int64_t* sizes, int32_t n, const mpt_config* cfg,
                        size_t* bytes);

/* Create a handle over a caller-owned device workspace d_workspace of
 * ws_bytes bytes (256-byte aligned, at least mpt_workspace_bytes).  Builds and
 * uploads the work tables and zeroes the three arenas and the control block,
 * synchronously.  The caller then writes the initial master weights through
 * mpt_tensor_views and calls mpt_refresh_half.  The workspace and the
 * gradient buffers belong to the caller and must outlive the handle; the
 * library owns only host tables and two small pinned host buffers.  The loss
 * scale starts at 1 with a clean-step counter of 0 (mpt_set_scaler_state).
 * Errors: MPT_ERR_INVALID_ARG, MPT_ERR_WORKSPACE, MPT_ERR_CUDA. */
int mpt_create(const int64_t* sizes, int32_t n, const mpt_config* cfg,
               void* d_workspace, size_t ws_bytes, mpt_handle** out);

/* Device pointers to tensor i's slices of the arenas: FP32 master, FP32
 * momentum and FP16 working copy (binary16, sizes[i] elements each, 64-byte
 * aligned).  Any output pointer may be NULL.
 * Errors: MPT_ERR_INVALID_ARG (h NULL, i out of range). */
int mpt_tensor_views(const mpt_handle* h, int32_t i, float** master,
                     float** momentum, void** w16_half);

/* Rewrite every FP16 working copy from its FP32 master: w16 = RNE_fp16(w)
 * (Step 1 of the training iteration).  Asynchronous on cuda_stream.
 * Errors: MPT_ERR_INVALID_ARG, MPT_ERR_CUDA, MPT_ERR_BROKEN. */
int mpt_refresh_half(mpt_handle* h, void* cuda_stream);

/* The loss-scale state (S and the clean-step counter) lives in the
 * workspace and is advanced on the device by every step, so steps can be
 * queued without the host waiting; the handle keeps a host mirror that every
 * waiting call (mpt_step, mpt_wait, mpt_set_scaler_state) refreshes. */

/* One optimizer step.  d_grads_half is a HOST array of n DEVICE pointers, the
 * FP16 (binary16) gradients of the n tensors, computed from a loss multiplied
 * by `scale` (any 2-byte alignment; contents are only read).  lr, momentum
 * and weight_decay are eta, mu and lambda; clip <= 0 disables clipping.
 * Work is queued on cuda_stream and the call waits for it (it reads the
 * 384-byte control block back).  The scale state advances from `scale`:
 * out->new_scale is the S for the next step.  On overflow the arenas are
 * untouched.  Errors: MPT_ERR_INVALID_ARG, MPT_ERR_CUDA,
 * MPT_ERR_DEVICE_CHECK (checked mode; the bins that passed their check were
 * updated), MPT_ERR_BROKEN; on an argument error nothing is queued. */
int mpt_step(mpt_handle* h, const void* const* d_grads_half, float scale,
             float lr, float momentum, float weight_decay, float clip,
             void* cuda_stream, mpt_step_result* out);

/* The same step, queued on cuda_stream without waiting: S is the device
 * scale state (see mpt_device_scale), the gradients must have been computed
 * from a loss multiplied by that device value, and the step advances the
 * state on the device.  Nothing is read back; call mpt_wait for the result
 * of the last queued step.  The gradient buffers must stay unchanged until
 * the queued work has run.
 * Gradient-pointer tables: the handle keeps device copies of the last four
 * distinct tables passed to its steps (in its workspace).  A step whose
 * d_grads_half equals one of them queues exactly the two kernel launches (no
 * copy, no host synchronisation); a new table is copied from pinned host
 * memory into the least recently used copy first, ordered on the step's
 * stream after the steps queued before it.  So queue a handle's steps on one
 * stream (or order its streams yourself).
 * CUDA graphs: a step whose table is already held queues only the two
 * kernel launches, so it can be captured into a CUDA graph (kernel timing
 * off); capture only after a first, uncaptured step with the same table (a
 * new table's copy must not be recorded).  Each replay reads the gradients
 * its buffers hold at replay time, the pointer copy that the capture used,
 * and reads and advances the device scale state; mpt_wait on the replay
 * stream returns the replayed step's result.  A later step with a fifth
 * distinct table may rewrite that copy: replay a captured step only while
 * its table is among the last four used.
 * Errors: MPT_ERR_INVALID_ARG, MPT_ERR_CUDA, MPT_ERR_BROKEN. */
int mpt_step_async(mpt_handle* h, const void* const* d_grads_half, float lr,
                   float momentum, float weight_decay, float clip, void* cuda_stream);

/* Wait for the work queued on cuda_stream and return the result of the last
 * step (out may be NULL); refreshes the host mirror of the scale state and
 * the counters.  Errors: MPT_ERR_INVALID_ARG, MPT_ERR_CUDA,
 * MPT_ERR_DEVICE_CHECK, MPT_ERR_BROKEN. */
int mpt_wait(mpt_handle* h, void* cuda_stream, mpt_step_result* out);

/* Device address of the binary32 loss scale S that the next
 * mpt_step_async uses (inside the workspace): a training loop multiplies its
 * loss by it on the device.  Errors: MPT_ERR_INVALID_ARG. */
int mpt_device_scale(const mpt_handle* h, float** d_scale);

/* ---- sharded step (optimizer state split across the ranks of a data-
 * parallel group) ---------------------------------------------------------
 *
 * The flat parameter list (all tensors concatenated, P elements) is cut into
 * `world` equal contiguous shards of mpt_shard_len(P, world) elements (the
 * last one padded with elements whose gradient is always zero).  Rank r
 * creates an ordinary handle over ONE tensor of shard_len elements: it owns
 * the FP32 master, FP32 momentum and FP16 copy of flat elements
 * [r*shard_len, (r+1)*shard_len).  Per step, with the loss scale on the
 * device (as mpt_step_async):
 *   1. the caller reduce-scatters the FP16 gradients so that each rank holds
 *      the summed gradients of its shard (an FP16 sum can itself overflow;
 *      step 2 catches it like any other inf);
 *   2. mpt_step_partial queues the check pass over the shard and returns the
 *      device address of its 32-byte record (MPT_PARTIAL_BYTES: binary64 sum
 *      of squares, non-finite count, largest finite |g16|, error bits);
 *   3. the caller all-gathers the records of all ranks, in rank order, into
 *      one device array (16-byte aligned);
 *   4. mpt_step_finish queues the update of the shard, which first adds the
 *      records in rank order (so every rank gets bit-identical totals and the
 *      same next S) and finishes the step;
 *   5. the caller all-gathers the FP16 copies of the shards.
 * Only 32 bytes per rank cross between the two kernels of a step.  The
 * halves are not timed by mpt_set_timing; mpt_wait returns the last result:
 * found_inf, n_nonfinite, grad_norm, the clip coefficient and the scale are
 * those of the whole list (equal on every rank), n_zero, n_subnormal and the
 * histogram those of this rank's shard. */
#define MPT_PARTIAL_BYTES 32

/* shard_len = ceil(total / world) rounded up to a multiple of 16.
 * Errors: MPT_ERR_INVALID_ARG. */
int mpt_shard_len(int64_t total, int32_t world, int64_t* shard_len);

/* Phase 2: queue the check pass over the handle's gradients (a host array of
 * its tensors' device pointers, as for mpt_step) with S from the device
 * state; *d_partial receives the device address of this rank's record
 * (valid until the next call on the handle).  Errors: MPT_ERR_INVALID_ARG,
 * MPT_ERR_CUDA, MPT_ERR_BROKEN. */
int mpt_step_partial(mpt_handle* h, const void* const* d_grads_half, void* cuda_stream,
                     void** d_partial);

/* Phase 4: d_partials = device array of `world` records in rank order;
 * queues the update over the gradients of the preceding mpt_step_partial,
 * which first adds the records and finishes the step (norm, clip
 * coefficient, loss-scale state).
 * Errors: MPT_ERR_INVALID_ARG (no check pass queued, misaligned records),
 * MPT_ERR_CUDA, MPT_ERR_BROKEN. */
int mpt_step_finish(mpt_handle* h, const void* d_partials, int32_t world, float lr,
                    float momentum, float weight_decay, float clip, void* cuda_stream);

/* Statistics mode: counts[e] = number of gradients of the last step whose
 * binary16 exponent field is e (e = 0: zeros and subnormals; e = 31: inf and
 * NaN; otherwise |g16| in [2^(e-15), 2^(e-14))), as of the last waiting
 * call; all zero without statistics.  Errors: MPT_ERR_INVALID_ARG. */
int mpt_grad_histogram(const mpt_handle* h, uint64_t counts[32]);

/* Counters and the last result, as of the last waiting call.
 * Errors: MPT_ERR_INVALID_ARG. */
int mpt_stats(const mpt_handle* h, mpt_stats_t* out);

/* Read the host mirror of the loss-scale state (as of the last waiting
 * call) / set the state on the device and the host (checkpoint and resume;
 * synchronous, call it with no step in flight).  set requires a finite
 * scale > 0 and clean_run >= 0.  Errors: MPT_ERR_INVALID_ARG, MPT_ERR_CUDA,
 * MPT_ERR_BROKEN. */
int mpt_get_scaler_state(const mpt_handle* h, float* scale, int32_t* clean_run);
int mpt_set_scaler_state(mpt_handle* h, float scale, int32_t clean_run);

/* Time both kernels of every `every`-th following step (the first step
 * queued after the call, then every `every`-th; 1 = every step) with CUDA
 * events recorded on the step's stream before the check kernel, between the
 * two kernels and after the update kernel.  The durations are summed into
 * mpt_stats_t at the next waiting call, or when 256 timed steps are pending.
 * The events cost time of their own (the update of a timed step cannot start
 * early, and three more stream operations sit in each timed step), so a
 * throughput measurement should sample: every = 10 keeps that cost to a
 * tenth.  every = 0 turns timing off (and waits for the pending events).
 * Whole steps only: the halves of a sharded step are not timed.
 * Errors: MPT_ERR_INVALID_ARG (h NULL, every < 0), MPT_ERR_CUDA. */
int mpt_set_timing(mpt_handle* h, int32_t every);

/* Test hook (the pages have no counterpart): the next step of this handle --
 * mpt_step, mpt_step_async, mpt_step_partial or mpt_step_finish -- fails as
 * if its kernel launch had failed: it queues nothing, returns MPT_ERR_CUDA,
 * and the handle becomes unusable (every later call returns MPT_ERR_BROKEN),
 * exactly as after a real CUDA error.  No CUDA call is made and no GPU fault
 * is involved; it exists so that a caller's error path can be tested.
 * Errors: MPT_ERR_INVALID_ARG (h NULL). */
int mpt_debug_fail_next_step(mpt_handle* h);

/* Release the handle's host resources.  The workspace is the caller's and is
 * not freed.  NULL is accepted. */
int mpt_destroy(mpt_handle* h);

/* Static description of a status code (never NULL). */
const char* mpt_error_string(int code);

/* ---- allocation-free check of one flat gradient buffer ------------------ */

/* The paper has no counterpart to this call: it serves callers of this
 * library, not a step of the method.
 *
 * Some callers cannot allocate device memory: a library loaded into a host
 * program whose memory pool already owns the device (a cudaMalloc there
 * fails, or takes memory the host program has counted on), and code whose
 * step loop must never enter the CUDA allocator (cudaMalloc and cudaFree can
 * synchronize the device and stall every stream).  mpt_step needs a
 * workspace allocated up front; this call needs none.  It runs the overflow
 * check and the global norm of the step (found_inf, the L2 norm of the
 * unscaled gradients, the clip coefficient, the count of +-inf/NaN) over ONE
 * contiguous FP16 buffer, keeping its scratch (one binary64 partial per
 * 32768 elements and two counters, about 256 KiB) in a fixed array inside the
 * library that every GPU which loads the library holds until the process
 * exits.
 *
 *   d_grads_half  device pointer to n binary16 gradients (2-byte aligned),
 *                 scaled by `scale`; only read
 *   n             1 <= n <= MPT_NOALLOC_MAX_ELEMS; longer inputs return
 *                 MPT_ERR_TOO_LARGE before any CUDA call
 *   scale, clip   as in mpt_step (clip <= 0: no clipping, coefficient 1)
 *   d_result      device pointer (8-byte aligned) that receives the
 *                 mpt_check_result when the queued work completes
 *   cuda_stream   stream to queue on; the call returns without waiting
 *
 * The first successful call on each device sets that device up, with it
 * current: it looks up the device address of the scratch array and loads the
 * call's kernels (both of its variants, for power-of-two and other S), so no
 * later call loads code.  Make that first call before any stream capture; a
 * set-up that fails (inside a capture, say) returns MPT_ERR_CUDA, keeps
 * nothing, and the next call tries again.  Every call on a device shares the
 * one scratch array, which keeps the last call's contents; each call clears
 * the counters it needs before its kernel runs.  Calls whose work overlaps on
 * the GPU (other streams, other host threads) race on that array and give
 * wrong results: serialize them.  The call checks the status each CUDA call
 * returns; it clears the runtime's last-error state only after a failure of
 * its own, so an error left pending by earlier work stays for the caller.
 * Errors: MPT_ERR_INVALID_ARG, MPT_ERR_TOO_LARGE, MPT_ERR_CUDA. */
#define MPT_NOALLOC_MAX_ELEMS (((int64_t)1) << 30)

typedef struct {
    int32_t found_inf;     /* 1: some gradient was +-inf/NaN                     */
    int32_t clipped;       /* 1: clip > 0 and grad_norm > clip                   */
    double grad_norm;      /* L2 norm of the unscaled gradients; +inf if found   */
    float clip_coef;       /* clip / grad_norm when clipped, else 1              */
    int32_t reserved;
    uint64_t n_nonfinite;  /* gradients that are +-inf or NaN                    */
} mpt_check_result;

int mpt_check_flat_noalloc(const void* d_grads_half, int64_t n, float scale, float clip,
                           mpt_check_result* d_result, void* cuda_stream);

#ifdef __cplusplus
}
#endif
#endif
