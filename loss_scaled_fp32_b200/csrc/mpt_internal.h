// mpt_internal.h -- work tables and the device control block of libmpt,
// shared by the host side (mpt.cu) and the kernels (mpt_kernels.cuh).
#pragma once

#include <stdint.h>

namespace mpt {

constexpr int kThreads = 256;              // threads per CTA of every kernel
constexpr int kWarps = kThreads / 32;
constexpr int kArenaAlign = 16;            // elements: 64 B FP32, 32 B FP16
constexpr int kDefaultCheckChunk = 65536;  // elements per check-pass bin
constexpr int kDefaultUpdateChunk = 4096;  // elements per update-pass bin
constexpr int kChunkQuantum = 2048;        // chunk sizes are multiples of this
constexpr int kMaxChunk = 1 << 20;
constexpr int kSmallTensor = 1024;         // tensors up to this size are packed
constexpr int kPackedMaxElems = 4096;      // elements per packed bin
constexpr int kMaxPackedSegs = 256;        // tensors per packed bin
constexpr int kFinishGroup = 64;           // check bins per first-level finish group
static_assert(kFinishGroup <= kThreads, "one thread per bin of a finish group");
constexpr int kOneLevelBins = 8 * kThreads; // up to this many check bins: one-level finish

enum BinKind : int32_t {
    kChunkBin = 0,   // one contiguous range of one tensor (vectorised)
    kPackedBin = 1,  // several whole small tensors (flattened, scalar)
};

// One whole small tensor inside a packed bin.
struct __align__(16) Seg {
    int64_t tensor_begin;  // first element, counted inside the tensor (0)
    int64_t arena_begin;   // the same element's index in the three arenas
    int32_t tensor;        // index into the gradient-pointer table
    int32_t len;           // elements
    int32_t local_begin;   // offset of this tensor inside its bin
    int32_t pad;
};

// The work of one CTA.  A chunk bin carries its range inline (one dependent
// load less before the first gradient load); a packed bin points at n_segs
// consecutive Seg entries.
struct __align__(16) Bin {
    int64_t tensor_begin;  // chunk bin: first element of the range in its tensor
    int64_t arena_begin;   // chunk bin: that element's index in the arenas
    int32_t tensor;        // chunk bin: tensor index; packed bin: first Seg index
    int32_t n_elems;       // elements in the bin
    int32_t n_segs;        // packed bin: number of tensors; chunk bin: 0
    int32_t kind;
};

// Per-tensor bounds, read by checked mode only.
struct __align__(16) TensorInfo {
    int64_t size;
    int64_t arena_off;
};

// Device control block.  The check kernel accumulates into the *_acc fields;
// CTA 0 of the update kernel turns them (in a sharded step: the ranks'
// records, which the check kernel's last CTA drew from them) into the step
// result and clears them for the next step.  The two
// kernels' atomic accumulators and the fields that every CTA reads when it
// starts (S, 1/S, the skip flag, the clip coefficient) sit on three separate
// 128-byte lines, so that a CTA's first read never queues behind the other
// CTAs' atomics on the same line.
struct __align__(128) Ctrl {
    // line 0: check-kernel accumulators
    unsigned long long nonfinite_acc;
    unsigned int ticket;
    unsigned int error_acc;
    unsigned int max_mag_acc;  // statistics mode: largest finite |g16| (atomicMax)
    unsigned int pad0a;
    unsigned long long zero_acc;       // FP16 gradients equal to +-0
    unsigned long long subnormal_acc;  // FP16 gradients with 0 < |g16| < 2^-14
    unsigned int pad0[22];
    // line 1: update-kernel accumulators and its work counter (before each
    // update CTA 0 of the check kernel zeroes the counter and moves the last
    // update's stale count into stale_total)
    unsigned long long stale_acc;
    unsigned int upd_next;     // update bins claimed beyond each CTA's first
    unsigned int pad1[29];
    // line 2: step result, written by CTA 0 of the update kernel (on an
    // overflow step of a whole step sumsq is NaN: the check kernel marks a
    // bin with an inf/NaN gradient that way)
    double sumsq;
    double norm;
    unsigned long long n_nonfinite;
    int32_t found_inf;
    int32_t clipped;
    float coef;
    unsigned int error;    // checked-mode error bits of both kernels
    float inv_scale;       // binary32 1/S of this step (read by the update)
    float scale_used;      // S of this step
    // loss-scale state, advanced by CTA 0 of the update kernel
    float scale;           // S for the next step
    int32_t clean_run;     // consecutive clean steps so far
    unsigned long long steps_total;
    unsigned long long skipped_total;
    // gradient statistics (statistics mode): the last step's largest finite
    // |g16| pattern and its unscaled value, fp32(max|g16|) * (1/S)
    unsigned int max_mag;
    float max_abs;
    // what the next check pass needs from `scale`, computed once when the
    // state is set (1/S and, for S = 2^e with -15 <= e <= 100, 2^(-2e))
    int32_t next_pow2;
    unsigned int pad2;
    double next_sq_unscale;
    float next_inv;
    unsigned int pad3;
    // range counts of this step's gradients (from the check pass)
    unsigned long long n_zero;
    unsigned long long n_subnormal;
    // stale counts of every update before the last one (the last update's
    // count is still in stale_acc)
    unsigned long long stale_total;
};

// What one rank's check pass contributes to a sharded step (32 bytes): its
// shard's sum of squares, non-finite count and largest finite magnitude.
// Every rank gathers all ranks' records and adds them in rank order.
struct __align__(16) Partial {
    double sumsq;
    unsigned long long n_nonfinite;
    unsigned int max_mag;
    unsigned int error;
    unsigned int pad[2];
};

// Histogram of binary16 exponent fields (statistics mode).
struct __align__(16) StatsBlock {
    unsigned long long hist_acc[32];  // accumulated by the check CTAs
    unsigned long long hist[32];      // the last step's
};

enum Optimizer : int32_t {
    kOptMomentum = 0,  // SGD with momentum (the pages' Step 7)
    kOptNesterov = 1,  // Nesterov momentum
    kOptAdagrad = 2,   // Adagrad (momentum arena holds the sum of squares)
};

enum ScalerMode : int32_t {
    kScalerDynamic = 0,  // backoff on overflow, growth after N clean steps
    kScalerDirect = 1,   // S = 65504 / (margin * max|g|) of each clean step
};

enum ErrorBits : unsigned int {
    kErrBadBin = 1u,
    kErrBadSeg = 2u,
};

}  // namespace mpt
