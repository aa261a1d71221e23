// mpt_kernels.cuh -- sm_100a kernels of the loss-scaled FP32-master step.
//
//   check_kernel   one pass over the FP16 gradients: overflow check (Step 6 of
//                  "The Integrated Training Procedure (Figure 1)"), sum of
//                  squares of the unscaled gradients (global-L2 clip), zero
//                  and subnormal counts, as per-bin (beyond 2 048 bins
//                  per-group) partial sums
//   update_kernel  adds those partials in a fixed order (every CTA the same
//                  sum; CTA 0 writes the step result and advances the loss
//                  scale), then the fused per-element update (Steps 5 and 7,
//                  weight decay, clip, FP16 copy) over a persistent grid; on
//                  an overflow step every CTA exits after the sum
//   refresh_kernel FP16 copy = round-to-nearest-even(master) (Step 1)
//
// The sharded step's check pass (mpt_step_partial) instead adds its own
// partials by atomic tickets into a 32-byte record; the update kernel then
// adds the ranks' records, in rank order, in place of the partials.
//
// All three are HBM-bound streaming kernels on the CUDA cores: there is no
// contraction, so no tensor-core path.  Per parameter the check reads 2 B and
// the update reads 10 B and writes 10 B.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "mpt_internal.h"

namespace mpt {

// ---------------------------------------------------------------------------
// arguments
// ---------------------------------------------------------------------------

struct Tables {
    const Bin* bins;
    const Seg* segs;
    const TensorInfo* tensors;
    const uint16_t* const* grads;  // device table: one FP16 gradient pointer per tensor
    int32_t nbins;
    int32_t nsegs;
    int32_t ntensors;
    int32_t pad;
    int64_t arena_total;
};

// Loss-scale state machine parameters.
struct ScalerParams {
    float backoff;
    float growth;
    int32_t growth_interval;
    float min_scale;
    float max_scale;
    int32_t mode;           // kScalerDynamic or kScalerDirect
    float direct_margin;    // direct mode: S = 65504 / (margin * max|g|)
};

struct CheckArgs {
    Tables t;
    double* partials;     // one binary64 partial sum of squares per bin
    double* group_partials;        // one per group of kFinishGroup bins
    unsigned int* group_tickets;   // one per group; zero between launches
    Ctrl* ctrl;
    float host_scale;     // S the gradients carry, when given by the host,
    float host_inv;       // with its binary32 reciprocal
    double host_sq_unscale;  // and 2^(-2e) when S = 2^e, -15 <= e <= 100
    int32_t host_pow2;
    int32_t scale_on_device;  // 1: S is ctrl->scale (asynchronous steps)
    StatsBlock* stats;    // statistics mode only
    Partial* partial_out; // sharded step: add the partials into this shard's
                          // 32-byte record here; nullptr (whole step): leave
                          // them to the update kernel
};

struct UpdateArgs {
    Tables t;
    float* master;
    float* momentum;
    uint16_t* w16;
    Ctrl* ctrl;           // check result: skip flag, clip coefficient, 1/S
    float lr;
    float mu;
    float wd;
    float eps;            // Adagrad only
    // What every CTA adds before it updates; CTA 0 then finishes the step.
    // Whole step: the check kernel's partial sums (per bin, or per group of
    // kFinishGroup bins beyond kOneLevelBins bins).  Sharded step: the
    // ranks' 32-byte records, in rank order.  Exactly one is set.
    const double* fin_partials;
    int32_t fin_n;
    const Partial* fin_records;
    int32_t fin_world;
    int32_t stats_level;  // kNoStats, kMaxOnly or kMaxHist
    float clip;
    ScalerParams scaler;
    StatsBlock* stats;
};

// What the squares need from S: the binary32 reciprocal 1/S and, when S is a
// power of two 2^e with -15 <= e <= 100, the binary64 constant 2^(-2e) that
// turns a sum of squared scaled gradients into the sum of squared unscaled
// ones.
struct SqParams {
    float inv_scale;
    double sq_unscale;
    bool pow2;
};

__device__ __forceinline__ SqParams sq_params(float S)
{
    SqParams q;
    q.inv_scale = __fdiv_rn(1.0f, S);
    const uint32_t b = __float_as_uint(S);
    const int biased = (int)((b >> 23) & 0xFFu);
    const int e = biased - 127;
    q.pow2 = (b & 0x807FFFFFu) == 0 && biased != 0 && e >= -15 && e <= 100;
    q.sq_unscale = q.pow2 ? __longlong_as_double((long long)(1023 - 2 * e) << 52) : 0.0;
    return q;
}

// Step result and loss-scale state from the step's totals (one thread): the
// norm, the clip coefficient, 1/S for the update, the range counts, the state
// machine, the previous update's stale count added to the running total, and
// the update kernel's counters cleared for this step.
__device__ __forceinline__ void finish_step(Ctrl* c, float S, const SqParams& q,
                                            unsigned long long n_nonfinite, double sumsq,
                                            unsigned int max_mag, bool have_max,
                                            unsigned int err, float clip, const ScalerParams& sp)
{
    const bool found = n_nonfinite != 0;
    const double norm = found ? __longlong_as_double(0x7ff0000000000000ll) : sqrt(sumsq);
    const bool clipped = !found && clip > 0.0f && norm > (double)clip;
    float max_abs = 0.0f;
    if (have_max) {
        c->max_mag = max_mag;
        max_abs = __fmul_rn(__half2float(__ushort_as_half((unsigned short)max_mag)), q.inv_scale);
        c->max_abs = max_abs;
    }
    c->sumsq = sumsq;
    c->norm = norm;
    c->n_nonfinite = n_nonfinite;
    c->found_inf = found ? 1 : 0;
    c->clipped = clipped ? 1 : 0;
    c->coef = clipped ? __double2float_rn((double)clip / norm) : 1.0f;
    // S, 1/S, the cleared error word, the update's bin counter and the stale
    // total were set by the check kernel's CTA 0; the update's own CTAs may
    // be adding error bits right now
    if (err)
        atomicOr(&c->error, err);
    // Loss-scale state machine: on overflow skip and multiply S by beta;
    // dynamic mode: after growth_interval consecutive clean steps multiply S
    // by alpha; direct mode: S = 65504 / (margin * max|g|) of this step
    // (binary64, rounded to binary32; all-zero gradients keep S).
    int32_t clean = c->clean_run;
    float next = S;
    if (found) {
        next = fmaxf(__fmul_rn(S, sp.backoff), sp.min_scale);
        clean = 0;
        c->skipped_total += 1;
    } else {
        clean += 1;
        if (sp.mode == kScalerDirect) {
            if (max_abs > 0.0f) {
                const double d = __ddiv_rn(65504.0, __dmul_rn((double)sp.direct_margin,
                                                              (double)max_abs));
                next = fminf(fmaxf(__double2float_rn(d), sp.min_scale), sp.max_scale);
            }
        } else if (sp.growth_interval > 0 && clean >= sp.growth_interval) {
            next = fminf(__fmul_rn(S, sp.growth), sp.max_scale);
            clean = 0;
        }
    }
    c->scale = next;
    const SqParams nq = sq_params(next);
    c->next_inv = nq.inv_scale;
    c->next_sq_unscale = nq.sq_unscale;
    c->next_pow2 = nq.pow2 ? 1 : 0;
    c->clean_run = clean;
    c->steps_total += 1;
}


// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ bool range_ok(int32_t tensor, int64_t tensor_begin, int64_t arena_begin,
                                         int64_t len, const Tables& t)
{
    if (tensor < 0 || tensor >= t.ntensors || len < 0 || tensor_begin < 0)
        return false;
    const TensorInfo ti = t.tensors[tensor];
    return tensor_begin + len <= ti.size && arena_begin == ti.arena_off + tensor_begin &&
           arena_begin + len <= t.arena_total;
}

// Checked mode: validate a bin (and every tensor of a packed bin) before any
// gradient, master or momentum address is formed from it.
__device__ __forceinline__ bool bin_ok(const Bin& bin, const Tables& t)
{
    if (bin.n_elems < 0)
        return false;
    if (bin.kind == kChunkBin)
        return bin.n_segs == 0 &&
               range_ok(bin.tensor, bin.tensor_begin, bin.arena_begin, bin.n_elems, t);
    if (bin.kind != kPackedBin || bin.tensor < 0 || bin.n_segs < 1 ||
        bin.n_segs > kMaxPackedSegs || bin.n_elems > kPackedMaxElems ||
        bin.tensor + bin.n_segs > t.nsegs)
        return false;
    int32_t expect = 0;
    for (int k = 0; k < bin.n_segs; ++k) {
        const Seg s = t.segs[bin.tensor + k];
        if (s.local_begin != expect || !range_ok(s.tensor, s.tensor_begin, s.arena_begin, s.len, t))
            return false;
        expect += s.len;
    }
    return expect == bin.n_elems;
}

// Index of the range of a packed bin that holds flattened element j: the
// last k with begin[k] <= j (begin[] ascending, begin[0] == 0).
__device__ __forceinline__ int find_seg(const int32_t* begin, int n, int j)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (begin[mid] <= j)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h)
{
    return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// check kernel: overflow flag + sum of squares of the unscaled gradients
// ---------------------------------------------------------------------------

struct SqAcc {
    double a0 = 0.0, a1 = 0.0;

    // Some element this thread saw was +-inf/NaN: the square of an inf or a
    // NaN is inf or NaN and stays so through every later addition, while a
    // sum of finite squares cannot overflow binary64 (each square is at most
    // 65504^2 / min(S, 1)^2).  With S not a power of two a huge 1/S can make
    // the binary32 product of a finite gradient inf; that only sends the CTA
    // through its exact recount, which then finds no non-finite element.
    __device__ __forceinline__ bool saw_nonfinite() const { return !isfinite(a0 + a1); }
};

// Square of one gradient, accumulated in binary64.
//
// Power-of-two S: x = fp32(g16) * (1/S) is exact, and so is the product of a
// binary64 sum with a power of two that stays in range.  So the squares of
// the scaled gradients themselves are summed -- widened exactly to binary64
// by the hardware conversions, squared exactly (an 11-bit significand) and
// added with one rounding each, like x*x + acc of the definition -- and the
// CTA's total is multiplied once by 2^(-2e) = 1/S^2 (SqParams::sq_unscale).
// Every partial sum is then the definition's partial sum times S^2, exactly,
// so the result is bit for bit that of summing x*x.
//
// Other S: x is rounded to binary32 first, as the definition says.
template <bool kPow2>
__device__ __forceinline__ double sq_value(float g, const SqParams& a)
{
    if constexpr (kPow2)
        return (double)g;
    else
        return (double)__fmul_rn(g, a.inv_scale);
}

template <bool kPow2>
__device__ __forceinline__ void sq_word(uint32_t w, const SqParams& a, SqAcc& s)
{
    double x0, x1;
    if constexpr (kPow2) {
        // the two binary16 lanes widened straight to binary64 (exact): one
        // conversion per gradient instead of two
        asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "cvt.f64.f16 %0, lo;\n\tcvt.f64.f16 %1, hi;\n\t}"
            : "=d"(x0), "=d"(x1) : "r"(w));
    } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        x0 = sq_value<kPow2>(f.x, a);
        x1 = sq_value<kPow2>(f.y, a);
    }
    s.a0 = fma(x0, x0, s.a0);
    s.a1 = fma(x1, x1, s.a1);
}

template <bool kPow2>
__device__ __forceinline__ void sq_half(uint16_t h, const SqParams& a, SqAcc& s)
{
    const double x = sq_value<kPow2>(__half2float(__ushort_as_half(h)), a);
    s.a0 = fma(x, x, s.a0);
}

// A CTA's sum of squares in the definition's scale (power-of-two S: the sum
// of the scaled squares times 1/S^2, exact).
__device__ __forceinline__ double unscaled_sum(double part, const SqParams& a)
{
    return a.pow2 ? part * a.sq_unscale : part;
}

template <bool kPow2>
__device__ __forceinline__ void sq_vec(uint4 v, const SqParams& a, SqAcc& s)
{
    sq_word<kPow2>(v.x, a, s);
    sq_word<kPow2>(v.y, a, s);
    sq_word<kPow2>(v.z, a, s);
    sq_word<kPow2>(v.w, a, s);
}

// Statistics mode: each thread counts the binary16 exponent fields it sees in
// its own row of a shared-memory table (rows padded to 33 words, so that
// threads of a warp incrementing the same bin hit different banks) and keeps
// the largest magnitude bit pattern.
struct StatsAcc {
    uint32_t* row;
    uint32_t mx = 0;
};

// Statistics levels: kNoStats; kMaxOnly (the direct scaler mode needs only
// the largest magnitude); kMaxHist (also the exponent histogram).
constexpr int kNoStats = 0, kMaxOnly = 1, kMaxHist = 2;

template <int kStats>
__device__ __forceinline__ void stats_half(uint32_t h, StatsAcc* st)
{
    if constexpr (kStats != kNoStats) {
        const uint32_t m = h & 0x7FFFu;
        if constexpr (kStats == kMaxHist)
            st->row[m >> 10] += 1;
        st->mx = max(st->mx, m);
    }
}

template <int kStats>
__device__ __forceinline__ void stats_word(uint32_t w, StatsAcc* st)
{
    if constexpr (kStats == kMaxOnly) {
        // both lanes at once: max of the two 15-bit magnitudes
        st->mx = max(st->mx, max(w & 0x7FFFu, (w >> 16) & 0x7FFFu));
    } else if constexpr (kStats == kMaxHist) {
        stats_half<kStats>(w & 0xFFFFu, st);
        stats_half<kStats>(w >> 16, st);
    }
}

template <int kStats>
__device__ __forceinline__ void stats_vec(uint4 v, StatsAcc* st)
{
    stats_word<kStats>(v.x, st);
    stats_word<kStats>(v.y, st);
    stats_word<kStats>(v.z, st);
    stats_word<kStats>(v.w, st);
}

// Range counts of the gradients (how many are +-0 and how many are
// subnormal in binary16: the part of the gradient distribution that FP16
// flushes or keeps only with reduced precision).
//
// Per gradient word (two binary16 lanes), with m = the lanes' magnitudes:
// m + 0x7FFF sets a lane's bit 15 iff the lane is not +-0, m + 0x7C00 iff it
// is at least 2^-14 (normal, inf or NaN).  One byte permute gathers the four
// flag bytes into byte lanes [nonzero lo, nonzero hi, normal lo, normal hi]
// that accumulate in b4 (at most 16 per byte between two folds: one batch of
// kCheckVecs 16-byte vectors); fold() moves them into lane-packed 16-bit
// counters, of which a thread fills at most 2^11 per lane (at most 2^20
// elements per bin), far below overflow.
struct RangeCounts {
    uint32_t nz2 = 0;  // lanes with |g16| != 0
    uint32_t ns2 = 0;  // lanes with |g16| >= 2^-14 (normal, inf or NaN)
    uint32_t b4 = 0;   // byte lanes, see above

    __device__ __forceinline__ void word(uint32_t w)
    {
        const uint32_t m = w & 0x7FFF7FFFu;
        const uint32_t p = __byte_perm(m + 0x7FFF7FFFu, m + 0x7C007C00u, 0x7531);
        b4 += (p >> 7) & 0x01010101u;
    }
    __device__ __forceinline__ void vec(uint4 v)
    {
        word(v.x);
        word(v.y);
        word(v.z);
        word(v.w);
    }
    __device__ __forceinline__ void fold()
    {
        nz2 += __byte_perm(b4, 0, 0x4140);  // bytes 0, 1 -> the two 16-bit lanes
        ns2 += __byte_perm(b4, 0, 0x4342);  // bytes 2, 3
        b4 = 0;
    }
    __device__ __forceinline__ void half(uint16_t h)
    {
        const uint32_t m = h & 0x7FFFu;
        nz2 += m != 0 ? 1u : 0u;
        ns2 += m >= 0x0400u ? 1u : 0u;
    }
    __device__ __forceinline__ unsigned int nonzero() const { return (nz2 & 0xFFFFu) + (nz2 >> 16); }
    __device__ __forceinline__ unsigned int normal() const { return (ns2 & 0xFFFFu) + (ns2 >> 16); }
};

// Gradients of the check pass per thread: 16-B loads, kCheckVecs of them in
// flight per thread (64 B).
constexpr int kCheckVecs = 4;

template <bool kPow2, bool kCount, int kStats>
__device__ __forceinline__ void check_half(uint16_t h, const SqParams& a, SqAcc& s,
                                           RangeCounts* rc, StatsAcc* st)
{
    sq_half<kPow2>(h, a, s);
    if constexpr (kCount)
        rc->half(h);
    stats_half<kStats>(h, st);
}

// One contiguous range of gradients starting on a 16-byte boundary.
template <bool kPow2, bool kCount, int kStats>
__device__ __forceinline__ void check_range_vec(const uint16_t* g, int len, const SqParams& a,
                                                SqAcc& s, RangeCounts* rc, StatsAcc* st)
{
    constexpr int kU = kCheckVecs;
    const uint4* gv = reinterpret_cast<const uint4*>(g);
    const int nv = len >> 3;
    int i = threadIdx.x;
    for (; i + (kU - 1) * kThreads < nv; i += kU * kThreads) {
        uint4 v[kU];
#pragma unroll
        for (int k = 0; k < kU; ++k)
            v[k] = __ldg(gv + i + k * kThreads);
#pragma unroll
        for (int k = 0; k < kU; ++k) {
            sq_vec<kPow2>(v[k], a, s);
            if constexpr (kCount)
                rc->vec(v[k]);
            stats_vec<kStats>(v[k], st);
        }
        if constexpr (kCount)
            rc->fold();
    }
    for (; i < nv; i += kThreads) {
        const uint4 v = __ldg(gv + i);
        sq_vec<kPow2>(v, a, s);
        if constexpr (kCount) {
            rc->vec(v);
            rc->fold();
        }
        stats_vec<kStats>(v, st);
    }
    for (int j = (nv << 3) + threadIdx.x; j < len; j += kThreads)
        check_half<kPow2, kCount, kStats>(__ldg(g + j), a, s, rc, st);
}

// One contiguous range at any 2-byte alignment: the elements before the
// first 16-byte boundary one per thread, the rest with 16-B loads.
template <bool kPow2, bool kCount, int kStats>
__device__ __forceinline__ void check_range(const uint16_t* g, int len, const SqParams& a,
                                            SqAcc& s, RangeCounts* rc, StatsAcc* st)
{
    const uintptr_t p = reinterpret_cast<uintptr_t>(g);
    const int head = min(len, (int)(((16u - (unsigned int)(p & 15u)) & 15u) >> 1));
    if ((int)threadIdx.x < head)
        check_half<kPow2, kCount, kStats>(__ldg(g + threadIdx.x), a, s, rc, st);
    check_range_vec<kPow2, kCount, kStats>(g + head, len - head, a, s, rc, st);
}

// Fixed-shape block sum (result valid in thread 0): deterministic for a fixed
// launch shape, independent of timing.
__device__ __forceinline__ double block_sum(double x, double* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_down_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = x;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            t += red[w];
    }
    __syncthreads();
    return t;
}

// The same fixed-shape reduction for a CTA's sum of squares together with its
// two range counters (results valid in thread 0; the binary64 sum is added in
// the same order as block_sum's).
struct CtaTotals {
    double sq;
    unsigned int nonzero, normal;
};

__device__ __forceinline__ CtaTotals block_totals(double x, unsigned int nz, unsigned int ns,
                                                  double* red, uint2* ured)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_down_sync(0xffffffffu, x, o);
    nz = __reduce_add_sync(0xffffffffu, nz);
    ns = __reduce_add_sync(0xffffffffu, ns);
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5] = x;
        ured[threadIdx.x >> 5] = make_uint2(nz, ns);
    }
    __syncthreads();
    CtaTotals t{0.0, 0u, 0u};
    if (threadIdx.x == 0) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            t.sq += red[w];
            t.nonzero += ured[w].x;
            t.normal += ured[w].y;
        }
    }
    __syncthreads();
    return t;
}

// This thread's share of the per-bin partials, k = threadIdx.x + i*kThreads in
// increasing i, eight loads issued before they are added (the same order of
// additions as one load at a time).  Slots past n read as +0.0, which leaves
// the running sum unchanged: the partials are non-negative, +inf or NaN, so
// the sum is never -0.0.  The last, partly filled batch is thereby issued at
// once like the others.
__device__ __forceinline__ double sum_partials(const double* partials, int n)
{
    constexpr int kU = 8;
    double x = 0.0;
    for (int k = threadIdx.x; k < n; k += kU * kThreads) {
        double p[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            const int j = k + i * kThreads;
            p[i] = j < n ? __ldcg(partials + j) : 0.0;
        }
#pragma unroll
        for (int i = 0; i < kU; ++i)
            x += p[i];
    }
    return x;
}

__device__ __forceinline__ unsigned int block_sum_u32(unsigned int x, unsigned int* red)
{
    x = __reduce_add_sync(0xffffffffu, x);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = x;
    __syncthreads();
    unsigned int t = 0;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            t += red[w];
    }
    __syncthreads();
    return t;
}

// Exact count of non-finite elements in n gradients (run only by a CTA that
// saw one).
__device__ __forceinline__ unsigned int count_nonfinite(const uint16_t* g, int n)
{
    unsigned int c = 0;
    for (int j = threadIdx.x; j < n; j += kThreads)
        c += ((g[j] & 0x7C00u) == 0x7C00u) ? 1u : 0u;
    return c;
}

// Packed bins: the gradient pointer and offset of each tensor are staged in
// shared memory once, then every thread handles several elements at a time
// (8 in the check pass, 4 in the update) with all of their loads issued
// before any is used.
struct PackedStage {
    int32_t begin[kMaxPackedSegs];
    const uint16_t* gptr[kMaxPackedSegs];
    int64_t arena[kMaxPackedSegs];
};

__device__ __forceinline__ void stage_packed(const Bin& bin, const Tables& t, PackedStage& st)
{
    for (int k = threadIdx.x; k < bin.n_segs; k += kThreads) {
        const Seg s = t.segs[bin.tensor + k];
        st.begin[k] = s.local_begin;
        st.gptr[k] = t.grads[s.tensor] + s.tensor_begin;
        st.arena[k] = s.arena_begin;
    }
    __syncthreads();
}

// Largest finite |g16| bit pattern among n gradients (statistics mode, CTAs
// that saw an inf/NaN: their running maximum included it).
__device__ __forceinline__ uint32_t finite_max(const uint16_t* g, int n)
{
    uint32_t mx = 0;
    for (int j = threadIdx.x; j < n; j += kThreads) {
        const uint32_t m = g[j] & 0x7FFFu;
        if (m < 0x7C00u)
            mx = max(mx, m);
    }
    return mx;
}

__device__ __forceinline__ unsigned int block_max_u32(unsigned int x, unsigned int* red)
{
    x = __reduce_max_sync(0xffffffffu, x);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = x;
    __syncthreads();
    unsigned int t = 0;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            t = max(t, red[w]);
    }
    __syncthreads();
    return t;
}

// kStats: also the largest finite |g16| and the histogram of binary16
// exponent fields (the FP16 binades of the scaled gradients), needed by the
// direct scaler mode and reported as statistics.
template <bool kChecked, int kStats>
__global__ void __launch_bounds__(kThreads, kStats == kMaxHist ? 4 : 8) check_kernel(CheckArgs a)
{
    constexpr int kRow = 33;  // 32 bins + 1 word of padding per thread
    __shared__ PackedStage st;
    __shared__ double s_red[kWarps];
    __shared__ unsigned int s_ured[kWarps];
    __shared__ uint2 s_cnt[kWarps];
    __shared__ uint32_t s_hist[kStats == kMaxHist ? kThreads * kRow : 1];
    __shared__ int s_last;

    // Let the update kernel (launched with programmatic stream serialization)
    // be scheduled as soon as every CTA of this grid is running; it waits for
    // this grid's completion before it reads the result.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const Tables& t = a.t;
    const Bin bin = t.bins[blockIdx.x];
    // S of these gradients: the host's, or the device state the previous
    // step left (written only by CTA 0 of the update kernel, which has
    // completed before this kernel starts)
    float S;
    SqParams q;
    if (a.scale_on_device) {
        const Ctrl* c = a.ctrl;
        S = c->scale;
        q.inv_scale = c->next_inv;
        q.sq_unscale = c->next_sq_unscale;
        q.pow2 = c->next_pow2 != 0;
    } else {
        S = a.host_scale;
        q.inv_scale = a.host_inv;
        q.sq_unscale = a.host_sq_unscale;
        q.pow2 = a.host_pow2 != 0;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // For the update kernel, which finishes this step: S and 1/S of
        // these gradients, a cleared error word, its bin counter at zero, and
        // the last update's stale count moved into the total (that update
        // has completed; nothing else touches these fields during the pass).
        Ctrl* c = a.ctrl;
        c->inv_scale = q.inv_scale;
        c->scale_used = S;
        c->error = 0u;
        c->upd_next = 0u;
        c->stale_total += c->stale_acc;
        c->stale_acc = 0ull;
    }
    SqAcc s;
    RangeCounts rc;
    StatsAcc sa;
    if constexpr (kStats == kMaxHist) {
        sa.row = s_hist + threadIdx.x * kRow;
#pragma unroll
        for (int k = 0; k < 32; ++k)
            sa.row[k] = 0;
    }
    bool valid = true;
    if constexpr (kChecked)
        valid = bin_ok(bin, t);

    const uint16_t* chunk_g = nullptr;
    if (valid) {
        if (bin.kind == kChunkBin) {
            chunk_g = t.grads[bin.tensor] + bin.tensor_begin;
            if (q.pow2)
                check_range<true, true, kStats>(chunk_g, bin.n_elems, q, s, &rc, &sa);
            else
                check_range<false, true, kStats>(chunk_g, bin.n_elems, q, s, &rc, &sa);
        } else {
            stage_packed(bin, t, st);
            constexpr int kU = 8;
            for (int base = 0; base < bin.n_elems; base += kU * kThreads) {
                uint16_t h[kU];
                bool in[kU];
#pragma unroll
                for (int i = 0; i < kU; ++i) {
                    const int j = base + threadIdx.x + i * kThreads;
                    h[i] = 0;  // +0: adds nothing, is finite
                    in[i] = j < bin.n_elems;
                    if (in[i]) {
                        const int k = find_seg(st.begin, bin.n_segs, j);
                        h[i] = __ldg(st.gptr[k] + (j - st.begin[k]));
                    }
                }
                if (q.pow2) {
#pragma unroll
                    for (int i = 0; i < kU; ++i)
                        sq_half<true>(h[i], q, s);
                } else {
#pragma unroll
                    for (int i = 0; i < kU; ++i)
                        sq_half<false>(h[i], q, s);
                }
#pragma unroll
                for (int i = 0; i < kU; ++i) {
                    if (in[i]) {
                        rc.half(h[i]);
                        stats_half<kStats>(h[i], &sa);
                    }
                }
            }
        }
    }

    // Non-finite count: exact, but only computed by a CTA that saw one (it
    // also redoes its maximum over the finite gradients only).
    unsigned int nf = 0;
    if (__syncthreads_or(s.saw_nonfinite())) {
        unsigned int c = 0;
        uint32_t mx = 0;
        if (bin.kind == kChunkBin) {
            c = count_nonfinite(chunk_g, bin.n_elems);
            if constexpr (kStats != kNoStats)
                mx = finite_max(chunk_g, bin.n_elems);
        } else {
            for (int j = threadIdx.x; j < bin.n_elems; j += kThreads) {
                const int k = find_seg(st.begin, bin.n_segs, j);
                const uint32_t m = st.gptr[k][j - st.begin[k]] & 0x7FFFu;
                c += m >= 0x7C00u ? 1u : 0u;
                if (m < 0x7C00u)
                    mx = max(mx, m);
            }
        }
        sa.mx = mx;
        nf = block_sum_u32(c, s_ured);
    }

    const CtaTotals tot = block_totals(s.a0 + s.a1, rc.nonzero(), rc.normal(), s_red, s_cnt);
    const double part = unscaled_sum(tot.sq, q);
    if constexpr (kStats != kNoStats) {
        const unsigned int mx = block_max_u32(sa.mx, s_ured);   // ends with __syncthreads
        if (kStats == kMaxHist && threadIdx.x < 32) {
            unsigned long long n = 0;
            for (int r = 0; r < kThreads; ++r)
                n += s_hist[r * kRow + threadIdx.x];
            if (n)
                atomicAdd(&a.stats->hist_acc[threadIdx.x], n);
            __threadfence();
        }
        if (threadIdx.x == 0 && mx)
            atomicMax(&a.ctrl->max_mag_acc, mx);
    }
    if (threadIdx.x == 0) {
        // deferred finish: a bin that holds an inf/NaN gradient leaves NaN,
        // so the total is NaN exactly when the step overflowed (every other
        // partial is in [0, +inf]: +inf only from a binary32 product that a
        // huge 1/S overflowed, and a sum of those is never NaN)
        a.partials[blockIdx.x] = (!a.partial_out && nf) ? __longlong_as_double(0x7ff8000000000000ll) : part;
        if (nf)
            atomicAdd(&a.ctrl->nonfinite_acc, (unsigned long long)nf);
        if (valid) {
            const unsigned int n_zero = (unsigned int)bin.n_elems - tot.nonzero;
            const unsigned int n_sub = tot.nonzero - tot.normal;
            if (n_zero)
                atomicAdd(&a.ctrl->zero_acc, (unsigned long long)n_zero);
            if (n_sub)
                atomicAdd(&a.ctrl->subnormal_acc, (unsigned long long)n_sub);
        } else {
            atomicOr(&a.ctrl->error_acc, (unsigned int)kErrBadBin);
        }
    }
    // Finish by atomic tickets (the last CTA to draw one sees every partial
    // and counter: fences before each ticket make them visible).  Up to
    // kOneLevelBins bins, one level: the last CTA adds all the partials (at
    // most eight loads per thread, issued together).  Beyond, two levels, so
    // that the serial work after the last bin stays small: the last CTA to
    // complete in each group of kFinishGroup consecutive bins adds that
    // group's partials; the last group to complete adds the group sums.
    // Either way the additions follow a fixed pattern (bin order within a
    // thread's share, a fixed tree across threads), whichever CTA is last.
    __syncthreads();  // every write of this CTA precedes its ticket
    if (!a.partial_out && (int)gridDim.x <= kOneLevelBins)
        return;  // the update kernel adds the per-bin partials
    double sumsq;
    if ((int)gridDim.x <= kOneLevelBins) {
        if (threadIdx.x == 0) {
            __threadfence();
            s_last = atomicAdd(&a.ctrl->ticket, 1u) == gridDim.x - 1;
        }
        __syncthreads();
        if (!s_last)
            return;
        __threadfence();
        sumsq = block_sum(sum_partials(a.partials, (int)gridDim.x), s_red);
    } else {
        const int grp = (int)blockIdx.x / kFinishGroup;
        const int g_begin = grp * kFinishGroup;
        const int g_len = min(kFinishGroup, (int)gridDim.x - g_begin);
        if (threadIdx.x == 0) {
            __threadfence();
            s_last = atomicAdd(&a.group_tickets[grp], 1u) == (unsigned int)g_len - 1;
        }
        __syncthreads();
        if (!s_last)
            return;
        __threadfence();
        const double gsum = block_sum(
            threadIdx.x < g_len ? __ldcg(a.partials + g_begin + threadIdx.x) : 0.0, s_red);
        const int ngroups = ((int)gridDim.x + kFinishGroup - 1) / kFinishGroup;
        if (!a.partial_out) {
            // the update kernel adds the group sums
            if (threadIdx.x == 0) {
                a.group_partials[grp] = gsum;
                a.group_tickets[grp] = 0;
            }
            return;
        }
        if (threadIdx.x == 0) {
            a.group_partials[grp] = gsum;
            a.group_tickets[grp] = 0;
            __threadfence();
            s_last = atomicAdd(&a.ctrl->ticket, 1u) == (unsigned int)ngroups - 1;
        }
        __syncthreads();
        if (!s_last)
            return;
        __threadfence();
        sumsq = block_sum(sum_partials(a.group_partials, ngroups), s_red);
    }

    // Last CTA of a sharded step's check pass: every CTA's partial and
    // counters are visible; they become this shard's record.
    Ctrl* c = a.ctrl;
    if constexpr (kStats == kMaxHist) {
        if (threadIdx.x < 32) {
            a.stats->hist[threadIdx.x] = atomicExch(&a.stats->hist_acc[threadIdx.x], 0ull);
        }
    }
    if (threadIdx.x == 0) {
        const unsigned long long n_nonfinite = atomicExch(&c->nonfinite_acc, 0ull);
        const unsigned int err = atomicExch(&c->error_acc, 0u);
        const unsigned int mm = kStats != kNoStats ? atomicExch(&c->max_mag_acc, 0u) : 0u;
        c->ticket = 0;
        // this shard's range counts go straight to the result, so that every
        // accumulator is clear again when the pass ends (a check pass whose
        // step is never finished leaves nothing for the next step)
        c->n_zero = atomicExch(&c->zero_acc, 0ull);
        c->n_subnormal = atomicExch(&c->subnormal_acc, 0ull);
        Partial p{};
        p.sumsq = sumsq;
        p.n_nonfinite = n_nonfinite;
        p.max_mag = mm;
        p.error = err;
        *a.partial_out = p;
    }
}

// ---------------------------------------------------------------------------
// update kernel: fused unscale, clip, weight decay, momentum, master, FP16
// ---------------------------------------------------------------------------

struct UpdParams {
    float inv_scale, coef, lr, mu, wd, eps;
};

// Sharded step: ranks' records staged in shared memory per round.
constexpr int kRecStage = 32;

// Elements of a chunk bin whose master, momentum and gradients the update
// kernel prefetches into L2 before it waits for the check result.
constexpr int kPrefetchElems = 8192;

// Bulk prefetch of [p, p + bytes) into L2 (non-multicast TMA; p 16-byte
// aligned, bytes a multiple of 16, both in bounds).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// One element, each operation rounded to binary32 on its own (no FMA).
//   momentum: v = mu*v + d;              w = w - lr*v
//   Nesterov: v = mu*v + d;              w = w - lr*(d + mu*v)
//   Adagrad:  v = v + d*d (sum of squares); w = w - lr*d/(sqrt(v) + eps)
template <int kOpt>
__device__ __forceinline__ void upd1(float g16f, float& w, float& v, const UpdParams& p)
{
    float g = __fmul_rn(g16f, p.inv_scale);  // unscale
    g = __fmul_rn(g, p.coef);                // global-L2 clip (coef 1: exact no-op)
    const float t = __fmul_rn(p.wd, w);      // weight decay on the FP32 master
    const float d = __fadd_rn(g, t);
    float step;
    if constexpr (kOpt == kOptAdagrad) {
        v = __fadd_rn(v, __fmul_rn(d, d));
        step = __fdiv_rn(d, __fadd_rn(__fsqrt_rn(v), p.eps));
    } else {
        const float u = __fmul_rn(p.mu, v);  // momentum
        v = __fadd_rn(u, d);
        step = v;
        if constexpr (kOpt == kOptNesterov)
            step = __fadd_rn(d, __fmul_rn(p.mu, v));
    }
    const float s = __fmul_rn(p.lr, step);   // master update
    w = __fsub_rn(w, s);
}

template <bool kStale>
__device__ __forceinline__ void stale1(float w_old, float w_new, uint32_t& stale)
{
    if constexpr (kStale) {
        if (w_new != w_old &&
            __half_as_ushort(__float2half_rn(w_new)) == __half_as_ushort(__float2half_rn(w_old)))
            ++stale;
    }
}

// Four elements: the four FP16 gradients (two words), 16-B master and
// momentum, 16-B + 16-B + 8-B stores (every warp access is 256 B or 512 B
// contiguous).
template <int kOpt, bool kStale>
__device__ __forceinline__ void upd4(uint2 g, float4& w, float4& v, uint2& h, const UpdParams& p,
                                     uint32_t& stale)
{
    const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&g.x));
    const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&g.y));
    const float4 w0 = w;
    upd1<kOpt>(g01.x, w.x, v.x, p);
    upd1<kOpt>(g01.y, w.y, v.y, p);
    upd1<kOpt>(g23.x, w.z, v.z, p);
    upd1<kOpt>(g23.y, w.w, v.w, p);
    h.x = h2_bits(__floats2half2_rn(w.x, w.y));
    h.y = h2_bits(__floats2half2_rn(w.z, w.w));
    stale1<kStale>(w0.x, w.x, stale);
    stale1<kStale>(w0.y, w.y, stale);
    stale1<kStale>(w0.z, w.z, stale);
    stale1<kStale>(w0.w, w.w, stale);
}

template <int kOpt, bool kStale>
__device__ __forceinline__ void upd_scalar(uint16_t g16, float* w, float* v, uint16_t* h,
                                           const UpdParams& p, uint32_t& stale)
{
    float wi = *w, vi = *v;
    const float w0 = wi;
    upd1<kOpt>(__half2float(__ushort_as_half(g16)), wi, vi, p);
    __stcs(w, wi);
    __stcs(v, vi);
    *h = __half_as_ushort(__float2half_rn(wi));
    stale1<kStale>(w0, wi, stale);
}

// The four gradients of quad i (elements 4i .. 4i+3) of a range that starts
// kS elements (2*kS bytes) past an 8-byte boundary, from the two aligned
// 8-byte words that hold them: the upper 4 - kS elements of word i and the
// lower kS of word i + 1 (word k holds elements 4k - kS .. 4k - kS + 3).
template <int kS>
__device__ __forceinline__ uint2 quad_from(uint2 lo, uint2 hi)
{
    uint2 q;
    if constexpr (kS == 0) {
        q = lo;
    } else if constexpr (kS == 1) {
        q.x = __funnelshift_r(lo.x, lo.y, 16);
        q.y = __funnelshift_r(lo.y, hi.x, 16);
    } else if constexpr (kS == 2) {
        q.x = lo.y;
        q.y = hi.x;
    } else {
        q.x = __funnelshift_r(lo.y, hi.x, 16);
        q.y = __funnelshift_r(hi.x, hi.y, 16);
    }
    return q;
}

// Quads [i0, i1) of a range: master, momentum and FP16 copy are 16-/8-byte
// aligned; the gradients start kS elements past an 8-byte boundary and are
// read as aligned 8-byte words (two per quad when kS != 0, which the caller
// keeps inside the range: i0 >= 1 and word i1 within it).  Each thread takes
// quads i0 + threadIdx.x + k*kThreads, all four iterations' loads issued
// before any is used (160 B in flight per thread).
template <int kOpt, bool kStale, int kS>
__device__ __forceinline__ void update_quads(const uint16_t* g, float* w, float* v, uint16_t* h,
                                             int i0, int i1, const UpdParams& p, uint32_t& stale)
{
    constexpr int kUnroll = 4;
    const uint2* gw = reinterpret_cast<const uint2*>(g - kS);
    float4* w4 = reinterpret_cast<float4*>(w);
    float4* v4 = reinterpret_cast<float4*>(v);
    uint2* h4 = reinterpret_cast<uint2*>(h);
    int i = i0 + (int)threadIdx.x;
    for (; i + (kUnroll - 1) * kThreads < i1; i += kUnroll * kThreads) {
        uint2 lo[kUnroll], hi[kUnroll], hq[kUnroll];
        float4 wq[kUnroll], vq[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            lo[k] = __ldcs(gw + i + k * kThreads);
            if constexpr (kS != 0)
                hi[k] = __ldcs(gw + i + 1 + k * kThreads);
            else
                hi[k] = lo[k];
            wq[k] = __ldcs(w4 + i + k * kThreads);
            vq[k] = __ldcs(v4 + i + k * kThreads);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k)
            upd4<kOpt, kStale>(quad_from<kS>(lo[k], hi[k]), wq[k], vq[k], hq[k], p, stale);
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            __stcs(w4 + i + k * kThreads, wq[k]);
            __stcs(v4 + i + k * kThreads, vq[k]);
            __stcs(h4 + i + k * kThreads, hq[k]);
        }
    }
    for (; i < i1; i += kThreads) {
        const uint2 lo = __ldcs(gw + i);
        uint2 hi = lo;
        if constexpr (kS != 0)
            hi = __ldcs(gw + i + 1);
        float4 wq = __ldcs(w4 + i), vq = __ldcs(v4 + i);
        uint2 hq;
        upd4<kOpt, kStale>(quad_from<kS>(lo, hi), wq, vq, hq, p, stale);
        __stcs(w4 + i, wq);
        __stcs(v4 + i, vq);
        __stcs(h4 + i, hq);
    }
}

// One contiguous range of a chunk bin at any 2-byte gradient alignment:
// aligned quads with vector accesses; when the gradients are not 8-byte
// aligned, the first quad and the elements past the last quad whose second
// gradient word lies inside the range one element per thread.
template <int kOpt, bool kStale>
__device__ __forceinline__ void update_range(const uint16_t* g, float* w, float* v, uint16_t* h,
                                             int len, const UpdParams& p, uint32_t& stale)
{
    const int sh = (int)((reinterpret_cast<uintptr_t>(g) & 7u) >> 1);
    int q1 = len >> 2;  // quads [q0, q1) go through the vector path
    if (sh != 0) {
        // quad i needs word i + 1, whose last element 4i + 7 - sh must be < len
        q1 = len - 8 + sh >= 0 ? ((len - 8 + sh) >> 2) + 1 : 1;
        if (q1 < 1)
            q1 = 1;
    }
    switch (sh) {
    case 0: update_quads<kOpt, kStale, 0>(g, w, v, h, 0, q1, p, stale); break;
    case 1: update_quads<kOpt, kStale, 1>(g, w, v, h, 1, q1, p, stale); break;
    case 2: update_quads<kOpt, kStale, 2>(g, w, v, h, 1, q1, p, stale); break;
    default: update_quads<kOpt, kStale, 3>(g, w, v, h, 1, q1, p, stale); break;
    }
    if (sh != 0 && (int)threadIdx.x < min(4, len)) {
        const int j = threadIdx.x;
        upd_scalar<kOpt, kStale>(__ldcs(g + j), w + j, v + j, h + j, p, stale);
    }
    for (int j = 4 * q1 + (int)threadIdx.x; j < len; j += kThreads)
        upd_scalar<kOpt, kStale>(__ldcs(g + j), w + j, v + j, h + j, p, stale);
}

// Persistent grid: one CTA per resident slot (4 per SM; Adagrad 3).  CTA c
// takes bin c first (counted from the end: the check kernel read the last
// bins last, so their gradients are the ones still in L2) and then, each time
// it finishes a bin, claims the next one, gridDim.x + k for the k-th claim,
// from a counter that the check kernel resets every step: bins start in
// order, and an SM that streams faster takes more of them.  An overflow step
// costs each CTA one sum of the check kernel's partials.
template <int kOpt, bool kStale, bool kChecked>
__global__ void __launch_bounds__(kThreads, kOpt == kOptAdagrad ? 3 : 4) update_kernel(UpdateArgs a)
{
    __shared__ PackedStage st;
    __shared__ int s_next[2];
    __shared__ unsigned int s_ured[kWarps];
    __shared__ double s_red[kWarps];
    __shared__ Partial s_rec[kRecStage];
    __shared__ int s_found;
    __shared__ float s_coef;

    const Tables& t = a.t;
    const int nb = t.nbins;
    int idx = (int)blockIdx.x;
    if (idx >= nb)
        return;
    {
        // While the check kernel drains, start this CTA's first reads: a
        // bulk (TMA) prefetch of the start of its first bin's master,
        // momentum and gradient ranges into L2.  Whether to prefetch follows
        // the overflow flag as the check kernel left it: this step's flag
        // for a CTA that starts after the check has finished, the previous
        // step's for one that starts while it drains.  It is only a hint:
        // the update itself reads the flag after the wait.
        const Bin bin = t.bins[nb - 1 - idx];
        bool ok = true;
        if constexpr (kChecked)
            ok = bin_ok(bin, t);
        if (ok && bin.kind == kChunkBin && threadIdx.x == 0 &&
            *reinterpret_cast<const volatile int32_t*>(&a.ctrl->found_inf) == 0) {
            const int n_pre = min(bin.n_elems, kPrefetchElems) & ~7;
            if (n_pre > 0) {
                prefetch_l2(a.master + bin.arena_begin, (uint32_t)n_pre * 4u);
                prefetch_l2(a.momentum + bin.arena_begin, (uint32_t)n_pre * 4u);
                const uint16_t* g = t.grads[bin.tensor] + bin.tensor_begin;
                if ((reinterpret_cast<uintptr_t>(g) & 15) == 0)
                    prefetch_l2(g, (uint32_t)n_pre * 2u);
            }
        }
    }
    // Wait until the check kernel has finished and its result is visible
    // (returns at once when this grid was launched without overlap).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Add what the check pass left -- the same additions in the same order
    // in every CTA, so every CTA obtains the same bits -- and derive the
    // overflow flag, the norm and the clip coefficient.  CTA 0 also finishes
    // the step: the result, the loss-scale state, the check kernel's
    // accumulators cleared (this CTA is their only reader).
    Ctrl* c = a.ctrl;
    const bool sharded = a.fin_records != nullptr;
    double sumsq = 0.0;
    if (!sharded)
        sumsq = block_sum(sum_partials(a.fin_partials, a.fin_n), s_red);  // valid in thread 0
    unsigned long long n_nonfinite = 0;
    unsigned int max_mag = 0, err = 0;
    if (sharded) {
        // the ranks' records, added in rank order (as every rank does, so
        // every rank obtains the same bits), staged 32 at a time
        for (int base = 0; base < a.fin_world; base += kRecStage) {
            const int m = min(kRecStage, a.fin_world - base);
            if ((int)threadIdx.x < m)
                s_rec[threadIdx.x] = a.fin_records[base + threadIdx.x];
            __syncthreads();
            if (threadIdx.x == 0) {
                for (int r = 0; r < m; ++r) {
                    sumsq += s_rec[r].sumsq;
                    n_nonfinite += s_rec[r].n_nonfinite;
                    max_mag = max(max_mag, s_rec[r].max_mag);
                    err |= s_rec[r].error;
                }
            }
            __syncthreads();
        }
    }
    if (threadIdx.x == 0) {
        // whole step: the sum is NaN exactly when some gradient was inf/NaN
        const bool found = sharded ? n_nonfinite != 0 : isnan(sumsq);
        const double norm = found ? __longlong_as_double(0x7ff0000000000000ll) : sqrt(sumsq);
        const bool clipped = !found && a.clip > 0.0f && norm > (double)a.clip;
        s_found = found ? 1 : 0;
        s_coef = clipped ? __double2float_rn((double)a.clip / norm) : 1.0f;
        if (blockIdx.x == 0) {
            const bool have_max = a.stats_level != kNoStats;
            if (!sharded) {
                // (a sharded step's check kernel moved these into its record
                // and its result fields)
                if (a.stats_level == kMaxHist)
                    for (int k = 0; k < 32; ++k)
                        a.stats->hist[k] = atomicExch(&a.stats->hist_acc[k], 0ull);
                n_nonfinite = atomicExch(&c->nonfinite_acc, 0ull);
                err = atomicExch(&c->error_acc, 0u);
                max_mag = have_max ? atomicExch(&c->max_mag_acc, 0u) : 0u;
                c->n_zero = atomicExch(&c->zero_acc, 0ull);
                c->n_subnormal = atomicExch(&c->subnormal_acc, 0ull);
            }
            SqParams q;
            q.inv_scale = __ldcg(&c->inv_scale);
            q.sq_unscale = 0.0;
            q.pow2 = false;
            finish_step(c, __ldcg(&c->scale_used), q, n_nonfinite, sumsq, max_mag, have_max, err,
                        a.clip, a.scaler);
        }
    }
    __syncthreads();
    if (s_found)
        return;  // Step 6: master, momentum and FP16 copy stay as they are
    const float coef = s_coef;
    const UpdParams p{__ldcg(&c->inv_scale), coef, a.lr, a.mu, a.wd, a.eps};
    uint32_t stale = 0;
    bool bad = false;

    for (int it = 0; idx < nb; ++it) {
        const Bin bin = t.bins[nb - 1 - idx];
        bool valid = true;
        if constexpr (kChecked)
            valid = bin_ok(bin, t);
        if (!valid) {
            bad = true;
        } else if (bin.kind == kChunkBin) {
            const uint16_t* g = t.grads[bin.tensor] + bin.tensor_begin;
            update_range<kOpt, kStale>(g, a.master + bin.arena_begin, a.momentum + bin.arena_begin,
                                       a.w16 + bin.arena_begin, bin.n_elems, p, stale);
        } else {
            stage_packed(bin, t, st);
            constexpr int kU = 4;
            for (int base = 0; base < bin.n_elems; base += kU * kThreads) {
                uint16_t gh[kU];
                int64_t e[kU];
                float w[kU], v[kU];
#pragma unroll
                for (int i = 0; i < kU; ++i) {
                    const int j = base + threadIdx.x + i * kThreads;
                    e[i] = -1;
                    if (j < bin.n_elems) {
                        const int k = find_seg(st.begin, bin.n_segs, j);
                        const int off = j - st.begin[k];
                        gh[i] = __ldcs(st.gptr[k] + off);
                        e[i] = st.arena[k] + off;
                        w[i] = __ldcs(a.master + e[i]);
                        v[i] = __ldcs(a.momentum + e[i]);
                    }
                }
#pragma unroll
                for (int i = 0; i < kU; ++i) {
                    if (e[i] < 0)
                        continue;
                    const float w0 = w[i];
                    upd1<kOpt>(__half2float(__ushort_as_half(gh[i])), w[i], v[i], p);
                    __stcs(a.master + e[i], w[i]);
                    __stcs(a.momentum + e[i], v[i]);
                    a.w16[e[i]] = __half_as_ushort(__float2half_rn(w[i]));
                    stale1<kStale>(w0, w[i], stale);
                }
            }
        }
        // claim the next bin once this one is done (claiming earlier holds a
        // bin back from CTAs that free up sooner and lengthens the tail);
        // the barrier also ends every read of the packed staging before the
        // next bin may overwrite it
        if (threadIdx.x == 0)
            s_next[it & 1] = (int)gridDim.x + (int)atomicAdd(&c->upd_next, 1u);
        __syncthreads();
        idx = s_next[it & 1];
    }

    if constexpr (kStale) {
        const unsigned int n_stale = block_sum_u32(stale, s_ured);
        if (threadIdx.x == 0 && n_stale)
            atomicAdd(&c->stale_acc, (unsigned long long)n_stale);
    }
    if (kChecked && bad && threadIdx.x == 0)
        atomicOr(&c->error, (unsigned int)kErrBadBin);
}

// ---------------------------------------------------------------------------
// refresh kernel: FP16 working copy from the FP32 master
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads) refresh_kernel(const float4* master, uint2* w16, int64_t n4)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n4; i += stride) {
        const float4 m = __ldcs(master + i);
        uint2 o;
        o.x = h2_bits(__floats2half2_rn(m.x, m.y));
        o.y = h2_bits(__floats2half2_rn(m.z, m.w));
        __stcs(w16 + i, o);
    }
}

}  // namespace mpt
