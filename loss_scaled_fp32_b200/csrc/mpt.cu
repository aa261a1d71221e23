// mpt.cu -- host side of libmpt: the C ABI declared in include/mpt.h.
//
// One step = two kernel launches on the caller's stream and, for the
// waiting call, one 384-byte read-back of the control block:
//   check_kernel  (2 B/param)  overflow flag, sum of squares, range counts as
//                              per-bin (or per-group) partials
//   update_kernel (20 B/param) every CTA adds the partials (norm, clip
//                              coefficient, overflow flag), CTA 0 writes the
//                              result and the next S; then the fused
//                              unscale/clip/decay/momentum/master/FP16 update
//                              over a persistent grid; on an overflow step
//                              each CTA exits after the sum
// The launch order alone carries the check result to the update, so no host
// decision sits between the two kernels.  The loss-scale state machine runs on
// the device and keeps S there, so that steps can be queued without waiting
// (mpt_step_async); the host mirrors it on read-back.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstddef>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/mpt.h"
#include "mpt_internal.h"
#include "mpt_kernels.cuh"

using namespace mpt;

static_assert(sizeof(Ctrl) == 384, "the control block read back each step is 384 bytes");
static_assert(offsetof(Ctrl, stale_acc) == 128 && offsetof(Ctrl, sumsq) == 256,
              "one 128-byte line per group of control fields");

namespace {

constexpr size_t kRegionAlign = 256;
// Device copies of the caller's gradient-pointer table kept at once: a step
// whose pointers match one of them queues no copy (a training loop that
// alternates a few gradient buffers switches between cached tables).
constexpr int kPtrSlots = 4;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
    std::vector<int64_t> arena_off;
    int64_t arena_total = 0;
    std::vector<Bin> bins_check;   // work of the check pass (one CTA each)
    std::vector<Bin> bins_update;  // work of the update pass
    std::vector<Seg> segs;
    size_t off_ctrl = 0, off_stats = 0, off_partial_rec = 0, off_partials = 0, off_groups = 0,
           off_group_tickets = 0, off_ptrs = 0,
           off_tinfo = 0, off_bins_check = 0, off_bins_update = 0, off_segs = 0, off_master = 0,
           off_momentum = 0, off_w16 = 0, total = 0;
};

bool config_ok(const mpt_config& c)
{
    if (!(c.backoff > 0.0f && c.backoff <= 1.0f) || !(c.growth >= 1.0f) || !std::isfinite(c.growth))
        return false;
    if (c.growth_interval < 0)
        return false;
    if (!(c.min_scale > 0.0f) || !std::isfinite(c.max_scale) || !(c.max_scale >= c.min_scale))
        return false;
    if (c.flags & ~(MPT_FLAG_CHECKED | MPT_FLAG_COUNT_STALE | MPT_FLAG_GRAD_STATS))
        return false;
    if (c.scaler_mode != MPT_SCALER_DYNAMIC && c.scaler_mode != MPT_SCALER_DIRECT)
        return false;
    if (!(c.direct_margin > 0.0f) || !std::isfinite(c.direct_margin))
        return false;
    if (c.optimizer != MPT_OPT_MOMENTUM && c.optimizer != MPT_OPT_NESTEROV &&
        c.optimizer != MPT_OPT_ADAGRAD)
        return false;
    if (!(c.eps >= 0.0f) || !std::isfinite(c.eps))
        return false;
    for (int32_t ch : {c.check_chunk_elems, c.update_chunk_elems})
        if (ch != 0 && (ch < kChunkQuantum || ch > kMaxChunk || ch % kChunkQuantum != 0))
            return false;
    return true;
}

mpt_config defaults()
{
    mpt_config c;
    c.backoff = 0.5f;
    c.growth = 2.0f;
    c.growth_interval = 0;
    c.min_scale = std::ldexp(1.0f, -24);
    c.max_scale = std::ldexp(1.0f, 24);
    c.flags = 0;
    c.check_chunk_elems = 0;
    c.update_chunk_elems = 0;
    c.scaler_mode = MPT_SCALER_DYNAMIC;
    c.direct_margin = 2.0f;
    c.optimizer = MPT_OPT_MOMENTUM;
    c.eps = 1e-10f;
    return c;
}

// Arena offsets (16-element aligned) and the work bins.  Every tensor larger
// than kSmallTensor is cut into chunk-sized ranges, one bin (one CTA) each;
// the small tensors are packed, in list order, into bins of at most
// kPackedMaxElems elements and kMaxPackedSegs tensors.  The two kernels get
// their own chunk size: the check pass (2 B/param, short-lived CTAs) wants
// large bins to amortise each CTA's prologue and finish, the update pass
// (20 B/param) small bins that keep every SM streaming to the end.
static void chunk_bins(const int64_t* sizes, int32_t n, int32_t chunk, const Layout& L,
                       std::vector<Bin>& out)
{
    for (int32_t i = 0; i < n; ++i) {
        if (sizes[i] <= kSmallTensor)
            continue;
        for (int64_t c = 0; c < sizes[i]; c += chunk) {
            Bin b{};
            b.tensor_begin = c;
            b.arena_begin = L.arena_off[i] + c;
            b.tensor = i;
            b.n_elems = (int32_t)std::min<int64_t>(chunk, sizes[i] - c);
            b.n_segs = 0;
            b.kind = kChunkBin;
            out.push_back(b);
        }
    }
}

int build_layout(const int64_t* sizes, int32_t n, int32_t check_chunk, int32_t update_chunk,
                 Layout& L)
{
    L.arena_off.resize(n);
    int64_t off = 0;
    for (int32_t i = 0; i < n; ++i) {
        if (sizes[i] <= 0)
            return MPT_ERR_INVALID_ARG;
        L.arena_off[i] = off;
        off += (sizes[i] + kArenaAlign - 1) / kArenaAlign * kArenaAlign;
    }
    L.arena_total = off;

    chunk_bins(sizes, n, check_chunk, L, L.bins_check);
    chunk_bins(sizes, n, update_chunk, L, L.bins_update);
    std::vector<Bin> packed;
    Bin open{};
    bool have_open = false;
    for (int32_t i = 0; i < n; ++i) {
        if (sizes[i] > kSmallTensor)
            continue;
        const int32_t len = (int32_t)sizes[i];
        if (have_open && (open.n_elems + len > kPackedMaxElems || open.n_segs == kMaxPackedSegs)) {
            packed.push_back(open);
            have_open = false;
        }
        if (!have_open) {
            open = Bin{};
            open.tensor = (int32_t)L.segs.size();
            open.kind = kPackedBin;
            have_open = true;
        }
        Seg s{};
        s.tensor_begin = 0;
        s.arena_begin = L.arena_off[i];
        s.tensor = i;
        s.len = len;
        s.local_begin = open.n_elems;
        L.segs.push_back(s);
        open.n_segs += 1;
        open.n_elems += len;
    }
    if (have_open)
        packed.push_back(open);
    L.bins_check.insert(L.bins_check.end(), packed.begin(), packed.end());
    L.bins_update.insert(L.bins_update.end(), packed.begin(), packed.end());
    if (L.bins_check.size() > 0x7fffffffu || L.bins_update.size() > 0x7fffffffu ||
        L.segs.size() > 0x7fffffffu)
        return MPT_ERR_INVALID_ARG;

    size_t p = 0;
    auto region = [&](size_t bytes) {
        const size_t at = p;
        p = round_up(p + bytes, kRegionAlign);
        return at;
    };
    L.off_ctrl = region(sizeof(Ctrl));
    L.off_stats = region(sizeof(StatsBlock));
    L.off_partial_rec = region(sizeof(Partial));
    L.off_partials = region(sizeof(double) * L.bins_check.size());
    const size_t ngroups = (L.bins_check.size() + kFinishGroup - 1) / kFinishGroup;
    L.off_groups = region(sizeof(double) * ngroups);
    L.off_group_tickets = region(sizeof(unsigned int) * ngroups);
    L.off_ptrs = region(sizeof(void*) * (size_t)n * kPtrSlots);
    L.off_tinfo = region(sizeof(TensorInfo) * (size_t)n);
    L.off_bins_check = region(sizeof(Bin) * L.bins_check.size());
    L.off_bins_update = region(sizeof(Bin) * L.bins_update.size());
    L.off_segs = region(sizeof(Seg) * L.segs.size());
    L.off_master = region(sizeof(float) * (size_t)L.arena_total);
    L.off_momentum = region(sizeof(float) * (size_t)L.arena_total);
    L.off_w16 = region(sizeof(uint16_t) * (size_t)L.arena_total);
    L.total = p;
    return MPT_OK;
}

bool finite(float x) { return std::isfinite(x); }

// Default check-pass bin: 65536 elements, halved (down to 2048) while the
// list would give fewer than kMinCheckBins bins (four per SM of a 148-SM
// B200), so that a small list still spreads over every SM instead of leaving
// a few CTAs each a long serial loop.  (Many more, shorter bins do not pay:
// a bin's fixed latency -- table loads, reductions, ticket -- then dominates;
// for the 25.6M-parameter ResNet-50 list 32K bins measured 22.4 us in the
// step, 64K 25.3 us and 16K 27.4 us.)
constexpr int64_t kMinCheckBins = 592;

int32_t check_chunk(const mpt_config& c, const int64_t* sizes, int32_t n)
{
    if (c.check_chunk_elems)
        return c.check_chunk_elems;
    int64_t total = 0;
    for (int32_t i = 0; i < n; ++i)
        total += sizes[i] > 0 ? sizes[i] : 0;
    int32_t chunk = kDefaultCheckChunk;
    while (chunk > kChunkQuantum && total / chunk < kMinCheckBins)
        chunk /= 2;
    return chunk;
}
int32_t update_chunk(const mpt_config& c) { return c.update_chunk_elems ? c.update_chunk_elems : kDefaultUpdateChunk; }

}  // namespace

constexpr int kTimingRing = 256;  // steps whose kernel events may be pending

struct mpt_handle {
    int device = 0;
    int32_t n = 0;
    mpt_config cfg{};
    Layout L;
    char* ws = nullptr;
    // device views into the workspace
    Ctrl* d_ctrl = nullptr;
    StatsBlock* d_stats = nullptr;
    Partial* d_partial_rec = nullptr;     // this rank's record (sharded step)
    double* d_partials = nullptr;
    double* d_groups = nullptr;
    unsigned int* d_group_tickets = nullptr;
    const uint16_t** d_ptrs = nullptr;
    TensorInfo* d_tinfo = nullptr;
    Bin* d_bins_check = nullptr;
    Bin* d_bins_update = nullptr;
    Seg* d_segs = nullptr;
    float* d_master = nullptr;
    float* d_momentum = nullptr;
    uint16_t* d_w16 = nullptr;
    int32_t upd_grid = 0;                // CTAs of the persistent update grid
    // host state
    // gradient-pointer tables: slot k holds a device copy (d_ptrs + k*n) of
    // the host table ptrs, staged through pinned; copied marks the end of its
    // last copy; used orders the slots by last use
    struct PtrSlot {
        std::vector<const void*> ptrs;
        bool valid = false;
        uint64_t used = 0;
        const void** pinned = nullptr;
        cudaEvent_t copied = nullptr;
    };
    PtrSlot slot[kPtrSlots];
    int cur_slot = -1;                   // the slot of the last step (-1: none)
    uint64_t slot_clock = 0;
    Ctrl* mailbox = nullptr;             // pinned copy of the control block
    unsigned long long* hist_box = nullptr;  // pinned copy of the histogram
    uint64_t hist[32] = {};
    float scale = 1.0f;                  // host mirror of the device scale state
    int32_t clean_run = 0;
    mpt_stats_t stats{};
    bool broken = false;
    bool fail_next = false;              // test hook: the next step fails as a launch would
    // kernel timing: ring of (start, between, end) events, one per timed step;
    // every timing_every-th step queued since mpt_set_timing is timed
    int32_t timing_every = 0;
    int64_t timing_count = 0;
    std::vector<cudaEvent_t> tev;
    int64_t t_head = 0, t_tail = 0;
};

static void release(mpt_handle* h)
{
    if (!h)
        return;
    for (cudaEvent_t e : h->tev)
        if (e)
            cudaEventDestroy(e);
    for (auto& sl : h->slot) {
        if (sl.copied)
            cudaEventDestroy(sl.copied);
        if (sl.pinned)
            cudaFreeHost(sl.pinned);
    }
    if (h->mailbox)
        cudaFreeHost(h->mailbox);
    if (h->hist_box)
        cudaFreeHost(h->hist_box);
    delete h;
}

// Add the durations of the oldest timed step (waits for its last event).
static bool timing_pop(mpt_handle* h)
{
    const int slot = (int)(h->t_tail % kTimingRing);
    cudaEvent_t* e = &h->tev[3 * slot];
    float t01 = 0.0f, t12 = 0.0f;
    if (cudaEventSynchronize(e[2]) != cudaSuccess ||
        cudaEventElapsedTime(&t01, e[0], e[1]) != cudaSuccess ||
        cudaEventElapsedTime(&t12, e[1], e[2]) != cudaSuccess)
        return false;
    h->stats.check_ms_total += t01;
    h->stats.update_ms_total += t12;
    h->stats.timed_steps += 1;
    h->t_tail += 1;
    return true;
}

template <bool kChecked, int kStats>
static void launch_check(const CheckArgs& a, cudaStream_t st)
{
    check_kernel<kChecked, kStats><<<a.t.nbins, kThreads, 0, st>>>(a);
}

// Statistics the check pass gathers: the histogram with MPT_FLAG_GRAD_STATS,
// the largest magnitude alone for the direct scaler mode.
static int stats_level(const mpt_handle* h)
{
    if (h->cfg.flags & MPT_FLAG_GRAD_STATS)
        return kMaxHist;
    return h->cfg.scaler_mode == MPT_SCALER_DIRECT ? kMaxOnly : kNoStats;
}

static bool stats_on(const mpt_handle* h) { return stats_level(h) != kNoStats; }

// The update kernel may start while the check kernel drains (programmatic
// dependent launch): its CTAs take the SMs the check CTAs free, load their
// work descriptors, then wait for the check result (griddepcontrol.wait).
template <int kOpt, bool kStale, bool kChecked>
static void launch_update(const UpdateArgs& a, int grid, cudaStream_t st)
{
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned int)grid);
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = 0;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    cudaLaunchKernelEx(&lc, update_kernel<kOpt, kStale, kChecked>, a);
}

template <int kOpt>
static void launch_update_opt(const UpdateArgs& a, int grid, bool stale, bool checked, cudaStream_t st)
{
    if (stale)
        checked ? launch_update<kOpt, true, true>(a, grid, st) : launch_update<kOpt, true, false>(a, grid, st);
    else
        checked ? launch_update<kOpt, false, true>(a, grid, st) : launch_update<kOpt, false, false>(a, grid, st);
}

// The update-kernel instantiation a handle launches (its optimizer and flags
// are fixed at creation).
template <int kOpt>
static const void* update_fn_opt(bool stale, bool checked)
{
    if (stale)
        return checked ? (const void*)update_kernel<kOpt, true, true> : (const void*)update_kernel<kOpt, true, false>;
    return checked ? (const void*)update_kernel<kOpt, false, true> : (const void*)update_kernel<kOpt, false, false>;
}

static const void* update_fn(const mpt_config& c)
{
    const bool stale = (c.flags & MPT_FLAG_COUNT_STALE) != 0;
    const bool checked = (c.flags & MPT_FLAG_CHECKED) != 0;
    switch (c.optimizer) {
    case MPT_OPT_NESTEROV: return update_fn_opt<kOptNesterov>(stale, checked);
    case MPT_OPT_ADAGRAD: return update_fn_opt<kOptAdagrad>(stale, checked);
    default: return update_fn_opt<kOptMomentum>(stale, checked);
    }
}

// Persistent update grid: every resident slot of every SM (the occupancy of
// the handle's instantiation), never more CTAs than bins.
static bool size_update_grid(mpt_handle* h)
{
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, update_fn(h->cfg), kThreads, 0) != cudaSuccess)
        return false;
    const int64_t slots = (int64_t)std::max(1, sms) * std::max(1, per_sm);
    h->upd_grid = (int32_t)std::min<int64_t>(slots, (int64_t)h->L.bins_update.size());
    return h->upd_grid > 0;
}

// What the check pass needs from S (the same values the device computes when
// its state machine sets S): 1/S in binary32 and, for S = 2^e with
// -15 <= e <= 100, the binary64 constant 2^(-2e) = 1/S^2.
struct HostScale {
    float inv;
    double sq_unscale;
    int32_t pow2;
};

static HostScale host_scale_params(float S)
{
    HostScale r;
    r.inv = 1.0f / S;
    int e2 = 0;
    const bool pow2 = std::frexp(S, &e2) == 0.5f && (e2 - 1) >= -15 && (e2 - 1) <= 100;
    r.pow2 = pow2 ? 1 : 0;
    r.sq_unscale = pow2 ? std::ldexp(1.0, -2 * (e2 - 1)) : 0.0;
    return r;
}

static void launch_check_level(const mpt_handle* h, const CheckArgs& ca, bool checked, cudaStream_t st)
{
    switch (stats_level(h)) {
    case kMaxHist:
        checked ? launch_check<true, kMaxHist>(ca, st) : launch_check<false, kMaxHist>(ca, st);
        break;
    case kMaxOnly:
        checked ? launch_check<true, kMaxOnly>(ca, st) : launch_check<false, kMaxOnly>(ca, st);
        break;
    default:
        checked ? launch_check<true, kNoStats>(ca, st) : launch_check<false, kNoStats>(ca, st);
        break;
    }
}

static void launch_update_any(const mpt_handle* h, const UpdateArgs& ua, bool stale, bool checked,
                              cudaStream_t st)
{
    const int g = h->upd_grid;
    switch (h->cfg.optimizer) {
    case MPT_OPT_NESTEROV: launch_update_opt<kOptNesterov>(ua, g, stale, checked, st); break;
    case MPT_OPT_ADAGRAD: launch_update_opt<kOptAdagrad>(ua, g, stale, checked, st); break;
    default: launch_update_opt<kOptMomentum>(ua, g, stale, checked, st); break;
    }
}

// What enqueue_step queues: the whole step, or one half of a sharded step
// (the check pass writing this shard's record / the update, which adds the
// ranks' records and finishes the step).
enum class Phase { kWhole, kShardCheck, kShardFinish };

// An NVTX range around the host work of one call (named ranges for a
// timeline profiler; near-free when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Queue a step (or a phase of a sharded step) on st.  scale_on_device: S
// comes from the device scale state instead of host_scale.
static int enqueue_step(mpt_handle* h, const void* const* d_grads_half, bool scale_on_device,
                        float host_scale, float lr, float momentum, float weight_decay,
                        float clip, cudaStream_t st, Phase phase = Phase::kWhole,
                        const void* d_parts = nullptr, int32_t world = 0)
{
    NvtxRange range(phase == Phase::kWhole ? "mpt.step" :
                    phase == Phase::kShardCheck ? "mpt.step_partial" : "mpt.step_finish");
    if (phase == Phase::kShardFinish)
        d_grads_half = h->slot[h->cur_slot].ptrs.data();  // the pointers of the check pass
    for (int32_t i = 0; i < h->n; ++i) {
        const uintptr_t p = reinterpret_cast<uintptr_t>(d_grads_half[i]);
        if (p == 0 || (p & 1))
            return MPT_ERR_INVALID_ARG;
    }
    if (h->fail_next) {
        // test hook: report what a failed kernel launch reports, queue nothing
        h->fail_next = false;
        return MPT_ERR_CUDA;
    }
    const size_t ptr_bytes = sizeof(void*) * (size_t)h->n;

    // The pointer table crosses to the device only when no cached slot holds
    // it: then the least recently used slot is rewritten (stream-ordered
    // after the steps queued before that read it; its staging buffer is
    // reused only once its previous copy has completed).
    int k = -1;
    if (h->cur_slot >= 0 && std::memcmp(h->slot[h->cur_slot].ptrs.data(), d_grads_half, ptr_bytes) == 0)
        k = h->cur_slot;
    for (int i = 0; k < 0 && i < kPtrSlots; ++i)
        if (h->slot[i].valid && std::memcmp(h->slot[i].ptrs.data(), d_grads_half, ptr_bytes) == 0)
            k = i;
    if (k < 0) {
        k = 0;
        for (int i = 1; i < kPtrSlots; ++i)
            if (!h->slot[i].valid ? h->slot[k].valid : (h->slot[k].valid && h->slot[i].used < h->slot[k].used))
                k = i;
        auto& sl = h->slot[k];
        if (sl.valid && cudaEventSynchronize(sl.copied) != cudaSuccess)
            return MPT_ERR_CUDA;
        sl.valid = false;
        std::memcpy(sl.pinned, d_grads_half, ptr_bytes);
        if (cudaMemcpyAsync(h->d_ptrs + (size_t)k * h->n, sl.pinned, ptr_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaEventRecord(sl.copied, st) != cudaSuccess)
            return MPT_ERR_CUDA;
        std::memcpy(sl.ptrs.data(), d_grads_half, ptr_bytes);
        sl.valid = true;
    }
    h->slot[k].used = ++h->slot_clock;
    h->cur_slot = k;

    Tables t;
    t.bins = h->d_bins_check;
    t.segs = h->d_segs;
    t.tensors = h->d_tinfo;
    t.grads = h->d_ptrs + (size_t)k * h->n;
    t.nbins = (int32_t)h->L.bins_check.size();
    t.nsegs = (int32_t)h->L.segs.size();
    t.ntensors = h->n;
    t.pad = 0;
    t.arena_total = h->L.arena_total;

    CheckArgs ca;
    ca.t = t;
    ca.partials = h->d_partials;
    ca.group_partials = h->d_groups;
    ca.group_tickets = h->d_group_tickets;
    ca.ctrl = h->d_ctrl;
    ca.host_scale = host_scale;
    {
        const HostScale hp = host_scale_params(scale_on_device ? 1.0f : host_scale);
        ca.host_inv = hp.inv;
        ca.host_sq_unscale = hp.sq_unscale;
        ca.host_pow2 = hp.pow2;
    }
    ca.scale_on_device = scale_on_device ? 1 : 0;
    ca.stats = h->d_stats;
    ca.partial_out = phase == Phase::kShardCheck ? h->d_partial_rec : nullptr;

    UpdateArgs ua;
    ua.t = t;
    ua.t.bins = h->d_bins_update;
    ua.t.nbins = (int32_t)h->L.bins_update.size();
    ua.master = h->d_master;
    ua.momentum = h->d_momentum;
    ua.w16 = h->d_w16;
    ua.ctrl = h->d_ctrl;
    ua.lr = lr;
    ua.mu = momentum;
    ua.wd = weight_decay;
    ua.eps = h->cfg.eps;
    {
        // whole step: the check kernel's per-bin (or per-group) partials;
        // sharded step: the ranks' records
        const int nbc = (int)h->L.bins_check.size();
        const bool one_level = nbc <= kOneLevelBins;
        const bool whole = phase == Phase::kWhole;
        ua.fin_partials = whole ? (one_level ? h->d_partials : h->d_groups) : nullptr;
        ua.fin_n = whole ? (one_level ? nbc : (nbc + kFinishGroup - 1) / kFinishGroup) : 0;
        ua.fin_records = whole ? nullptr : static_cast<const Partial*>(d_parts);
        ua.fin_world = whole ? 0 : world;
    }
    ua.stats_level = stats_level(h);
    ua.clip = clip;
    ua.scaler.backoff = h->cfg.backoff;
    ua.scaler.growth = h->cfg.growth;
    ua.scaler.growth_interval = h->cfg.growth_interval;
    ua.scaler.min_scale = h->cfg.min_scale;
    ua.scaler.max_scale = h->cfg.max_scale;
    ua.scaler.mode = h->cfg.scaler_mode;
    ua.scaler.direct_margin = h->cfg.direct_margin;
    ua.stats = h->d_stats;

    const bool checked = (h->cfg.flags & MPT_FLAG_CHECKED) != 0;
    const bool stale = (h->cfg.flags & MPT_FLAG_COUNT_STALE) != 0;
    if (phase != Phase::kWhole) {  // sharded step halves (not timed)
        if (phase == Phase::kShardCheck)
            launch_check_level(h, ca, checked, st);
        else
            launch_update_any(h, ua, stale, checked, st);
        return cudaGetLastError() == cudaSuccess ? MPT_OK : MPT_ERR_CUDA;
    }

    cudaEvent_t* ev = nullptr;
    if (h->timing_every > 0 && h->timing_count++ % h->timing_every == 0) {
        if (h->t_head - h->t_tail == kTimingRing && !timing_pop(h))
            return MPT_ERR_CUDA;
        ev = &h->tev[3 * (int)(h->t_head % kTimingRing)];
        h->t_head += 1;
    }
    bool ok = true;
    if (ev)
        ok = ok && cudaEventRecord(ev[0], st) == cudaSuccess;
    launch_check_level(h, ca, checked, st);
    if (ev)
        ok = ok && cudaEventRecord(ev[1], st) == cudaSuccess;
    launch_update_any(h, ua, stale, checked, st);
    if (ev)
        ok = ok && cudaEventRecord(ev[2], st) == cudaSuccess;
    ok = ok && cudaGetLastError() == cudaSuccess;
    return ok ? MPT_OK : MPT_ERR_CUDA;
}

// Read the control block back (waits for the stream), mirror the device
// state on the host and turn it into a step result.
static int read_result(mpt_handle* h, cudaStream_t st, mpt_step_result* out)
{
    if (cudaMemcpyAsync(h->mailbox, h->d_ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MPT_ERR_CUDA;
    if (stats_level(h) == kMaxHist && cudaMemcpyAsync(h->hist_box, h->d_stats->hist, sizeof(h->hist),
                                       cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MPT_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return MPT_ERR_CUDA;
    while (h->t_tail < h->t_head)
        if (!timing_pop(h))
            return MPT_ERR_CUDA;
    const Ctrl& c = *h->mailbox;
    if (c.error != 0)
        return MPT_ERR_DEVICE_CHECK;
    const bool stale = (h->cfg.flags & MPT_FLAG_COUNT_STALE) != 0;
    mpt_step_result r{};
    r.found_inf = c.found_inf;
    r.clipped = c.clipped;
    r.grad_norm = c.norm;
    r.clip_coef = c.coef;
    r.n_zero = c.n_zero;
    r.n_subnormal = c.n_subnormal;
    r.n_nonfinite = c.n_nonfinite;
    r.n_fp16_stale = stale ? c.stale_acc : 0;
    r.new_scale = c.scale;
    r.clean_run = c.clean_run;
    if (stats_on(h))
        r.max_abs_grad = c.max_abs;
    if (stats_level(h) == kMaxHist)
        for (int k = 0; k < 32; ++k)
            h->hist[k] = h->hist_box[k];
    h->scale = c.scale;
    h->clean_run = c.clean_run;
    // every step's stale count, queued steps included, is summed on the device
    h->stats.n_fp16_stale_total = stale ? c.stale_total + c.stale_acc : 0;
    h->stats.steps = c.steps_total;
    h->stats.skipped = c.skipped_total;
    h->stats.scale = h->scale;
    h->stats.clean_run = h->clean_run;
    h->stats.last = r;
    if (out)
        *out = r;
    return MPT_OK;
}

static int fail_cuda(mpt_handle* h)
{
    cudaGetLastError();
    h->broken = true;
    for (auto& sl : h->slot)
        sl.valid = false;
    h->cur_slot = -1;
    return MPT_ERR_CUDA;
}

static bool upload_scaler_state(mpt_handle* h, float scale, int32_t clean_run)
{
    const HostScale p = host_scale_params(scale);
    char* c = reinterpret_cast<char*>(h->d_ctrl);
    return cudaMemcpy(c + offsetof(Ctrl, scale), &scale, sizeof scale, cudaMemcpyHostToDevice) == cudaSuccess &&
           cudaMemcpy(c + offsetof(Ctrl, clean_run), &clean_run, sizeof clean_run, cudaMemcpyHostToDevice) == cudaSuccess &&
           cudaMemcpy(c + offsetof(Ctrl, next_inv), &p.inv, sizeof p.inv, cudaMemcpyHostToDevice) == cudaSuccess &&
           cudaMemcpy(c + offsetof(Ctrl, next_sq_unscale), &p.sq_unscale, sizeof p.sq_unscale, cudaMemcpyHostToDevice) == cudaSuccess &&
           cudaMemcpy(c + offsetof(Ctrl, next_pow2), &p.pow2, sizeof p.pow2, cudaMemcpyHostToDevice) == cudaSuccess;
}

extern "C" {

int mpt_config_init(mpt_config* cfg)
{
    if (!cfg)
        return MPT_ERR_INVALID_ARG;
    *cfg = defaults();
    return MPT_OK;
}

int mpt_workspace_bytes(const int64_t* sizes, int32_t n, const mpt_config* cfg, size_t* bytes)
{
    if (!sizes || !bytes || n <= 0)
        return MPT_ERR_INVALID_ARG;
    const mpt_config c = cfg ? *cfg : defaults();
    if (!config_ok(c))
        return MPT_ERR_INVALID_ARG;
    Layout L;
    const int rc = build_layout(sizes, n, check_chunk(c, sizes, n), update_chunk(c), L);
    if (rc != MPT_OK)
        return rc;
    *bytes = L.total;
    return MPT_OK;
}

int mpt_create(const int64_t* sizes, int32_t n, const mpt_config* cfg, void* d_workspace,
               size_t ws_bytes, mpt_handle** out)
{
    if (!sizes || n <= 0 || !out)
        return MPT_ERR_INVALID_ARG;
    *out = nullptr;
    const mpt_config c = cfg ? *cfg : defaults();
    if (!config_ok(c))
        return MPT_ERR_INVALID_ARG;
    mpt_handle* h = new (std::nothrow) mpt_handle();
    if (!h)
        return MPT_ERR_INVALID_ARG;
    h->cfg = c;
    h->n = n;
    int rc = build_layout(sizes, n, check_chunk(c, sizes, n), update_chunk(c), h->L);
    if (rc != MPT_OK) {
        release(h);
        return rc;
    }
    if (!d_workspace || (reinterpret_cast<uintptr_t>(d_workspace) % kRegionAlign) != 0 ||
        ws_bytes < h->L.total) {
        release(h);
        return MPT_ERR_WORKSPACE;
    }
    if (cudaGetDevice(&h->device) != cudaSuccess) {
        release(h);
        return MPT_ERR_CUDA;
    }
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, d_workspace) != cudaSuccess ||
        attr.type != cudaMemoryTypeDevice || attr.device != h->device) {
        cudaGetLastError();
        release(h);
        return MPT_ERR_WORKSPACE;
    }

    char* ws = static_cast<char*>(d_workspace);
    const Layout& L = h->L;
    h->ws = ws;
    h->d_ctrl = reinterpret_cast<Ctrl*>(ws + L.off_ctrl);
    h->d_stats = reinterpret_cast<StatsBlock*>(ws + L.off_stats);
    h->d_partial_rec = reinterpret_cast<Partial*>(ws + L.off_partial_rec);
    h->d_partials = reinterpret_cast<double*>(ws + L.off_partials);
    h->d_groups = reinterpret_cast<double*>(ws + L.off_groups);
    h->d_group_tickets = reinterpret_cast<unsigned int*>(ws + L.off_group_tickets);
    h->d_ptrs = reinterpret_cast<const uint16_t**>(ws + L.off_ptrs);
    h->d_tinfo = reinterpret_cast<TensorInfo*>(ws + L.off_tinfo);
    h->d_bins_check = reinterpret_cast<Bin*>(ws + L.off_bins_check);
    h->d_bins_update = reinterpret_cast<Bin*>(ws + L.off_bins_update);
    h->d_segs = reinterpret_cast<Seg*>(ws + L.off_segs);
    h->d_master = reinterpret_cast<float*>(ws + L.off_master);
    h->d_momentum = reinterpret_cast<float*>(ws + L.off_momentum);
    h->d_w16 = reinterpret_cast<uint16_t*>(ws + L.off_w16);

    std::vector<TensorInfo> tinfo(n);
    for (int32_t i = 0; i < n; ++i) {
        tinfo[i].size = sizes[i];
        tinfo[i].arena_off = L.arena_off[i];
    }
    bool ok = cudaMemcpy(h->d_tinfo, tinfo.data(), sizeof(TensorInfo) * n, cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMemcpy(h->d_bins_check, L.bins_check.data(), sizeof(Bin) * L.bins_check.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMemcpy(h->d_bins_update, L.bins_update.data(), sizeof(Bin) * L.bins_update.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMemcpy(h->d_segs, L.segs.data(), sizeof(Seg) * L.segs.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMemset(h->d_ctrl, 0, sizeof(Ctrl)) == cudaSuccess &&
              cudaMemset(h->d_group_tickets, 0, L.off_ptrs - L.off_group_tickets) == cudaSuccess &&
              cudaMemset(h->d_stats, 0, sizeof(StatsBlock)) == cudaSuccess &&
              cudaMemset(h->d_ptrs, 0, sizeof(void*) * n * kPtrSlots) == cudaSuccess &&
              cudaMemset(ws + L.off_master, 0, L.total - L.off_master) == cudaSuccess &&
              cudaHostAlloc(reinterpret_cast<void**>(&h->mailbox), sizeof(Ctrl), cudaHostAllocDefault) == cudaSuccess &&
              cudaHostAlloc(reinterpret_cast<void**>(&h->hist_box), sizeof(h->hist), cudaHostAllocDefault) == cudaSuccess &&
              upload_scaler_state(h, 1.0f, 0) &&
              size_update_grid(h) &&
              cudaDeviceSynchronize() == cudaSuccess;
    for (auto& sl : h->slot) {
        if (!ok)
            break;
        sl.ptrs.assign(n, nullptr);
        ok = cudaHostAlloc(reinterpret_cast<void**>(&sl.pinned), sizeof(void*) * n, cudaHostAllocDefault) == cudaSuccess &&
             cudaEventCreateWithFlags(&sl.copied, cudaEventDisableTiming) == cudaSuccess;
    }
    if (!ok) {
        cudaGetLastError();
        release(h);
        return MPT_ERR_CUDA;
    }
    h->stats.scale = h->scale;
    *out = h;
    return MPT_OK;
}

int mpt_tensor_views(const mpt_handle* h, int32_t i, float** master, float** momentum,
                     void** w16_half)
{
    if (!h || i < 0 || i >= h->n)
        return MPT_ERR_INVALID_ARG;
    const int64_t off = h->L.arena_off[i];
    if (master)
        *master = h->d_master + off;
    if (momentum)
        *momentum = h->d_momentum + off;
    if (w16_half)
        *w16_half = h->d_w16 + off;
    return MPT_OK;
}

int mpt_refresh_half(mpt_handle* h, void* cuda_stream)
{
    if (!h)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    const int64_t n4 = h->L.arena_total / 4;
    const int64_t want = (n4 + kThreads - 1) / kThreads;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, 148 * 16));
    refresh_kernel<<<blocks, kThreads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
        reinterpret_cast<const float4*>(h->d_master), reinterpret_cast<uint2*>(h->d_w16), n4);
    if (cudaGetLastError() != cudaSuccess) {
        h->broken = true;
        return MPT_ERR_CUDA;
    }
    return MPT_OK;
}

int mpt_step(mpt_handle* h, const void* const* d_grads_half, float scale, float lr, float momentum,
             float weight_decay, float clip, void* cuda_stream, mpt_step_result* out)
{
    if (!h || !d_grads_half || !out)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    if (!finite(scale) || !(scale > 0.0f) || !finite(lr) || !finite(momentum) ||
        !finite(weight_decay) || !finite(clip))
        return MPT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    int rc = enqueue_step(h, d_grads_half, false, scale, lr, momentum, weight_decay, clip, st);
    if (rc == MPT_ERR_CUDA)
        return fail_cuda(h);
    if (rc != MPT_OK)
        return rc;
    rc = read_result(h, st, out);
    return rc == MPT_ERR_CUDA ? fail_cuda(h) : rc;
}

int mpt_step_async(mpt_handle* h, const void* const* d_grads_half, float lr, float momentum,
                   float weight_decay, float clip, void* cuda_stream)
{
    if (!h || !d_grads_half)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    if (!finite(lr) || !finite(momentum) || !finite(weight_decay) || !finite(clip))
        return MPT_ERR_INVALID_ARG;
    const int rc = enqueue_step(h, d_grads_half, true, 0.0f, lr, momentum, weight_decay, clip,
                                static_cast<cudaStream_t>(cuda_stream));
    return rc == MPT_ERR_CUDA ? fail_cuda(h) : rc;
}

int mpt_shard_len(int64_t total, int32_t world, int64_t* shard_len)
{
    if (total <= 0 || world <= 0 || !shard_len)
        return MPT_ERR_INVALID_ARG;
    const int64_t per = (total + world - 1) / world;
    *shard_len = (per + kArenaAlign - 1) / kArenaAlign * kArenaAlign;
    return MPT_OK;
}

int mpt_step_partial(mpt_handle* h, const void* const* d_grads_half, void* cuda_stream,
                     void** d_partial)
{
    if (!h || !d_grads_half || !d_partial)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    const int rc = enqueue_step(h, d_grads_half, true, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f,
                                static_cast<cudaStream_t>(cuda_stream), Phase::kShardCheck);
    if (rc == MPT_ERR_CUDA)
        return fail_cuda(h);
    if (rc == MPT_OK)
        *d_partial = h->d_partial_rec;
    return rc;
}

int mpt_step_finish(mpt_handle* h, const void* d_partials, int32_t world, float lr,
                    float momentum, float weight_decay, float clip, void* cuda_stream)
{
    if (!h || !d_partials || world <= 0 || (reinterpret_cast<uintptr_t>(d_partials) & 15) != 0)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    if (!finite(lr) || !finite(momentum) || !finite(weight_decay) || !finite(clip))
        return MPT_ERR_INVALID_ARG;
    if (h->cur_slot < 0)
        return MPT_ERR_INVALID_ARG;  // no check pass queued before
    const int rc = enqueue_step(h, nullptr, true, 0.0f, lr, momentum, weight_decay, clip,
                                static_cast<cudaStream_t>(cuda_stream), Phase::kShardFinish,
                                d_partials, world);
    return rc == MPT_ERR_CUDA ? fail_cuda(h) : rc;
}

int mpt_wait(mpt_handle* h, void* cuda_stream, mpt_step_result* out)
{
    NvtxRange range("mpt.wait");
    if (!h)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    const int rc = read_result(h, static_cast<cudaStream_t>(cuda_stream), out);
    return rc == MPT_ERR_CUDA ? fail_cuda(h) : rc;
}

int mpt_device_scale(const mpt_handle* h, float** d_scale)
{
    if (!h || !d_scale)
        return MPT_ERR_INVALID_ARG;
    *d_scale = &h->d_ctrl->scale;
    return MPT_OK;
}

int mpt_grad_histogram(const mpt_handle* h, uint64_t counts[32])
{
    if (!h || !counts)
        return MPT_ERR_INVALID_ARG;
    for (int k = 0; k < 32; ++k)
        counts[k] = h->hist[k];
    return MPT_OK;
}

int mpt_stats(const mpt_handle* h, mpt_stats_t* out)
{
    if (!h || !out)
        return MPT_ERR_INVALID_ARG;
    *out = h->stats;
    return MPT_OK;
}

int mpt_get_scaler_state(const mpt_handle* h, float* scale, int32_t* clean_run)
{
    if (!h || !scale || !clean_run)
        return MPT_ERR_INVALID_ARG;
    *scale = h->scale;
    *clean_run = h->clean_run;
    return MPT_OK;
}

int mpt_set_scaler_state(mpt_handle* h, float scale, int32_t clean_run)
{
    if (!h || !finite(scale) || !(scale > 0.0f) || clean_run < 0)
        return MPT_ERR_INVALID_ARG;
    if (h->broken)
        return MPT_ERR_BROKEN;
    if (!upload_scaler_state(h, scale, clean_run))
        return fail_cuda(h);
    h->scale = scale;
    h->clean_run = clean_run;
    h->stats.scale = scale;
    h->stats.clean_run = clean_run;
    return MPT_OK;
}

int mpt_set_timing(mpt_handle* h, int32_t every)
{
    if (!h || every < 0)
        return MPT_ERR_INVALID_ARG;
    if (every && h->tev.empty()) {
        h->tev.assign(3 * kTimingRing, nullptr);
        for (cudaEvent_t& e : h->tev) {
            if (cudaEventCreate(&e) != cudaSuccess) {
                cudaGetLastError();
                return MPT_ERR_CUDA;
            }
        }
    }
    if (!every) {
        while (h->t_tail < h->t_head)
            if (!timing_pop(h))
                return fail_cuda(h);
    }
    h->timing_every = every;
    h->timing_count = 0;
    return MPT_OK;
}

int mpt_debug_fail_next_step(mpt_handle* h)
{
    if (!h)
        return MPT_ERR_INVALID_ARG;
    h->fail_next = true;
    return MPT_OK;
}

int mpt_destroy(mpt_handle* h)
{
    release(h);
    return MPT_OK;
}

const char* mpt_error_string(int code)
{
    switch (code) {
    case MPT_OK: return "ok";
    case MPT_ERR_INVALID_ARG: return "invalid argument";
    case MPT_ERR_WORKSPACE: return "workspace too small, misaligned or not device memory";
    case MPT_ERR_CUDA: return "CUDA runtime error";
    case MPT_ERR_DEVICE_CHECK: return "checked mode found an out-of-bounds work-table entry";
    case MPT_ERR_BROKEN: return "handle unusable after an earlier CUDA error";
    case MPT_ERR_TOO_LARGE: return "input longer than MPT_NOALLOC_MAX_ELEMS (2^30) elements";
    default: return "unknown status";
    }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free check of one flat FP16 buffer (mpt_check_flat_noalloc).
//
// The same per-CTA work as check_kernel (check_range, block sums, exact
// non-finite count, last-CTA fixed-order finish), over bins cut from one
// contiguous buffer by block index, so no work tables are needed.  Its scratch
// -- two counters and one binary64 partial per bin -- lives in the file-scope
// array below instead of a caller workspace.
// ---------------------------------------------------------------------------

namespace {

constexpr int kNoAllocChunk = 32768;
constexpr int64_t kNoAllocMaxBins = MPT_NOALLOC_MAX_ELEMS / kNoAllocChunk;
constexpr size_t kNoAllocCtrlBytes = 256;
constexpr size_t kNoAllocScratchBytes = kNoAllocCtrlBytes + sizeof(double) * kNoAllocMaxBins;
constexpr int kNoAllocMaxDevices = 64;

struct NoAllocCtrl {
    unsigned long long nonfinite_acc;
    unsigned int ticket;
    unsigned int pad;
};
static_assert(sizeof(NoAllocCtrl) <= kNoAllocCtrlBytes, "counters fit their slot");
static_assert(MPT_NOALLOC_MAX_ELEMS % kNoAllocChunk == 0, "whole bins");

// Host-side lookup of the scratch array's device address, per device: only a
// successful lookup is kept, so a call that failed (say, inside a stream
// capture) leaves the next call free to try again.
std::mutex g_noalloc_mu;
std::atomic<unsigned char*> g_noalloc_addr[kNoAllocMaxDevices];

}  // namespace

// About 256 KiB on every device that loads the library, held until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

template <bool kPow2>
__global__ void __launch_bounds__(kThreads)
check_flat_kernel(const uint16_t* g, int64_t n, unsigned char* scratch, mpt_check_result* out,
                  float inv_scale, double sq_unscale, float clip)
{
    __shared__ double s_red[kWarps];
    __shared__ unsigned int s_ured[kWarps];
    __shared__ int s_last;

    NoAllocCtrl* c = reinterpret_cast<NoAllocCtrl*>(scratch);
    double* partials = reinterpret_cast<double*>(scratch + kNoAllocCtrlBytes);
    const int64_t begin = (int64_t)blockIdx.x * kNoAllocChunk;
    const int len = (int)(n - begin < kNoAllocChunk ? n - begin : kNoAllocChunk);

    SqParams a{};
    a.inv_scale = inv_scale;
    a.sq_unscale = sq_unscale;
    a.pow2 = kPow2;
    SqAcc s;
    check_range<kPow2, false, kNoStats>(g + begin, len, a, s, nullptr, nullptr);

    unsigned int nf = 0;
    if (__syncthreads_or(s.saw_nonfinite())) {
        unsigned int cnt = 0;
        for (int j = threadIdx.x; j < len; j += kThreads)
            cnt += ((g[begin + j] & 0x7C00u) == 0x7C00u) ? 1u : 0u;
        nf = block_sum_u32(cnt, s_ured);
    }
    const double part = unscaled_sum(block_sum(s.a0 + s.a1, s_red), a);
    if (threadIdx.x == 0) {
        partials[blockIdx.x] = part;
        if (nf)
            atomicAdd(&c->nonfinite_acc, (unsigned long long)nf);
        __threadfence();
        s_last = (atomicAdd(&c->ticket, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last)
        return;

    __threadfence();
    const double sumsq = block_sum(sum_partials(partials, (int)gridDim.x), s_red);
    if (threadIdx.x == 0) {
        const unsigned long long nnf = atomicAdd(&c->nonfinite_acc, 0ull);
        const bool found = nnf != 0;
        const double norm = found ? __longlong_as_double(0x7ff0000000000000ll) : sqrt(sumsq);
        const bool clipped = !found && clip > 0.0f && norm > (double)clip;
        mpt_check_result r;
        r.found_inf = found ? 1 : 0;
        r.clipped = clipped ? 1 : 0;
        r.grad_norm = norm;
        r.clip_coef = clipped ? __double2float_rn((double)clip / norm) : 1.0f;
        r.reserved = 0;
        r.n_nonfinite = nnf;
        *out = r;
        c->nonfinite_acc = 0;
        c->ticket = 0;
    }
}

// Set-up of one device, with that device current: the device address of the
// scratch array (in host code its name is only a host-side stand-in) and the
// loading of both kernel instantiations, so that no later call has to load a
// module (under lazy loading that could otherwise happen inside a capture).
static int noalloc_scratch(int dev, unsigned char** out)
{
    unsigned char* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        p = g_noalloc_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            void* addr = nullptr;
            cudaFuncAttributes fa;
            if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr ||
                cudaFuncGetAttributes(&fa, check_flat_kernel<true>) != cudaSuccess ||
                cudaFuncGetAttributes(&fa, check_flat_kernel<false>) != cudaSuccess) {
                cudaGetLastError();  // this failure's own error; a later call retries
                return MPT_ERR_CUDA;
            }
            p = static_cast<unsigned char*>(addr);
            g_noalloc_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return MPT_OK;
}

extern "C" int mpt_check_flat_noalloc(const void* d_grads_half, int64_t n, float scale,
                                      float clip, mpt_check_result* d_result,
                                      void* cuda_stream)
{
    if (!d_grads_half || !d_result || n <= 0 ||
        (reinterpret_cast<uintptr_t>(d_grads_half) & 1) != 0 ||
        (reinterpret_cast<uintptr_t>(d_result) & 7) != 0)
        return MPT_ERR_INVALID_ARG;
    if (!finite(scale) || !(scale > 0.0f) || !finite(clip))
        return MPT_ERR_INVALID_ARG;
    if (n > MPT_NOALLOC_MAX_ELEMS)
        return MPT_ERR_TOO_LARGE;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MPT_ERR_CUDA;
    }
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return MPT_ERR_CUDA;
    unsigned char* scratch = nullptr;
    if (noalloc_scratch(dev, &scratch) != MPT_OK)
        return MPT_ERR_CUDA;

    // Each runtime call's own status is checked (not the thread's last-error
    // state, which may hold an error the caller has yet to collect); only an
    // error of this call is cleared.
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    // the counters must start at zero whatever the previous call left
    if (cudaMemsetAsync(scratch, 0, kNoAllocCtrlBytes, st) != cudaSuccess) {
        cudaGetLastError();
        return MPT_ERR_CUDA;
    }
    const float inv_scale = 1.0f / scale;
    int e2 = 0;
    const bool pow2 = std::frexp(scale, &e2) == 0.5f && (e2 - 1) >= -15 && (e2 - 1) <= 100;
    const double sq_unscale = pow2 ? std::ldexp(1.0, -2 * (e2 - 1)) : 0.0;
    const unsigned int bins = (unsigned int)((n + kNoAllocChunk - 1) / kNoAllocChunk);
    const uint16_t* g = static_cast<const uint16_t*>(d_grads_half);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(bins);
    lc.blockDim = dim3(kThreads);
    lc.stream = st;
    const cudaError_t e =
        pow2 ? cudaLaunchKernelEx(&lc, check_flat_kernel<true>, g, n, scratch, d_result, inv_scale, sq_unscale, clip)
             : cudaLaunchKernelEx(&lc, check_flat_kernel<false>, g, n, scratch, d_result, inv_scale, sq_unscale, clip);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MPT_ERR_CUDA;
    }
    return MPT_OK;
}
