#!/usr/bin/env python3
"""Benchmark: the loss-scaled FP32-master optimizer step (libmpt) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mpt|reference]
                    [--workload gpt2_medium] [--workloads a,b,...] [--sharded]

One step = the whole step over the whole parameter list: the check kernel
(overflow flag, range counts, global sum of squares, loss-scale state) and the
fused update kernel (unscale, global-L2 clip, weight decay, momentum, FP32
master, FP16 copy).  The timed loop queues K steps with mpt_step_async (the
loss scale stays on the device, as in a training loop that multiplies its loss
by the device scalar) and waits once at the end.  The headline workload is the
GPT-2-medium-shaped list (292 tensors, 354 823 168 parameters, clip 1.0): the
first of the workloads at >= 100M parameters, the size the 80%-of-HBM target is
set at.  Inputs are seeded synthetic FP16 gradients (two sets drawn at the
workload's initial S, alternated) and random-initialised FP32 masters,
resident in HBM before timing; each headline step moves 7.8 GB, far more than
the 126 MB L2, so no L2 flush is needed.

After the headline, the same measurement runs on the other workloads
(``per_workload``): the ResNet-50 list, the 1.3B-parameter list, the 20 000
ragged tensors, and the ragged list again with every third gradient pointer
2 bytes past an aligned address.

Per workload: ``ms_per_step`` from CUDA events around K queued steps (no kernel
events inside; a short GPU wait queued before the opening event lets the host
queue the first steps before the region starts); ``kernels_ms`` from a separate loop of at least 10 steps with
CUDA events around both kernels of every step (on the launching stream); the
overflow step (a +inf planted in the gradients: the check pass alone moves
data) timed apart; ``roofline`` for the update kernel (the dominant one)
against the measured HBM copy bandwidth, with the check kernel inside it, both
as timed in the step and alone (L2 cold, from a CUDA graph, without event
overhead, in the sharded step's form that also adds its own partials;
``kernels_ms.event_pair_floor`` is what two CUDA events with nothing between
them read).  ``e2e`` (headline) times the same
step through the public API with the gradients copied from pinned host memory
every step and each step's result read back; ``cpu_baseline`` times the CPU
oracle (single thread) on a bounded leading slice of the workload.

``--gpus N`` (under torchrun) runs N independent replicas, one per GPU: the
step has no exchange.  ``--sharded`` instead runs the sharded step (optimizer
state split across the ranks): NCCL reduce-scatter of the FP16 gradients, the
check pass over each rank's shard, an all-gather of the 32-byte records, the
combine-and-update, and the FP16 all-gather, with each phase timed.

``--impl reference`` times the CPU oracle instead, on host cores, on bounded
leading slices of the same workload (the oracle is the only reference
implementation of this path).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "params/sec and achieved HBM GB/s (fraction of B200 peak) per optimizer step"
DEFAULT_WORKLOAD = "gpt2_medium"
# the other workloads measured after the headline; "ragged20k_shift2B" is the
# ragged list with every third gradient pointer offset by 2 bytes
DEFAULT_EXTRA = "flat1m,resnet50,gpt_1p3b,ragged20k,ragged20k_shift2B"
BYTES_UPDATE = 20        # per parameter: read g16 2 + w 4 + v 4, write w 4 + v 4 + w16 2
BYTES_CHECK = 2          # per parameter: read g16
BYTES_SKIP = 2           # per parameter on an overflow step: the check pass only
MIN_KERNEL_STEPS = 10      # steps with kernel events, after the headline loop
ALONE_LAUNCHES = 10        # the check pass alone: launches per graph,
ALONE_REPLAYS = 5          # graph replays per timing,
SWEEP_BYTES = 512 << 20    # and the read sweep that evicts L2 before each launch
SKIP_STEPS = 20          # overflow steps timed apart
LEAD_CYCLES = 400_000    # GPU wait before a timed loop (about 0.2 ms at 1.9 GHz)
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 2 ** 20
READBACK_BYTES = 384     # the control block mpt_step copies back each step
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mpt", "reference"], default="mpt")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--workloads", default=DEFAULT_EXTRA,
                    help="comma-separated workloads measured after the headline ('' for none)")
    ap.add_argument("--sharded", action="store_true",
                    help="time the sharded step (NCCL collectives) instead of replicas")
    ap.add_argument("--max-params", type=int, default=0,
                    help="time only the leading N parameters of the workload (profiling)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="approximate CPU time spent timing the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def l2_note(P):
    moved = (BYTES_UPDATE + BYTES_CHECK) * P
    state = (4 + 4 + 2 + 2 * 2) * P    # master, momentum, FP16 copy, two gradient sets
    fits = "all state fits in L2 (L2-resident number)" if state <= L2_BYTES else "state larger than L2"
    return f"{moved / 1e9:.3g} GB moved per step, {state / 1e9:.3g} GB of state vs 126 MB L2: {fits}"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def load_traffic(kernel, n_params):
    """DRAM bytes per launch of ``kernel`` from the ncu figures committed in
    profiles/dram_traffic.json (bytes per parameter of one capture, scaled to
    ``n_params``), if they were taken on the device code as it is now;
    else (None, reason)."""
    try:
        from loss_scaled_fp32_b200 import build as mbuild
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[kernel]
        if rec["kernel_source_sha256"] != mbuild.kernel_digest():
            return None, "ncu figures predate the current kernel source"
        return float(rec["dram_bytes_per_param"]) * n_params, \
            f"ncu dram__bytes_read.sum + dram__bytes_write.sum, {rec['capture']}; " \
            f"bytes per parameter scaled to {n_params} parameters"
    except Exception as e:  # missing file or kernel entry
        return None, f"no ncu figures ({type(e).__name__})"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(gpu_index), "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s, p in zip(sm, power) if p >= 0.5 * max(power)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(cfg, max_params, device):
    """Inputs of a bounded leading slice of the workload, on the host."""
    import numpy as np
    import oracle
    import workloads as W
    from workloads.configs import truncated

    sub = truncated(cfg, max_params)
    layout = W.GradLayout(sub.sizes)
    grads = W.make_grads(sub, 1, sub.scale0, layout, device).cpu()
    hv = [v.numpy().view(np.uint16) for v in layout.views(grads)]
    master = [m.cpu().numpy() for m in W.make_master(sub, device)]
    return sub, hv, oracle.State.from_master(master)


def time_oracle(cfg, sub, hv, state, steps):
    import oracle
    ocfg = oracle.scaler_cfg(backoff=cfg.backoff, growth=cfg.growth,
                             growth_interval=cfg.growth_interval)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.step(state, hv, sub.scale0, cfg.lr, cfg.momentum, cfg.weight_decay,
                    clip=cfg.clip, cfg=ocfg)
        times.append(time.perf_counter() - t0)
    return times


def cpu_baseline(cfg, seconds, device):
    # ~25-40 M params/s on one core: size the slice for a few steps of ~1/4 s each
    sub, hv, state = oracle_sample(cfg, 8_000_000, device)
    time_oracle(cfg, sub, hv, state, 1)                         # warm-up
    per = statistics.median(time_oracle(cfg, sub, hv, state, 2))
    steps = max(3, int(seconds / max(per, 1e-3)))
    times = time_oracle(cfg, sub, hv, state, steps)
    total = sum(times)
    return {"value": sub.n_params * steps / total, "unit": "params/s", "cores": 1,
            "kind": "oracle",
            "sample": f"leading {sub.n_params} params of {cfg.name} ({len(sub.sizes)} tensors), "
                      f"{steps} steps, single-threaded C oracle",
            "host_cores": host_cores(), "cpu_model": cpu_model(), "seconds": total}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    device = "cuda" if torch.cuda.is_available() else "cpu"
    sub, hv, state = oracle_sample(cfg, 4_000_000, device)
    time_oracle(cfg, sub, hv, state, args.warmup)
    times = time_oracle(cfg, sub, hv, state, args.steps)
    total = sum(times)
    value = sub.n_params * args.steps / total
    sample = (f"each step: the leading {sub.n_params} params of {cfg.name} "
              f"({len(sub.sizes)} tensors), single-threaded C oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "params/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "params": cfg.n_params, "tensors": len(cfg.sizes),
                   "sample_params": sub.n_params},
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "host_cores": host_cores(), "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the GPU arm: one workload, replicas
# ---------------------------------------------------------------------------

class Ranks:
    """Rank bookkeeping and the few host-side collectives of the timing."""

    def __init__(self, world, rank, local, dev):
        self.world, self.rank, self.local, self.dev = world, rank, local, dev

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x):
        if self.world == 1:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=self.dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def without_injections(cfg):
    """The workload with its planted inf/NaN steps removed: the timed loops
    draw two gradient sets once and replay them, and the overflow step is
    timed apart."""
    import dataclasses
    return dataclasses.replace(cfg, injections=lambda step: [])


def workload_of(name):
    """(workload config, gradient pointers shifted?) for a workload name."""
    import workloads as W
    if name.endswith("_shift2B"):
        return W.get(name[:-len("_shift2B")]), True
    return W.get(name), False


def measure(cfg, args, R, shift=False, e2e=False, clocks=True):
    """Time the step over one workload on this rank's GPU.  Returns a dict of
    figures (times are the max over ranks)."""
    import torch
    import workloads as W
    from loss_scaled_fp32_b200 import MPT, Config, grad_pointers

    dev = R.dev
    cfg = without_injections(cfg)
    P = cfg.n_params
    # S stays at the workload's initial value while timing (the gradients are
    # drawn at that S once, before timing); the dynamic rule is exercised by
    # the tests, not by the timed loop
    opt = MPT(cfg.sizes, Config(growth_interval=0), device=dev)
    for i, m in enumerate(W.make_master(cfg, dev)):
        opt.master(i).copy_(m)
    opt.refresh_half()
    shifted = set(range(0, len(cfg.sizes), 3)) if shift else ()
    layout = W.GradLayout(cfg.sizes, shifted=shifted)
    sets = [W.make_grads(cfg, s, cfg.scale0, layout, dev) for s in (1, 2)]
    ptrs = [grad_pointers(layout.views(g)) for g in sets]
    S = cfg.scale0
    opt.set_scaler_state(S, 0)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    def step(k):
        # queued without a host wait; S is the device scale state
        opt.step_async(ptrs[k % 2], cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip,
                       stream=stream)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def lead():
        # a short GPU-side wait queued before a timed region's opening event:
        # by the time it ends the host has queued the first steps, so the
        # region holds no idle gap while the first launch is issued (the
        # wait itself lies before the region)
        torch.cuda._sleep(LEAD_CYCLES)

    for k in range(args.warmup):
        step(k)
    opt.wait(stream)

    # the headline loop: K queued steps, no kernel events inside
    sampler = ClockSampler(R.local) if (clocks and R.rank == 0) else None
    time.sleep(0.3 if sampler else 0)                 # let nvidia-smi start sampling
    R.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = ev(), ev()
    w0 = time.perf_counter()
    lead()
    e0.record(stream)
    for k in range(args.steps):
        step(k)
    e1.record(stream)
    last = opt.wait(stream)
    torch.cuda.synchronize(dev)
    wall_ms = (time.perf_counter() - w0) * 1e3
    R.barrier()
    clock_info = sampler.stop() if sampler else None
    ms_step = R.max(e0.elapsed_time(e1)) / args.steps
    skipped = last["found_inf"]

    # per-kernel durations: CUDA events around the two kernels of every step
    # of a separate loop (events inside the headline loop would cost it the
    # overlap of the two kernels and three stream operations per step); the
    # two kernels of such a step run one after the other, so these are
    # isolated durations
    ksteps = max(MIN_KERNEL_STEPS, min(args.steps, 50))
    opt.set_timing(1)
    before = opt.stats()
    for k in range(ksteps):
        step(k)
    opt.wait(stream)
    after = opt.stats()
    opt.set_timing(0)
    timed = after["timed_steps"] - before["timed_steps"]
    check_ms = R.max((after["check_ms_total"] - before["check_ms_total"]) / timed)
    update_ms = R.max((after["update_ms_total"] - before["update_ms_total"]) / timed)

    # the same step replayed from a CUDA graph (one gradient set, so the
    # pointers stay fixed and a queued step is only its two kernel launches):
    # the GPU-side step time without host launch gaps, which is what limits
    # the queued loop on the small lists
    gsteps, greps = 10, max(2, min(20, args.steps // 10))
    opt.step_async(ptrs[0], cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip, stream=stream)
    opt.wait(stream)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(gsteps):
            opt.step_async(ptrs[0], cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip,
                           stream=side)
    graph.replay()
    opt.wait(stream)
    R.barrier()
    torch.cuda.synchronize(dev)
    r0, r1 = ev(), ev()
    r0.record(stream)
    for _ in range(greps):
        graph.replay()
    r1.record(stream)
    opt.wait(stream)
    torch.cuda.synchronize(dev)
    ms_graph = R.max(r0.elapsed_time(r1)) / (greps * gsteps)
    del graph

    # overflow (skipped) steps, reported apart: one +inf planted in the
    # gradients, so every step takes the skip path -- the check pass reads
    # the gradients, each update CTA adds the check's partials, finds NaN and
    # exits -- and halves S on the device
    flat0 = sets[0]
    at = layout.offsets[0]
    saved = flat0[at].item()
    flat0[at] = 0x7C00
    for k in range(2):
        step(0)
    opt.wait(stream)
    s_before = opt.stats()["skipped"]
    R.barrier()
    torch.cuda.synchronize(dev)
    g0, g1 = ev(), ev()
    lead()
    g0.record(stream)
    for k in range(SKIP_STEPS):
        step(0)
    g1.record(stream)
    opt.wait(stream)
    torch.cuda.synchronize(dev)
    skip_ms = R.max(g0.elapsed_time(g1)) / SKIP_STEPS
    skip_all = opt.stats()["skipped"] - s_before == SKIP_STEPS
    flat0[at] = saved
    opt.set_scaler_state(S, 0)

    peak, peak_kind = measured_peak()
    achieved_update = BYTES_UPDATE * P / (update_ms * 1e-3) / 1e9
    achieved_check = BYTES_CHECK * P / (check_ms * 1e-3) / 1e9
    traffic_u, source_u = load_traffic("update_kernel", P)
    traffic_c, source_c = load_traffic("check_kernel", P)
    step_gbs = (BYTES_UPDATE + BYTES_CHECK) * P / (ms_step * 1e-3) / 1e9
    out = {
        "workload": cfg.name + ("_shift2B" if shift else ""),
        "params": P, "tensors": len(cfg.sizes),
        "shifted_pointers": len(shifted),
        "ms_per_step": ms_step,
        "value": R.world * P / (ms_step * 1e-3),
        "wall_ms_per_step": wall_ms / args.steps,
        "ms_per_step_graph": ms_graph,
        "graph_steps": greps * gsteps,
        "hbm_gbs": step_gbs,
        "hbm_frac_of_measured": step_gbs / peak,
        "hbm_frac_of_nominal_8tbs": step_gbs / NOMINAL_HBM_GBS,
        "steps": args.steps, "skipped_in_timed_loop": skipped,
        "clip": cfg.clip, "scale": S, "last_step_clipped": last["clipped"],
        "l2": l2_note(P),
        "kernels_ms": {"check": check_ms, "update": update_ms,
                       "step_minus_kernels": ms_step - check_ms - update_ms,
                       "timed_steps": timed, "timed_every": 1},
        "roofline": {"kernel": "update_kernel", "bound": "hbm",
                     "achieved": achieved_update, "peak": peak, "unit": "GB/s",
                     "frac": achieved_update / peak, "peak_kind": peak_kind,
                     "frac_of_nominal_8tbs": achieved_update / NOMINAL_HBM_GBS,
                     "traffic": traffic_u, "traffic_source": source_u,
                     "algorithmic_bytes_per_launch": BYTES_UPDATE * P,
                     "check_kernel": {"achieved": achieved_check,
                                      "frac": achieved_check / peak,
                                      "traffic": traffic_c, "traffic_source": source_c,
                                      "algorithmic_bytes_per_launch": BYTES_CHECK * P}},
        "skipped_step": {"ms": skip_ms, "steps": SKIP_STEPS, "all_skipped": skip_all,
                         "bytes_per_param": BYTES_SKIP,
                         "gbs": BYTES_SKIP * P / (skip_ms * 1e-3) / 1e9},
        "clocks": clock_info,
        "gpu_launches": 2 * args.steps,
    }
    if e2e:
        out["e2e"] = measure_e2e(cfg, args, R, opt, sets, ptrs, stream)

    # The check pass on its own, with L2 cold: before each launch a read-only
    # sweep of a 512 MB buffer (four times L2) evicts the gradients without
    # leaving dirty lines behind.  A CUDA graph of (sweep, check) pairs minus
    # a graph of the sweeps alone gives the check's cost per launch (its
    # launch included, no event overhead), and the median of three such
    # differences is reported.  mpt_step_partial queues the check kernel
    # alone as the sharded step runs it: it also adds its own partials
    # (atomic tickets, the 32-byte record), which a whole step leaves to the
    # update kernel, so it is an upper bound of the check in a whole step.
    # Run last: partial steps leave the handle's range counters to a finish
    # that never comes.
    sweep = torch.ones(SWEEP_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)

    def sweep_graph_ms(with_check):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for k in range(ALONE_LAUNCHES):
                torch.sum(sweep, dim=0, out=sink)
                if with_check:
                    opt.step_partial(ptrs[k % len(ptrs)], stream=side)
        graph.replay()
        torch.cuda.synchronize(dev)
        R.barrier()
        c0, c1 = ev(), ev()
        c0.record(stream)
        for _ in range(ALONE_REPLAYS):
            graph.replay()
        c1.record(stream)
        torch.cuda.synchronize(dev)
        del graph
        return R.max(c0.elapsed_time(c1)) / (ALONE_REPLAYS * ALONE_LAUNCHES)

    diffs = []
    for _ in range(3):
        with_check = sweep_graph_ms(True)
        diffs.append(with_check - sweep_graph_ms(False))
    iso_ms = statistics.median(diffs)
    # what a pair of CUDA events with nothing between them reads after such a
    # sweep: the part of an event-timed kernel duration that is not the kernel
    floor = []
    for _ in range(10):
        torch.sum(sweep, dim=0, out=sink)
        f0, f1 = ev(), ev()
        f0.record(stream)
        f1.record(stream)
        floor.append((f0, f1))
    torch.cuda.synchronize(dev)
    out["kernels_ms"]["event_pair_floor"] = R.max(statistics.median(a.elapsed_time(b) for a, b in floor))
    del sweep, sink
    iso_gbs = BYTES_CHECK * P / (iso_ms * 1e-3) / 1e9
    out["roofline"]["check_kernel"]["alone"] = {
        "ms": iso_ms, "achieved": iso_gbs, "frac": iso_gbs / peak,
        "how": ("check kernel alone with L2 cold: CUDA graph of %d (512 MB read sweep, "
                "mpt_step_partial) pairs minus the sweeps alone, median of 3; the sharded "
                "step's form of the pass, which also adds its own partials" % ALONE_LAUNCHES)}
    opt.close()
    del sets
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return out


def measure_e2e(cfg, args, R, opt, sets, ptrs, stream):
    """End to end through the public API: every step's gradients cross from
    pinned host memory, and every step's result is read back to the host
    (mpt_wait).  Two device gradient buffers: the copy of step k+1's
    gradients runs on a second stream while step k computes, as a caller
    feeding gradients from the host would arrange it."""
    import torch
    dev = R.dev
    P = cfg.n_params
    host = [torch.empty(g.numel(), dtype=torch.int16, pin_memory=True) for g in sets]
    for h, g in zip(host, sets):
        h.copy_(g)
    torch.cuda.synchronize(dev)
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def h2d(k):
        b = k % 2
        with torch.cuda.stream(copy_stream):
            if k >= 2:
                copy_stream.wait_event(consumed[b])   # step k-2 is done with buffer b
            sets[b].copy_(host[b], non_blocking=True)
            copied[b].record(copy_stream)

    R.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    copy_stream.wait_event(f0)
    h2d(0)
    for k in range(args.e2e_steps):
        b = k % 2
        stream.wait_event(copied[b])
        opt.step_async(ptrs[b], cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip, stream=stream)
        consumed[b].record(stream)
        if k + 1 < args.e2e_steps:
            h2d(k + 1)
        opt.wait(stream)                              # the step's result, on the host
    f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = R.max(f0.elapsed_time(f1) / max(1, args.e2e_steps))
    return {"value": R.world * P / (e2e_ms * 1e-3), "unit": "params/s",
            "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": sets[0].numel() * 2,
            "d2h_bytes_per_step": READBACK_BYTES,
            "api": "mpt_step_async + mpt_wait per step; H2D of step k+1 on a second stream "
                   "overlapping step k"}


def init_ranks(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1 or args.sharded:
        from datetime import timedelta
        if "MASTER_ADDR" not in os.environ:          # one process, no launcher
            import socket
            with socket.socket() as s:
                s.bind(("127.0.0.1", 0))
                os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(s.getsockname()[1]),
                                  RANK="0", WORLD_SIZE="1")
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    return Ranks(world, rank, local, dev)


def run_mpt(args, cfg):
    import torch.distributed as dist
    R = init_ranks(args)
    head = measure(cfg, args, R, e2e=True)
    extra = []
    if not args.max_params:
        for name in [w for w in args.workloads.split(",") if w]:
            wcfg, shift = workload_of(name)
            if wcfg.name == cfg.name and not shift:
                continue
            extra.append(measure(wcfg, args, R, shift=shift))

    base = None
    if R.rank == 0 and R.world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(cfg, args.cpu_seconds, R.dev)

    if R.rank == 0:
        P = cfg.n_params
        line = {
            "metric": METRIC,
            "value": head["value"],
            "unit": "params/s",
            "n_gpus": R.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"],
            # host wall clock around the same loop, through the final result read
            "wall_ms_per_step": head["wall_ms_per_step"],
            # the same step replayed from a CUDA graph (GPU-side time, no host gaps)
            "ms_per_step_graph": head["ms_per_step_graph"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded FP16 gradients, random-init FP32 masters)",
            "hbm_gbs": head["hbm_gbs"],
            "hbm_frac_of_measured": head["hbm_frac_of_measured"],
            "hbm_frac_of_nominal_8tbs": head["hbm_frac_of_nominal_8tbs"],
            "config": {"workload": cfg.name, "params": P, "tensors": len(cfg.sizes),
                       "bytes_per_param": BYTES_UPDATE + BYTES_CHECK,
                       "scale": head["scale"], "clip": cfg.clip, "lr": cfg.lr,
                       "momentum": cfg.momentum, "weight_decay": cfg.weight_decay,
                       "grad_sets": 2, "l2": head["l2"],
                       "parallelism": f"replicas x{R.world}" if R.world > 1 else "single GPU",
                       "last_step_clipped": head["last_step_clipped"],
                       "skipped_steps": head["skipped_in_timed_loop"],
                       "api": "mpt_step_async (queued steps, S on the device)"},
            "kernels_ms": head["kernels_ms"],
            "roofline": head["roofline"],
            "skipped_step": head["skipped_step"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"],
            "cpu_baseline": base,
            "per_workload": extra,
        }
        print(json.dumps(line), flush=True)
    if R.world > 1:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# the sharded step (optimizer state split across the ranks)
# ---------------------------------------------------------------------------

PHASES = ("reduce_scatter", "check", "record_allgather", "finish_update", "w16_allgather")


def run_sharded(args, cfg):
    import torch
    import torch.distributed as dist
    import workloads as W
    from loss_scaled_fp32_b200 import Config
    from loss_scaled_fp32_b200.sharded import ShardedMPT

    R = init_ranks(args)
    dev = R.dev
    cfg = without_injections(cfg)
    P = cfg.n_params
    opt = ShardedMPT(P, Config(growth_interval=0), device=dev)
    opt.load_master(torch.cat(W.make_master(cfg, dev)))
    # each rank's gradients of the whole list (contiguous, padded with zeros),
    # drawn at S / N: the FP16 sum over the N ranks then carries S, as with a
    # loss averaged over the data-parallel group
    S = cfg.scale0
    layout = W.GradLayout(cfg.sizes, align=1)
    sets = []
    for s in (1, 2):
        g = torch.zeros(opt.padded, dtype=torch.int16, device=dev)
        W.make_grads(cfg, 2 * R.rank + s, S / R.world, layout, dev, out=g)
        sets.append(g.view(torch.float16))
    opt.set_scale(S, 0)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    def step(k, marks=None):
        opt.step(sets[k % 2], cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip, marks=marks)

    for k in range(args.warmup):
        step(k)
    opt.wait()
    sampler = ClockSampler(R.local) if R.rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    R.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(LEAD_CYCLES)     # as in measure(): the host queues ahead
    e0.record(stream)
    for k in range(args.steps):
        step(k)
    e1.record(stream)
    last = opt.wait()
    torch.cuda.synchronize(dev)
    R.barrier()
    clock_info = sampler.stop() if sampler else None
    ms_step = R.max(e0.elapsed_time(e1)) / args.steps

    # phase durations of a separate loop: events on the step's stream at the
    # phase boundaries
    ksteps = max(MIN_KERNEL_STEPS, min(args.steps, 50))
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(len(PHASES) + 1)]
             for _ in range(ksteps)]
    R.barrier()
    for k in range(ksteps):
        step(k, marks[k])
    opt.wait()
    torch.cuda.synchronize(dev)
    phases = {}
    for i, name in enumerate(PHASES):
        phases[name] = R.max(sum(m[i].elapsed_time(m[i + 1]) for m in marks) / ksteps)
    kernels = phases["check"] + phases["finish_update"]

    # end to end: this rank's gradients copied from pinned host memory each
    # step, each step's result read back
    host = torch.empty(opt.padded, dtype=torch.float16, pin_memory=True)
    host.copy_(sets[0])
    R.barrier()
    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for k in range(args.e2e_steps):
        sets[0].copy_(host, non_blocking=True)
        step(0)
        opt.wait()
    f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = R.max(f0.elapsed_time(f1) / max(1, args.e2e_steps))

    if R.rank == 0:
        peak, peak_kind = measured_peak()
        shard = opt.shard
        upd_gbs = BYTES_UPDATE * shard / (phases["finish_update"] * 1e-3) / 1e9
        line = {
            "metric": METRIC,
            "value": P / (ms_step * 1e-3),
            "unit": "params/s",
            "n_gpus": R.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded FP16 gradients per rank, random-init FP32 masters)",
            "config": {"workload": cfg.name, "params": P, "tensors": len(cfg.sizes),
                       "parallelism": f"sharded x{R.world}", "shard_params": shard,
                       "scale": S, "clip": cfg.clip, "l2": l2_note(shard),
                       "api": "ShardedMPT.step: NCCL reduce-scatter, mpt_step_partial, "
                              "record all-gather, mpt_step_finish, FP16 all-gather"},
            "phases_ms": phases,
            "kernels_ms": {"check": phases["check"], "finish_update": phases["finish_update"],
                           "total": kernels, "timed_steps": ksteps},
            "collectives_ms": phases["reduce_scatter"] + phases["record_allgather"] +
                              phases["w16_allgather"],
            "roofline": {"kernel": "update_kernel (with the one-thread finish before it)",
                         "bound": "hbm", "achieved": upd_gbs, "peak": peak, "unit": "GB/s",
                         "frac": upd_gbs / peak, "peak_kind": peak_kind, "traffic": None,
                         "traffic_source": "not captured for the sharded step",
                         "algorithmic_bytes_per_launch": BYTES_UPDATE * shard},
            "e2e": {"value": P / (e2e_ms * 1e-3), "unit": "params/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": opt.padded * 2, "d2h_bytes_per_step": READBACK_BYTES,
                    "api": "H2D of this rank's gradients, ShardedMPT.step, mpt_wait"},
            "last_step_found_inf": last["found_inf"],
            "gpu_launches": 3 * args.steps,
            "clocks": clock_info,
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    opt.close()
    dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    import workloads as W
    from workloads.configs import truncated
    cfg = W.get(args.workload)
    if args.max_params:
        cfg = truncated(cfg, args.max_params)
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.sharded:
        return run_sharded(args, cfg)
    return run_mpt(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
