#!/usr/bin/env python3
"""Benchmark: the loss-scaled FP32-master optimizer step (libmpt) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mpt|reference]
                    [--workload gpt2_medium]

One step = the whole step over the whole parameter list: the check kernel
(overflow flag, range counts, global sum of squares, loss-scale state) and the
fused update kernel (unscale, global-L2 clip, weight decay, momentum, FP32
master, FP16 copy).  The timed loop queues K steps with mpt_step_async (the
loss scale stays on the device, as in a training loop that multiplies its loss
by the device scalar) and waits once at the end; ``e2e`` uses the waiting
mpt_step, which also reads the 384-byte result back every step.  The workload
is the GPT-2-medium-shaped list (292 tensors, 354 823 168 parameters, clip
1.0): the first of the workloads at >= 100M parameters, the size the
80%-of-HBM target is set at.  Inputs are seeded synthetic FP16 gradients (two
sets drawn at S = 2^16, alternated) and random-initialised FP32 masters,
resident in HBM before timing; each step moves 7.8 GB, far more than the 126 MB
L2, so no L2 flush is needed.

Printed: one JSON line (rank 0).  ``value`` is whole-job params/s over the K
timed steps (CUDA events on the launching stream, max over ranks; N > 1 runs
independent replicas, one per GPU, since the step itself has no exchange);
``roofline`` reports the update kernel (the dominant one) against the measured
HBM copy bandwidth; ``e2e`` times the same step through the public API with the
gradients copied from pinned host memory every step; ``cpu_baseline`` times
the CPU oracle (single thread) on a bounded leading slice of the workload.

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
BYTES_UPDATE = 20        # per parameter: read g16 2 + w 4 + v 4, write w 4 + v 4 + w16 2
BYTES_CHECK = 2          # per parameter: read g16
TIMING_EVERY = 10       # kernel events on every 10th timed step
SKIP_STEPS = 20         # overflow steps timed apart
BYTES_SKIP = 4          # per parameter on an overflow step: check 2 + counting pass 2
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 2 ** 20
READBACK_BYTES = 384     # the control block mpt_step copies back each step
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mpt", "reference"], default="mpt")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
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
# the GPU arm
# ---------------------------------------------------------------------------

def run_mpt(args, cfg):
    import torch
    import torch.distributed as dist
    import workloads as W
    from loss_scaled_fp32_b200 import MPT, Config, grad_pointers

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    P = cfg.n_params
    # S stays at the workload's initial value while timing (the gradients are
    # drawn at that S once, before timing); the dynamic rule is exercised by
    # the tests, not by the timed loop
    opt = MPT(cfg.sizes, Config(growth_interval=0), device=dev)
    for i, m in enumerate(W.make_master(cfg, dev)):
        opt.master(i).copy_(m)
    opt.refresh_half()
    layout = W.GradLayout(cfg.sizes)
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

    for k in range(args.warmup):
        step(k)
    opt.wait(stream)
    clocks = ClockSampler(local) if rank == 0 else None
    time.sleep(0.3 if clocks else 0)                  # let nvidia-smi start sampling
    # per-kernel durations: CUDA events around the two kernels of every
    # TIMING_EVERY-th timed step (events on every step would cost the step
    # its overlap of the two kernels and three stream operations)
    opt.set_timing(TIMING_EVERY)
    before = opt.stats()
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.perf_counter()
    e0.record(stream)
    for k in range(args.steps):
        step(k)
    e1.record(stream)
    last = opt.wait(stream)
    torch.cuda.synchronize(dev)
    wall_ms = (time.perf_counter() - w0) * 1e3
    barrier()
    clock_info = clocks.stop() if clocks else None
    opt.set_timing(False)
    ms = e0.elapsed_time(e1)
    after = opt.stats()
    skipped = after["skipped"] - before["skipped"]
    clipped_last = last["clipped"]
    timed = after["timed_steps"] - before["timed_steps"]
    check_ms = (after["check_ms_total"] - before["check_ms_total"]) / timed
    update_ms = (after["update_ms_total"] - before["update_ms_total"]) / timed

    ms_max = ms
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())

    # overflow (skipped) steps, reported apart: one +inf planted in the
    # gradients, so every step takes the skip path -- the check pass plus the
    # update kernel's counting pass (4 B/param) -- and halves S on the device
    skip_steps = SKIP_STEPS
    flat0 = sets[0]
    saved = flat0[0].item()
    flat0[0] = 0x7C00
    for k in range(2):
        step(0)
    opt.wait(stream)
    s_before = opt.stats()["skipped"]
    barrier()
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for k in range(skip_steps):
        step(0)
    g1.record(stream)
    opt.wait(stream)
    torch.cuda.synchronize(dev)
    skip_ms = g0.elapsed_time(g1) / skip_steps
    skip_all = opt.stats()["skipped"] - s_before == skip_steps
    flat0[0] = saved
    opt.set_scaler_state(S, 0)
    if world > 1:
        t = torch.tensor([skip_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        skip_ms = float(t.item())

    # end to end through the public API: every step's gradients cross from
    # pinned host memory, and every step's result is read back to the host
    # (mpt_wait).  Two device gradient buffers: the copy of step k+1's
    # gradients runs on a second stream while step k computes, as a caller
    # feeding gradients from the host would arrange it.
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

    barrier()
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
    e2e_ms = f0.elapsed_time(f1) / max(1, args.e2e_steps)
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(cfg, args.cpu_seconds, dev)

    if rank == 0:
        peak, peak_kind = measured_peak()
        ms_step = ms_max / args.steps
        achieved_update = BYTES_UPDATE * P / (update_ms * 1e-3) / 1e9
        achieved_check = BYTES_CHECK * P / (check_ms * 1e-3) / 1e9
        traffic = load_traffic(P)
        line = {
            "metric": METRIC,
            "value": world * P / (ms_step * 1e-3),
            "unit": "params/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            # host wall clock around the same loop, through the final result read
            "wall_ms_per_step": wall_ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded FP16 gradients, random-init FP32 masters)",
            "hbm_gbs": (BYTES_UPDATE + BYTES_CHECK) * P / (ms_step * 1e-3) / 1e9,
            "hbm_frac_of_measured": (BYTES_UPDATE + BYTES_CHECK) * P / (ms_step * 1e-3) / 1e9 / peak,
            "hbm_frac_of_nominal_8tbs": (BYTES_UPDATE + BYTES_CHECK) * P / (ms_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
            "config": {"workload": cfg.name, "params": P, "tensors": len(cfg.sizes),
                       "bytes_per_param": BYTES_UPDATE + BYTES_CHECK,
                       "scale": S, "clip": cfg.clip, "lr": cfg.lr, "momentum": cfg.momentum,
                       "weight_decay": cfg.weight_decay, "grad_sets": len(sets),
                       "l2": l2_note(P),
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "last_step_clipped": clipped_last, "skipped_steps": skipped,
                       "api": "mpt_step_async (queued steps, S on the device)"},
            # isolated durations (a timed step's update starts after its check
            # ends); untimed steps overlap the two, so the remainder can be < 0
            "kernels_ms": {"check": check_ms, "update": update_ms,
                           "step_minus_kernels": ms_step - check_ms - update_ms,
                           "timed_steps": timed, "timed_every": TIMING_EVERY},
            "roofline": {"kernel": "update_kernel", "bound": "hbm",
                         "achieved": achieved_update, "peak": peak, "unit": "GB/s",
                         "frac": achieved_update / peak, "peak_kind": peak_kind,
                         "frac_of_nominal_8tbs": achieved_update / NOMINAL_HBM_GBS,
                         "traffic": traffic,
                         "algorithmic_bytes_per_launch": BYTES_UPDATE * P,
                         "check_kernel": {"achieved": achieved_check,
                                          "frac": achieved_check / peak,
                                          "algorithmic_bytes_per_launch": BYTES_CHECK * P}},
            "skipped_step": {"ms": skip_ms, "steps": skip_steps, "all_skipped": skip_all,
                             "bytes_per_param": BYTES_SKIP,
                             "gbs": BYTES_SKIP * P / (skip_ms * 1e-3) / 1e9},
            "e2e": {"value": world * P / (e2e_ms * 1e-3), "unit": "params/s",
                    "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": sets[0].numel() * 2,
                    "d2h_bytes_per_step": READBACK_BYTES,
                    "api": "mpt_step_async + mpt_wait per step; H2D of step k+1 on a "
                           "second stream overlapping step k"},
            "gpu_launches": 2 * args.steps,
            "clocks": clock_info,
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def load_traffic(n_params):
    """DRAM bytes per launch of the update kernel, scaled from the committed
    ncu summary (profiles/update_kernel_*.md: `dram_bytes_per_param = X`),
    if that summary was taken on the kernel source as it is now
    (`kernel_source_sha256 = ...`); else None."""
    import glob
    import re
    try:
        from loss_scaled_fp32_b200 import build as mbuild
        digest = mbuild.kernel_digest()
        for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "update_kernel_*.md"))):
            with open(path) as f:
                text = f.read()
            sha = re.search(r"kernel_source_sha256 = ([0-9a-f]{64})", text)
            per = re.search(r"dram_bytes_per_param = ([0-9.]+)", text)
            if sha and per and sha.group(1) == digest:
                return float(per.group(1)) * n_params
    except Exception:
        pass
    return None


def main():
    args = parse_args()
    import workloads as W
    from workloads.configs import truncated
    cfg = W.get(args.workload)
    if args.max_params:
        cfg = truncated(cfg, args.max_params)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_mpt(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
