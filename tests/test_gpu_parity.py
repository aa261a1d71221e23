"""GPU parity: libmpt (through its C ABI) against the CPU oracle, element by
element, on seeded inputs shaped like the five workloads, at sizes the oracle
finishes in seconds (several work bins and ragged tails each)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from workloads.configs import Config as WConfig, TensorSpec, miniature
from loss_scaled_fp32_b200 import (MPT, Config, MPT_FLAG_CHECKED, MPT_FLAG_COUNT_STALE,
                                   MPT_FLAG_GRAD_STATS)

from parity import Pair

pytestmark = pytest.mark.gpu


def custom(sizes, law=("log2_uniform", -30.0, -6.0), scale0=1024.0, growth_interval=0,
           clip=0.0, steps=3, seed=7, lr=0.01, momentum=0.9, weight_decay=1e-4, injections=None):
    tensors = [TensorSpec(f"t{i}", (int(s),), ("normal", 0.05)) for i, s in enumerate(sizes)]
    return WConfig(name="custom", tensors=tensors, grad_law=law, scale0=scale0,
                   growth_interval=growth_interval, lr=lr, momentum=momentum,
                   weight_decay=weight_decay, clip=clip, steps=steps, seed=seed,
                   injections=injections or (lambda step: []))


# ---------------------------------------------------------------------------
# the five workloads (reduced where the oracle would take minutes)
# ---------------------------------------------------------------------------

def test_flat1m_full_with_overflow_step():
    cfg = W.get("flat1m")
    p = Pair(cfg)
    scales = []
    for _ in range(cfg.steps):
        r, _ = p.step()
        scales.append(r["new_scale"])
    assert scales == [1024.0] * 4 + [512.0] * 6          # backoff at step 5, no growth
    assert p.bitexact_steps == cfg.steps + 1


def test_resnet50_first_steps():
    cfg = W.get("resnet50")
    p = Pair(cfg)
    for _ in range(3):
        r, _ = p.step()
        assert r["found_inf"] == 0
    assert p.bitexact_steps == 4


def test_gpt2_medium_sample_dynamic_scale_and_clip():
    cfg = miniature("gpt2_medium")
    p = Pair(cfg)
    clipped = 0
    for i in range(8):
        # a threshold below the norm of the sample exercises the clip path
        r, ro = p.step(clip=0.05)
        clipped += r["clipped"]
    assert clipped > 0


def test_gpt_1p3b_sample():
    cfg = miniature("gpt_1p3b")
    p = Pair(cfg)
    for _ in range(3):
        p.step()


def test_ragged_sample_with_unaligned_pointers_and_injections():
    full = W.get("ragged20k")
    sizes = W.configs.ragged_sizes(n=3000, seed=11, log_max=14)
    plan = {2: [(5, 0, 0x7C00)], 4: [(100, int(sizes[100]) - 1, 0xFC00)],
            7: [(2999, int(sizes[2999]) // 2, 0x7E00)]}
    cfg = custom(sizes, law=full.grad_law, scale0=2.0 ** 10, growth_interval=4, steps=10,
                 injections=lambda s: plan.get(s, []))
    shifted = set(range(0, 3000, 3))
    p = Pair(cfg, shifted=shifted)
    found = []
    for _ in range(cfg.steps):
        r, _ = p.step()
        found.append(r["found_inf"])
    assert found[1] == 1 and found[3] == 1 and found[6] == 1


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [2048 * 2048, 2048 * 2048 + 1, 2110 * 2048 + 5])
def test_partial_sum_levels_at_their_boundary(n):
    """2 048-element check bins over one tensor: exactly 2 048 bins (the
    largest list whose per-bin partials the update kernel adds directly),
    2 049 bins (the smallest with sums per group of 64 bins: 33 groups, the
    last of one bin) and 2 111 bins (a last group of 63).  The check kernel
    and the host must choose the same level; a clipped, an overflowing and
    another clipped step match the oracle (bit for bit where the two clip
    coefficients agree, as everywhere)."""
    plan = {2: [(0, n - 1, 0x7C00)]}
    cfg = custom([n], law=("log2_uniform", -26.0, -4.0), scale0=2.0 ** 12, clip=0.05, steps=3,
                 injections=lambda s: plan.get(s, []))
    p = Pair(cfg, chunk=2048)
    found, clipped = [], []
    for _ in range(cfg.steps):
        r, _ = p.step()
        found.append(r["found_inf"])
        clipped.append(r["clipped"])
    assert found == [0, 1, 0] and clipped == [1, 0, 1]


def test_an_abandoned_sharded_check_leaves_nothing_for_the_next_step():
    """A check pass queued by mpt_step_partial whose step is never finished
    (no mpt_step_finish follows) must leave no count, flag or statistic
    behind: the whole steps after it match the oracle for their own gradients
    alone (range counts, non-finite count, histogram, state)."""
    cfg = custom([70_001, 999, 4097], growth_interval=2, steps=2)
    p = Pair(cfg, flags=MPT_FLAG_GRAD_STATS)
    junk = p.grads(9, p.scale)
    junk[5] = 0x7C00                 # +inf
    junk[10:200] = 0                 # zeros
    junk[300:400] = 1                # the smallest subnormal
    p.flat.copy_(junk)
    p.opt.step_partial(p.gviews)
    torch.cuda.synchronize()
    for _ in range(cfg.steps):
        r, _ = p.step()
        assert r["found_inf"] == 0


@pytest.mark.parametrize("sizes", [[1], [2, 3], list(range(1, 18)), [7] * 5000,
                                   [1024, 1025, 1023], [32768], [32769, 32767, 65536 + 5],
                                   [200_003]])
def test_edge_sizes(sizes):
    p = Pair(custom(sizes, steps=2))
    p.step()
    p.step()


@pytest.mark.parametrize("shift", [0, 1, 2, 3, 4, 5, 6, 7])
def test_unaligned_gradient_pointers(shift):
    # 2-, 4-, 6-, 8-, ... byte offsets: the check pass's per-thread head
    # before the first 16-byte boundary, the update's shifted gradient words
    # (0-3 elements past an 8-byte boundary) and its scalar first quad and
    # tail; update bins of 1025 elements and tails of 1, 5, 7 and 8 elements
    cfg = custom([10_000, 70_001, 33, 1025, 4097, 4101, 4103, 4104, 4105], steps=2)
    p = Pair(cfg)
    for step in (1, 2):
        host = p.grads(step, p.scale)
        # every tensor placed `shift` elements after its aligned offset
        flat = torch.zeros(p.layout.total + 64, dtype=torch.int16, device="cuda")
        views = []
        for off, n, hv in zip(p.layout.offsets, p.layout.sizes, p.layout.views(host)):
            flat[off + shift: off + shift + n].copy_(hv)
            views.append(flat[off + shift: off + shift + n])
        p.step(host=host, gpu_grads=views)


@pytest.mark.parametrize("scale", [1000.0, 3.0, 2.0 ** -20, 2.0 ** 40, 0.7])
def test_non_power_of_two_and_extreme_scales(scale):
    cfg = custom([50_000, 999, 4097], law=("log2_uniform", -40.0, -20.0), scale0=scale, steps=2)
    p = Pair(cfg)
    p.step()
    p.step()


@pytest.mark.parametrize("scale,law", [
    (2.0 ** -15, (-9.0, 30.0)),     # lowest exponent of the exact power-of-two path
    (2.0 ** -16, (-8.0, 31.0)),     # just below it: binary32 products first
    (2.0 ** 100, (-124.0, -85.0)),  # highest exponent of the power-of-two path
    (2.0 ** 101, (-125.0, -86.0)),  # just above it
    (2.0 ** 127, (-151.0, -112.0)), # 1/S subnormal: products round in the subnormal range
])
def test_scale_exponent_edges(scale, law):
    """S = 2^e at and beyond the ends of the range where the check pass sums
    the squares of the scaled gradients and multiplies by 2^(-2e) once; the
    gradients are drawn so that |g S| spans the binary16 range."""
    cfg = custom([50_000, 999, 70_001], law=("log2_uniform",) + law, scale0=scale, steps=2)
    p = Pair(cfg)
    p.step()
    p.step()


def test_huge_inverse_scale_overflows_products_not_the_check():
    """S = 2^-120: the binary32 products fp32(g16) * (1/S) of the larger
    gradients overflow to inf although every gradient is finite.  The
    definition then has an infinite sum of squares, but no non-finite
    gradient: the step is not skipped, and the state (with its infinities,
    no NaN after one step from zero momentum) matches the oracle bit for bit."""
    cfg = custom([70_000, 3001], law=("log2_uniform", 112.0, 130.0), scale0=2.0 ** -120, steps=1)
    p = Pair(cfg)
    host = p.grads(1, p.scale)
    p.flat.copy_(host)
    hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
    r = p.opt.step(p.gviews, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay, 0.0)
    ro = oracle.step(p.state, hv, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay, clip=0.0,
                     cfg=p.ocfg)
    assert ro["found_inf"] == 0 and r["found_inf"] == 0 and r["n_nonfinite"] == 0
    assert math.isinf(ro["norm"]) and math.isinf(r["grad_norm"]) and r["clip_coef"] == 1.0
    assert r["n_zero"] == ro["n_zero"] and r["n_subnormal"] == ro["n_subnormal"]
    assert r["new_scale"] == ro["new_scale"]
    p.compare_state("huge 1/S", exact=True)


def test_huge_inverse_scale_with_one_inf_gradient_is_skipped():
    """The same S = 2^-120, now with one +inf gradient in the second tensor:
    some bins' sums are +inf from overflowing products alone, one bin holds a
    non-finite gradient.  Only the latter makes the step an overflow step: it
    is skipped, the non-finite count is exact and the state stays bitwise
    unchanged, as in the oracle."""
    cfg = custom([70_000, 3001], law=("log2_uniform", 112.0, 130.0), scale0=2.0 ** -120, steps=1)
    p = Pair(cfg)
    host = p.grads(1, p.scale)
    host[p.layout.offsets[1] + 1234] = 0x7C00
    p.flat.copy_(host)
    hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
    r = p.opt.step(p.gviews, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay, 1.0)
    ro = oracle.step(p.state, hv, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay, clip=1.0,
                     cfg=p.ocfg)
    assert ro["found_inf"] == 1 and r["found_inf"] == 1
    assert r["n_nonfinite"] == ro["n_nonfinite"] == 1
    assert math.isinf(r["grad_norm"]) and r["clip_coef"] == 1.0
    assert r["n_zero"] == ro["n_zero"] and r["n_subnormal"] == ro["n_subnormal"]
    assert r["new_scale"] == ro["new_scale"]
    p.compare_state("huge 1/S, one inf", exact=True)


def test_steps_write_nothing_outside_the_tensors():
    """Guard canaries: every byte of the master, momentum and FP16 arenas that
    belongs to no tensor (the 16-element padding after each tensor and the
    alignment gaps between the arenas) is filled with a pattern after the FP16
    refresh; steps over chunk bins with ragged tails, packed bins, an
    overflow step and a clipped step must leave every one of them intact."""
    plan = {3: [(2, 100, 0x7C00)]}
    sizes = [1, 17, 1025, 4097, 70_001, 3, 65_536 + 5, 1000]
    cfg = custom(sizes, law=("log2_uniform", -26.0, -4.0), scale0=2.0 ** 12, growth_interval=2,
                 clip=0.05, steps=5, injections=lambda s: plan.get(s, []))
    p = Pair(cfg)
    ws = p.opt.workspace
    base = ws.data_ptr()
    spans = []
    for i in range(len(sizes)):
        for t in (p.opt.master(i), p.opt.momentum(i), p.opt.w16(i)):
            spans.append((t.data_ptr() - base, t.data_ptr() - base + t.numel() * t.element_size()))
    spans.sort()
    gaps = [(a_end, b_start) for (_, a_end), (b_start, _) in zip(spans, spans[1:]) if b_start > a_end]
    tail = (spans[-1][1], (spans[-1][1] + 31) // 32 * 32)       # the last tensor's padding
    if tail[1] > tail[0]:
        gaps.append(tail)
    assert len(gaps) >= len(sizes)                                # at least one per tensor
    idx = torch.cat([torch.arange(a, b, device="cuda") for a, b in gaps])
    pattern = (torch.arange(idx.numel(), device="cuda") * 37 % 251 + 3).to(torch.uint8)
    ws[idx] = pattern
    torch.cuda.synchronize()
    for _ in range(cfg.steps):
        p.step()
    assert p.bitexact_steps >= 3
    assert torch.equal(ws[idx], pattern)


def test_injected_launch_failure_breaks_the_handle():
    """The test hook makes the next step fail as a failed kernel launch would
    (no CUDA call, no GPU fault): MPT_ERR_CUDA, then MPT_ERR_BROKEN for every
    later call; the handle can still be destroyed."""
    from loss_scaled_fp32_b200 import MptError
    cfg = custom([5000, 33], steps=2)
    p = Pair(cfg)
    p.step()
    p.opt.debug_fail_next_step()
    with pytest.raises(MptError) as e:
        p.opt.step(p.gviews, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay)
    assert e.value.code == -3                                     # MPT_ERR_CUDA
    for call in (lambda: p.opt.step(p.gviews, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay),
                 lambda: p.opt.step_async(p.gviews, cfg.lr, cfg.momentum, cfg.weight_decay),
                 lambda: p.opt.wait()):
        with pytest.raises(MptError) as e:
            call()
        assert e.value.code == -5                                 # MPT_ERR_BROKEN
    p.opt.close()


def test_checked_mode_and_stale_counts():
    cfg = custom([100_000, 17, 3000], steps=3, lr=1e-3)
    p = Pair(cfg, flags=MPT_FLAG_CHECKED | MPT_FLAG_COUNT_STALE)
    for _ in range(3):
        r, ro = p.step()
        assert r["n_fp16_stale"] == ro["n_stale"]
        assert r["n_fp16_stale"] > 0


@pytest.mark.parametrize("chunk", [2048, 4096, 1 << 20])
def test_chunk_sizes(chunk):
    cfg = custom([300_000, 5, 2049, 100_000], steps=2)
    p = Pair(cfg, chunk=chunk)
    p.step()
    p.step()


@pytest.mark.parametrize("pattern", [0x7C00, 0xFC00, 0x7E00, 0x7C01, 0xFFFF])
def test_overflow_leaves_state_bitwise_unchanged(pattern):
    cfg = custom([40_000, 3, 1500], steps=2)
    p = Pair(cfg)
    p.step()
    before = [x.copy() for x in sum(p.gpu_state(), [])]
    host = p.grads(2, p.scale)
    host[p.layout.offsets[2] + 1499] = pattern - 65536 if pattern >= 0x8000 else pattern
    r, _ = p.step(host=host)
    assert r["found_inf"] == 1 and r["n_nonfinite"] == 1 and math.isinf(r["grad_norm"])
    after = sum(p.gpu_state(), [])
    assert all(a.tobytes() == b.tobytes() for a, b in zip(before, after))


def test_all_zero_and_all_subnormal_gradients():
    cfg = custom([10_000, 333], steps=1)
    p = Pair(cfg)
    host = torch.zeros(p.layout.total, dtype=torch.int16)
    r, _ = p.step(host=host)
    assert r["n_zero"] == 10_333 and r["grad_norm"] == 0.0
    host = torch.full((p.layout.total,), 0x0123, dtype=torch.int16)
    r, _ = p.step(host=host)
    assert r["n_subnormal"] == 10_333


def test_determinism_bitwise():
    cfg = miniature("gpt2_medium")
    runs = []
    for _ in range(2):
        p = Pair(cfg)
        out = [p.step(clip=0.05)[0]["grad_norm"] for _ in range(3)]
        runs.append((out, [x.tobytes() for x in sum(p.gpu_state(), [])]))
    assert runs[0] == runs[1]


def test_checkpoint_resume_matches_straight_run():
    cfg = custom([123_457, 64, 4096], growth_interval=2, scale0=2.0 ** 14, steps=10,
                 law=("log2_uniform", -24.0, 1.0))
    straight = Pair(cfg)
    for _ in range(10):
        straight.step()
    a = Pair(cfg)
    for _ in range(5):
        a.step()
    # save: master + momentum (the workspace arenas) and the scaler state
    saved = [(a.opt.master(i).clone(), a.opt.momentum(i).clone()) for i in range(3)]
    scale, clean = a.opt.scaler_state()
    b = Pair(cfg)
    for i, (m, v) in enumerate(saved):
        b.opt.master(i).copy_(m)
        b.opt.momentum(i).copy_(v)
    b.opt.refresh_half()
    b.opt.set_scaler_state(scale, clean)
    b.state, b.scale, b.step_no = a.state, scale, 5
    for _ in range(5):
        b.step()
    s1 = [x.tobytes() for x in sum(straight.gpu_state(), [])]
    s2 = [x.tobytes() for x in sum(b.gpu_state(), [])]
    assert s1 == s2
    assert straight.opt.scaler_state() == b.opt.scaler_state()


def test_stats_and_timing():
    cfg = custom([70_000], steps=3)
    p = Pair(cfg)
    p.opt.set_timing(True)
    for _ in range(3):
        p.step()
    st = p.opt.stats()
    assert st["steps"] == 3 and st["timed_steps"] == 3
    assert st["check_ms_total"] > 0 and st["update_ms_total"] > 0
    assert st["scale"] == p.scale
    # sampled: every third step from the next one on
    p.opt.set_timing(3)
    for _ in range(7):
        p.step()
    assert p.opt.stats()["timed_steps"] == 3 + 3
    p.opt.set_timing(0)
    p.step()
    assert p.opt.stats()["timed_steps"] == 6


# ---------------------------------------------------------------------------
# queued (asynchronous) steps with the loss scale kept on the device
# ---------------------------------------------------------------------------

def test_cuda_graph_replays_follow_the_oracle():
    """One queued step captured into a CUDA graph and replayed: the gradient
    pointers are those of the step before, so the capture holds the two
    kernel launches only (no pointer-table copy); each replay reads and
    advances the device scale state and the gradients the buffers hold at
    replay time.  Every replay must match the oracle, overflow steps too."""
    plan = {4: [(1, 7, 0x7C00)]}
    cfg = custom([60_000, 1031, 5, 40_000], law=("log2_uniform", -26.0, -2.0), scale0=2.0 ** 12,
                 growth_interval=2, clip=0.3, steps=8, injections=lambda s: plan.get(s, []))
    p = Pair(cfg)
    p.step()                                   # uploads the pointer table of p.gviews
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        p.opt.step_async(p.gviews, cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip, stream=side)
    torch.cuda.synchronize()
    skipped = 0
    for _ in range(5):
        p.step_no += 1
        host = p.grads(p.step_no, p.scale)
        p.flat.copy_(host)
        torch.cuda.synchronize()
        graph.replay()
        r = p.opt.wait()
        hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
        ro = oracle.step(p.state, hv, p.scale, cfg.lr, cfg.momentum, cfg.weight_decay,
                         clip=cfg.clip, cfg=p.ocfg, flags=p.oflags, eps=p.eps)
        p.compare_result(r, ro)
        p.compare_state(f"replay {p.step_no}", exact=(r["clip_coef"] == ro["clip_coef"]))
        p.scale = r["new_scale"]
        skipped += r["found_inf"]
    assert skipped == 1
    del graph


def test_async_steps_follow_the_oracle():
    """Steps queued back to back with mpt_step_async: S is read from and
    advanced on the device; each step's gradients are drawn at the S the
    oracle's state machine predicts, so the device must agree with it."""
    plan = {3: [(1, 7, 0x7C00)], 8: [(0, 0, 0x7E00)]}
    cfg = custom([60_000, 1031, 5, 40_000], law=("log2_uniform", -26.0, -2.0), scale0=2.0 ** 12,
                 growth_interval=2, clip=0.3, steps=10, injections=lambda s: plan.get(s, []))
    p = Pair(cfg)
    ocfg, S, clean = p.ocfg, cfg.scale0, 0
    bufs = []
    for k in range(1, cfg.steps + 1):
        host = p.grads(k, S)
        dev = host.cuda()
        bufs.append(dev)                       # must outlive the queued step
        p.opt.step_async(p.layout.views(dev), cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip)
        hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
        ro = oracle.step(p.state, hv, S, cfg.lr, cfg.momentum, cfg.weight_decay, clip=cfg.clip,
                         cfg=ocfg)
        S = ro["new_scale"]
    r = p.opt.wait()
    assert r["new_scale"] == S and p.opt.scaler_state() == (S, p.state.clean_run)
    assert p.opt.device_scale().item() == S
    st = p.opt.stats()
    assert st["steps"] == cfg.steps and st["skipped"] == 2
    p.compare_state("after queued steps", exact=True)


def test_queued_steps_over_more_buffer_sets_than_cached_tables():
    """Queued steps that cycle through five gradient buffers, one more than
    the four pointer tables the handle keeps on the device: steps that reuse
    a cached table queue no copy, a fifth buffer set rewrites the least
    recently used table.  Every step must follow the oracle (the device state
    is compared bit for bit at the end), one of them an overflow."""
    plan = {7: [(2, 3, 0x7C00)]}
    cfg = custom([30_000, 1031, 7, 20_000], law=("log2_uniform", -26.0, -4.0), scale0=2.0 ** 12,
                 growth_interval=3, clip=0.3, steps=14, injections=lambda s: plan.get(s, []))
    p = Pair(cfg)
    bufs = [torch.zeros(p.layout.total, dtype=torch.int16, device="cuda") for _ in range(5)]
    S, skipped = cfg.scale0, 0
    order = [0, 1, 2, 3, 4, 0, 1, 4, 2, 0, 3, 3, 1, 0]
    for k, b in enumerate(order, start=1):
        host = p.grads(k, S)
        torch.cuda.current_stream().synchronize()      # earlier steps are done with bufs[b]
        bufs[b].copy_(host)
        p.opt.step_async(p.layout.views(bufs[b]), cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip)
        hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
        ro = oracle.step(p.state, hv, S, cfg.lr, cfg.momentum, cfg.weight_decay, clip=cfg.clip,
                         cfg=p.ocfg)
        S = ro["new_scale"]
        skipped += ro["found_inf"]
    r = p.opt.wait()
    assert skipped == 1 and r["new_scale"] == S
    assert p.opt.stats()["steps"] == len(order) and p.opt.stats()["skipped"] == 1
    p.compare_state("after steps over five buffer sets", exact=True)


def test_stale_total_over_queued_steps():
    """With MPT_FLAG_COUNT_STALE, the running total of stale FP16 elements
    (master moved, rounded copy did not) must count every step queued between
    two waits, not only the last one; an overflow step adds nothing."""
    plan = {3: [(0, 11, 0x7C00)]}
    cfg = custom([60_000, 1031, 5, 40_000], law=("log2_uniform", -26.0, -6.0), scale0=2.0 ** 12,
                 growth_interval=0, lr=1e-3, steps=6, injections=lambda s: plan.get(s, []))
    p = Pair(cfg, flags=MPT_FLAG_COUNT_STALE)
    S, per_step, bufs = cfg.scale0, [], []
    for k in range(1, 6):
        host = p.grads(k, S)
        dev = host.cuda()
        bufs.append(dev)
        p.opt.step_async(p.layout.views(dev), cfg.lr, cfg.momentum, cfg.weight_decay)
        hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
        ro = oracle.step(p.state, hv, S, cfg.lr, cfg.momentum, cfg.weight_decay, cfg=p.ocfg)
        per_step.append(ro["n_stale"])
        S = ro["new_scale"]
    r = p.opt.wait()
    assert per_step[2] == 0 and min(per_step[:2] + per_step[3:]) > 0
    assert r["n_fp16_stale"] == per_step[-1]
    assert p.opt.stats()["n_fp16_stale_total"] == sum(per_step)
    # a waiting step after the queued ones adds its own count
    r2, ro2 = p.step()
    assert r2["n_fp16_stale"] == ro2["n_stale"]
    assert p.opt.stats()["n_fp16_stale_total"] == sum(per_step) + ro2["n_stale"]
    p.compare_state("after queued stale steps", exact=True)


def test_sync_and_async_steps_share_the_scale_state():
    cfg = custom([30_000], scale0=2.0 ** 8, growth_interval=1, steps=4)
    p = Pair(cfg)
    r, _ = p.step()                            # S = 2^8 given by the host
    assert r["new_scale"] == 2.0 ** 9
    assert p.opt.device_scale().item() == 2.0 ** 9
    host = p.grads(2, 2.0 ** 9)
    dev = host.cuda()
    p.opt.step_async(p.layout.views(dev), cfg.lr, cfg.momentum, cfg.weight_decay)
    hv = [v.numpy().view(np.uint16) for v in p.layout.views(host)]
    oracle.step(p.state, hv, 2.0 ** 9, cfg.lr, cfg.momentum, cfg.weight_decay, cfg=p.ocfg)
    assert p.opt.wait()["new_scale"] == 2.0 ** 10
    p.compare_state("mixed", exact=True)
    p.opt.set_scaler_state(3.0, 0)             # any S, also not a power of two
    assert p.opt.device_scale().item() == 3.0


# ---------------------------------------------------------------------------
# gradient statistics and the direct choice of S
# ---------------------------------------------------------------------------

from loss_scaled_fp32_b200 import MPT_FLAG_GRAD_STATS  # noqa: E402


def test_grad_statistics_ragged_unaligned_with_overflow():
    """Largest finite |g16| (unscaled) and the exponent-field histogram, exact,
    over packed and chunked bins, unaligned pointers and inf/NaN steps."""
    sizes = W.configs.ragged_sizes(n=800, seed=5, log_max=15)
    plan = {2: [(3, 0, 0x7C00), (700, 0, 0x7E00)]}
    cfg = custom(sizes, law=("log2_uniform", -30.0, 0.0), scale0=2.0 ** 10, growth_interval=2,
                 steps=4, injections=lambda s: plan.get(s, []))
    p = Pair(cfg, shifted=set(range(0, 800, 5)), flags=MPT_FLAG_GRAD_STATS)
    for _ in range(cfg.steps):
        r, ro = p.step()
        assert sum(ro["exp_hist"]) == sum(sizes)
    assert any(p.opt.grad_histogram()[e] for e in range(1, 31))


@pytest.mark.parametrize("margin", [2.0, 1.5])
def test_direct_scaler_mode_follows_the_oracle(margin):
    plan = {4: [(1, 2, 0xFC00)]}
    cfg = custom([200_000, 77, 9000], law=("log2_normal", -14.0, 2.0), scale0=2.0 ** 8,
                 steps=8, clip=0.0, injections=lambda s: plan.get(s, []))
    p = Pair(cfg, direct_margin=margin)
    scales = []
    for _ in range(cfg.steps):
        r, ro = p.step()
        scales.append(r["new_scale"])
    assert len(set(scales)) > 2 and scales[3] == scales[2] * 0.5     # overflow at step 4


# ---------------------------------------------------------------------------
# Nesterov momentum and Adagrad
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("optimizer", ["nesterov", "adagrad"])
def test_optimizer_variants_follow_the_oracle(optimizer):
    sizes = W.configs.ragged_sizes(n=600, seed=9, log_max=16)
    plan = {3: [(10, 0, 0x7C00)]}
    cfg = custom(sizes, law=("log2_uniform", -26.0, -4.0), scale0=2.0 ** 12, growth_interval=2,
                 clip=0.2, steps=6, injections=lambda s: plan.get(s, []))
    p = Pair(cfg, shifted=set(range(1, 600, 7)), optimizer=optimizer)
    for _ in range(cfg.steps):
        p.step()
    assert p.bitexact_steps >= cfg.steps


@pytest.mark.parametrize("optimizer", ["nesterov", "adagrad"])
def test_optimizer_variants_gpt2_miniature(optimizer):
    p = Pair(miniature("gpt2_medium"), optimizer=optimizer, eps=1e-8)
    for _ in range(4):
        p.step(clip=0.05)
