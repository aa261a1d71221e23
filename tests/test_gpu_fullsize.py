"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (default chunking, one mpt_step call per step).

The whole step runs on the GPU over every parameter.  The oracle checks it
the way its definition allows at any size:
  * pass 1 of the oracle (overflow flag, range counts, sum of squares) runs
    over the FULL gradient list every step -> found_inf, the counts, the new S
    and the clean-step counter exact, the norm within 1e-5 relative;
  * pass 2 (the per-element update) runs on a sample of elements -- random
    positions plus the first and last element of every tensor -- whose FP32
    master, FP32 momentum and FP16 copy the oracle carries from step to step;
    they must match the GPU's bit for bit (whenever the two clip
    coefficients agree, which they do unless two summation orders of the
    binary64 norm straddle a binary32 rounding boundary).
The loss scale evolves as in training: each step's gradients are drawn at the
S the previous step returned, so overflow, backoff and growth happen
naturally (plus each workload's injected inf/NaN steps).
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from loss_scaled_fp32_b200 import (MPT, Config, MPT_FLAG_GRAD_STATS, MPT_SCALER_DIRECT,
                                   MPT_OPT_ADAGRAD, MPT_OPT_NESTEROV)

pytestmark = pytest.mark.gpu

THREADS = min(16, os.cpu_count() or 1)


class Sampled:
    def __init__(self, cfg, n_random=200_000, seed=0, mpt_kw=None, ocfg_kw=None, shifted=()):
        self.cfg = cfg
        sizes = np.array(cfg.sizes, dtype=np.int64)
        starts = np.concatenate([[0], np.cumsum(sizes)[:-1]])
        rng = np.random.default_rng(seed)
        idx = rng.integers(0, cfg.n_params, n_random)
        idx = np.unique(np.concatenate([idx, starts, starts + sizes - 1]))
        self.tensor = np.searchsorted(starts, idx, side="right") - 1
        self.elem = idx - starts[self.tensor]
        self.layout = W.GradLayout(cfg.sizes, shifted=shifted)
        mpt_kw = mpt_kw or {}
        self.opt = MPT(cfg.sizes, Config(backoff=cfg.backoff, growth=cfg.growth,
                                         growth_interval=cfg.growth_interval, **mpt_kw))
        self.hist = bool(mpt_kw.get("flags", 0) & MPT_FLAG_GRAD_STATS)
        self.oflags = {MPT_OPT_NESTEROV: oracle.NESTEROV,
                       MPT_OPT_ADAGRAD: oracle.ADAGRAD}.get(mpt_kw.get("optimizer", 0), 0)
        self.stats = self.hist or mpt_kw.get("scaler_mode", 0) == MPT_SCALER_DIRECT
        for i, m in enumerate(W.make_master(cfg, "cuda")):
            self.opt.master(i).copy_(m)
        self.opt.refresh_half()
        self.opt.set_scaler_state(cfg.scale0, 0)
        # flat arena views through the tensor views' addresses
        base = self.opt.master(0).data_ptr()
        arena_off = np.array([(self.opt.master(i).data_ptr() - base) // 4
                              for i in range(len(cfg.sizes))], dtype=np.int64)
        self.arena_idx = torch.from_numpy(arena_off[self.tensor] + self.elem).cuda()
        total = int(arena_off[-1] + sizes[-1])
        self.m_flat = self.opt.master(0).view(-1).as_strided((total,), (1,))
        self.v_flat = self.opt.momentum(0).view(-1).as_strided((total,), (1,))
        self.h_flat = self.opt.w16(0).view(-1).as_strided((total,), (1,))
        m, v, h = self.gather()
        assert np.array_equal(h, oracle.rne16(m))
        self.w, self.v, self.h = m, v, h
        self.grad_idx = torch.from_numpy(np.array(self.layout.offsets)[self.tensor] + self.elem).cuda()
        self.ocfg = oracle.scaler_cfg(backoff=cfg.backoff, growth=cfg.growth,
                                      growth_interval=cfg.growth_interval, **(ocfg_kw or {}))
        self.scale = cfg.scale0
        self.clean = 0
        self.flat = torch.zeros(self.layout.total, dtype=torch.int16, device="cuda")
        self.views = self.layout.views(self.flat)
        self.host = torch.empty(self.layout.total, dtype=torch.int16, pin_memory=True)

    def gather(self):
        m = self.m_flat.index_select(0, self.arena_idx).cpu().numpy()
        v = self.v_flat.index_select(0, self.arena_idx).cpu().numpy()
        h = self.h_flat.index_select(0, self.arena_idx).cpu().numpy().view(np.uint16)
        return m, v, h

    def full_check(self, scale):
        """Oracle pass 1 over every tensor (threads over groups of tensors; the
        binary64 partials are added in list order)."""
        hv = [v.numpy().view(np.uint16) for v in self.layout.views(self.host)]
        groups = np.array_split(np.arange(len(hv)), min(THREADS, len(hv)))
        res = list(ThreadPoolExecutor(THREADS).map(
            lambda g: oracle.check([hv[i] for i in g], scale), groups))
        total = res[0]
        for r in res[1:]:
            total.found_inf |= r.found_inf
            total.n_zero += r.n_zero
            total.n_subnormal += r.n_subnormal
            total.n_nonfinite += r.n_nonfinite
            total.sumsq += r.sumsq
            total.max_mag16 = max(total.max_mag16, r.max_mag16)
            total.max_abs = max(total.max_abs, r.max_abs)
            for b in range(32):
                total.exp_hist[b] += r.exp_hist[b]
        return total

    def step(self, k, queued=False):
        cfg = self.cfg
        W.make_grads(cfg, k, self.scale, self.layout, "cuda", out=self.flat)
        self.host.copy_(self.flat)
        if queued:
            # the benchmark's path: S is the device state the previous step left
            self.opt.step_async(self.views, cfg.lr, cfg.momentum, cfg.weight_decay, cfg.clip)
            r = self.opt.wait()
        else:
            r = self.opt.step(self.views, self.scale, cfg.lr, cfg.momentum, cfg.weight_decay,
                              cfg.clip)
        ro = oracle.clip_coef(self.full_check(self.scale), cfg.clip)
        for key in ("found_inf", "clipped", "n_zero", "n_subnormal", "n_nonfinite"):
            assert r[key] == getattr(ro, key), (k, key, r[key], getattr(ro, key))
        new_scale, self.clean = oracle.scaler_next(self.ocfg, ro.found_inf, self.scale, self.clean,
                                                   ro.max_abs)
        assert r["new_scale"] == new_scale and r["clean_run"] == self.clean, k
        if self.stats:
            assert r["max_abs_grad"] == ro.max_abs, (k, r["max_abs_grad"], ro.max_abs)
        if self.hist:
            assert self.opt.grad_histogram() == list(ro.exp_hist), k
        if ro.found_inf:
            assert math.isinf(r["grad_norm"])
        else:
            assert abs(r["grad_norm"] - ro.norm) <= 1e-5 * ro.norm
            g16 = self.flat.index_select(0, self.grad_idx).cpu().numpy().view(np.uint16)
            oracle.update(g16, self.w, self.v, self.h, self.scale, ro.clipped, ro.clip_coef,
                          cfg.lr, cfg.momentum, cfg.weight_decay, flags=self.oflags)
        m, v, h = self.gather()
        if r["clip_coef"] == ro.clip_coef:
            assert m.tobytes() == self.w.tobytes(), k
            assert v.tobytes() == self.v.tobytes(), k
            assert h.tobytes() == self.h.tobytes(), k
        else:  # one-ulp coefficient difference at a rounding boundary
            from parity import ulp_diff_f16, ulp_diff_f32
            assert ulp_diff_f32(m, self.w).max() <= 1 and ulp_diff_f32(v, self.v).max() <= 1
            assert ulp_diff_f16(h, self.h).max() <= 1
            self.w, self.v, self.h = m, v, h
        self.scale = r["new_scale"]
        return r


def run(name, steps=None, queued=False, **kw):
    cfg = W.get(name)
    s = Sampled(cfg, **kw)
    out = [s.step(k, queued) for k in range(1, (steps or cfg.steps) + 1)]
    s.opt.close()
    return out


def test_fullsize_resnet50():
    rs = run("resnet50")
    assert all(r["found_inf"] == 0 for r in rs)


def test_fullsize_gpt2_medium_dynamic_scale_and_clip():
    rs = run("gpt2_medium")
    assert any(r["found_inf"] for r in rs)           # S grows until it overflows
    assert any(r["clipped"] for r in rs)


def test_fullsize_gpt2_medium_queued_steps():
    """The benchmark's launch configuration: mpt_step_async with S kept on the
    device, default bins, full list."""
    rs = run("gpt2_medium", steps=16, queued=True)
    assert any(r["found_inf"] for r in rs)           # S reaches 2^18-2^19 by step 9-13


def test_fullsize_gpt2_medium_direct_scale_and_statistics():
    """Direct scaler mode (S from each step's largest gradient, so S is not a
    power of two: the check pass takes its binary32-product route) with the
    exponent histogram, over the full list: the largest magnitude, the
    histogram and each next S exact."""
    rs = run("gpt2_medium", steps=6,
             mpt_kw=dict(scaler_mode=MPT_SCALER_DIRECT, flags=MPT_FLAG_GRAD_STATS),
             ocfg_kw=dict(mode=oracle.SCALER_DIRECT))
    assert any(math.frexp(r["new_scale"])[0] != 0.5 for r in rs)


@pytest.mark.parametrize("optimizer", [MPT_OPT_NESTEROV, MPT_OPT_ADAGRAD])
def test_fullsize_gpt2_medium_optimizer_variants(optimizer):
    """Nesterov momentum and Adagrad over the full list (the Adagrad kernel
    runs at 3 CTAs per SM): sampled elements bit-exact with the oracle."""
    rs = run("gpt2_medium", steps=6, mpt_kw=dict(optimizer=optimizer))
    assert sum(r["found_inf"] == 0 for r in rs) >= 4     # mostly full updates


def test_fullsize_gpt_1p3b():
    rs = run("gpt_1p3b")
    assert all(r["found_inf"] == 0 for r in rs)


def test_fullsize_ragged20k():
    rs = run("ragged20k")
    assert sum(r["found_inf"] for r in rs) >= 20      # 20 injected + natural overflow


def test_fullsize_ragged20k_shifted_pointers():
    """The benchmark's misaligned case: every third gradient tensor starts 2
    bytes past an aligned address (the check pass's per-thread head, the
    update's shifted gradient words), queued steps over the full list."""
    cfg = W.get("ragged20k")
    rs = run("ragged20k", steps=8, queued=True, shifted=set(range(0, len(cfg.sizes), 3)))
    assert sum(r["found_inf"] == 0 for r in rs) >= 6
