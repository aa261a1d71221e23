"""Shared harness of the parity tests: runs the CUDA library (through its C
ABI, via the Python binding) and the CPU oracle side by side on the same
seeded inputs and compares every output.

Tolerances (stated by the benchmark spec for this path, tightened where the arithmetic
allows): found_inf, S, the clean-step counter and the FP16 range counts
exact; global norm relative 1e-5; FP32 master and momentum within 1 binary32
ulp; FP16 copy within 1 binary16 ulp.  Both sides round every binary32
operation the same way and reach the same clip coefficient unless the two
binary64 sums of squares (different summation orders) straddle a binary32
rounding boundary of clip/norm, so the arrays are in fact compared bit for
bit whenever the clip coefficients agree.
"""
import math

import numpy as np
import torch

import oracle
import workloads as W
from loss_scaled_fp32_b200 import (MPT, MPT_FLAG_GRAD_STATS, MPT_SCALER_DIRECT,
                                   MPT_SCALER_DYNAMIC, Config)


def ulp_diff_f32(a, b):
    """|a - b| in binary32 ulps (ordered-integer distance); NaN == NaN."""
    ia = a.view(np.int32).astype(np.int64)
    ib = b.view(np.int32).astype(np.int64)
    ia = np.where(ia < 0, -(ia & 0x7FFFFFFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFFFFFF), ib)
    d = np.abs(ia - ib)
    both_nan = np.isnan(a) & np.isnan(b)
    return np.where(both_nan, 0, d)


def ulp_diff_f16(a, b):
    ia = a.astype(np.int64)
    ib = b.astype(np.int64)
    ia = np.where(ia & 0x8000, -(ia & 0x7FFF), ia)
    ib = np.where(ib & 0x8000, -(ib & 0x7FFF), ib)
    d = np.abs(ia - ib)
    nan = lambda x: ((x & 0x7C00) == 0x7C00) & ((x & 0x3FF) != 0)
    return np.where(nan(a) & nan(b), 0, d)


class Pair:
    """GPU optimizer + oracle state over the same workload."""

    def __init__(self, cfg, shifted=(), flags=0, chunk=0, master=None, direct_margin=None,
                 optimizer="momentum", eps=1e-10):
        self.cfg = cfg
        self.layout = W.GradLayout(cfg.sizes, shifted=shifted)
        self.direct = direct_margin is not None
        self.hist = bool(flags & MPT_FLAG_GRAD_STATS)
        self.stats = self.hist or self.direct
        mc = Config(backoff=cfg.backoff, growth=cfg.growth, growth_interval=cfg.growth_interval,
                    flags=flags, check_chunk_elems=chunk, update_chunk_elems=chunk,
                    scaler_mode=MPT_SCALER_DIRECT if self.direct else MPT_SCALER_DYNAMIC,
                    direct_margin=direct_margin if self.direct else 2.0,
                    optimizer={"momentum": 0, "nesterov": 1, "adagrad": 2}[optimizer], eps=eps)
        self.oflags = {"momentum": 0, "nesterov": oracle.NESTEROV, "adagrad": oracle.ADAGRAD}[optimizer]
        self.eps = eps
        self.opt = MPT(cfg.sizes, mc)
        # inputs are drawn on the GPU (same integer recipe as on the CPU) and
        # copied to the host, so both sides see identical bits
        master = master if master is not None else [m.cpu() for m in W.make_master(cfg, "cuda")]
        for i, m in enumerate(master):
            self.opt.master(i).copy_(m)
        self.opt.refresh_half()
        self.opt.set_scaler_state(cfg.scale0, 0)
        self.state = oracle.State.from_master([m.numpy() for m in master])
        self.ocfg = oracle.scaler_cfg(backoff=cfg.backoff, growth=cfg.growth,
                                      growth_interval=cfg.growth_interval,
                                      mode=oracle.SCALER_DIRECT if self.direct else oracle.SCALER_DYNAMIC,
                                      direct_margin=direct_margin if self.direct else 2.0)
        self.scale = cfg.scale0
        self.flat = torch.zeros(self.layout.total, dtype=torch.int16, device="cuda")
        self.gviews = self.layout.views(self.flat)
        self.step_no = 0
        self.bitexact_steps = 0
        torch.cuda.synchronize()
        self.compare_state("after refresh")

    def grads(self, step, scale):
        return W.make_grads(self.cfg, step, scale, self.layout, "cuda").cpu()

    def step(self, clip=None, host=None, gpu_grads=None):
        """One step on both sides.  ``host``: flat int16 gradient bits in this
        pair's layout (default: the workload's next step); ``gpu_grads``:
        device tensors already holding the same gradients (default: copy)."""
        self.step_no += 1
        cfg = self.cfg
        clip = cfg.clip if clip is None else clip
        if host is None:
            host = self.grads(self.step_no, self.scale)
        if gpu_grads is None:
            self.flat.copy_(host)
            gpu_grads = self.gviews
        hv = [v.numpy().view(np.uint16) for v in self.layout.views(host)]
        r = self.opt.step(gpu_grads, self.scale, cfg.lr, cfg.momentum, cfg.weight_decay, clip)
        ro = oracle.step(self.state, hv, self.scale, cfg.lr, cfg.momentum, cfg.weight_decay,
                         clip=clip, cfg=self.ocfg, flags=self.oflags, eps=self.eps)
        self.compare_result(r, ro)
        self.compare_state(f"step {self.step_no}", exact=(r["clip_coef"] == ro["clip_coef"]))
        self.scale = r["new_scale"]
        return r, ro

    def compare_result(self, r, ro):
        for k in ("found_inf", "clipped", "n_zero", "n_subnormal", "n_nonfinite"):
            assert r[k] == ro[k], (self.step_no, k, r[k], ro[k])
        assert r["new_scale"] == ro["new_scale"], (self.step_no, r["new_scale"], ro["new_scale"])
        if self.stats:
            assert r["max_abs_grad"] == ro["max_abs"], (self.step_no, r["max_abs_grad"], ro["max_abs"])
            hist = self.opt.grad_histogram()
            if self.hist:
                assert hist == ro["exp_hist"], self.step_no
            else:
                assert hist == [0] * 32
        else:
            assert r["max_abs_grad"] == 0.0
        assert r["clean_run"] == ro["new_clean_run"]
        if ro["found_inf"]:
            assert math.isinf(r["grad_norm"]) and r["clip_coef"] == 1.0
        else:
            assert abs(r["grad_norm"] - ro["norm"]) <= 1e-5 * ro["norm"] + 1e-300, \
                (r["grad_norm"], ro["norm"])
            # coefficient: equal, or one binary32 ulp apart at a rounding boundary
            assert abs(np.float32(r["clip_coef"]) - np.float32(ro["clip_coef"])) <= \
                np.spacing(np.float32(ro["clip_coef"]))

    def gpu_state(self):
        m = [self.opt.master(i).cpu().numpy() for i in range(len(self.cfg.sizes))]
        v = [self.opt.momentum(i).cpu().numpy() for i in range(len(self.cfg.sizes))]
        h = [self.opt.w16(i).cpu().numpy().view(np.uint16) for i in range(len(self.cfg.sizes))]
        return m, v, h

    def compare_state(self, where, exact=True):
        m, v, h = self.gpu_state()
        gm, gv, gh = np.concatenate(m), np.concatenate(v), np.concatenate(h)
        om, ov, oh = (np.concatenate(self.state.master), np.concatenate(self.state.momentum),
                      np.concatenate(self.state.w16))
        if exact:
            same = (gm.tobytes() == om.tobytes() and gv.tobytes() == ov.tobytes()
                    and gh.tobytes() == oh.tobytes())
            if not same:
                bad = np.flatnonzero(gm.view(np.uint32) != om.view(np.uint32))
                raise AssertionError(f"{where}: state not bit-exact; master differs at "
                                     f"{bad[:8].tolist()} ({len(bad)} elements)")
            self.bitexact_steps += 1
        else:
            assert ulp_diff_f32(gm, om).max(initial=0) <= 1, where
            assert ulp_diff_f32(gv, ov).max(initial=0) <= 1, where
            assert ulp_diff_f16(gh, oh).max(initial=0) <= 1, where
