"""Pins of the CPU oracle to facts fixed outside it.

Each test checks the oracle against something it cannot have produced itself:
numbers the pages state (``tests/golden/pages_fp16_facts.json``), exact
rational arithmetic, closed forms, hand-written scaler tables, IEEE-754
identities and a brute-force restatement that computes every binary32
operation as a correctly rounded binary64 operation (Python/numpy).

Only numpy and the oracle are imported so that the mutation test can rerun
this file quickly against deliberately broken builds of the oracle.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_fp16_facts.json")
INF16, NINF16, NAN16 = 0x7C00, 0xFC00, 0x7E00


def facts():
    with open(GOLDEN) as f:
        return {x["id"]: x for x in json.load(f)["facts"]}


def hx(s):
    return float.fromhex(s)


def f32(x):
    return np.float32(x)


def rne16_scalar(x):
    return int(oracle.rne16(np.array([x], np.float32))[0])


def widen_scalar(h):
    return float(oracle.widen16(np.array([h], np.uint16))[0])


def one_tensor_state(w0):
    return oracle.State.from_master([np.array(w0, np.float32)])


# ---------------------------------------------------------------------------
# Golden facts the pages state (codec and loss-scaling arithmetic)
# ---------------------------------------------------------------------------

def test_golden_fp16_range_limits():
    F = facts()
    for key in ("fp16_max", "fp16_min_normal", "fp16_min_subnormal"):
        v, bits = hx(F[key]["value"]), int(F[key]["f16_bits"], 16)
        assert rne16_scalar(v) == bits, key
        assert widen_scalar(bits) == v, key
    # overflow just beyond the largest finite value (round to nearest even:
    # 65520 is the midpoint to 2^16 and rounds away to infinity)
    assert rne16_scalar(65520.0) == INF16
    assert rne16_scalar(-65520.0) == NINF16
    assert rne16_scalar(float(np.nextafter(f32(65520.0), f32(0)))) == 0x7BFF
    for big in (65536.0, 1.0e6, 3.0e38):
        assert rne16_scalar(big) == INF16 and rne16_scalar(-big) == NINF16


def test_golden_flush_to_zero_below_min_subnormal():
    F = facts()["flush_below_min_subnormal"]
    for s in F["zero_inputs"]:
        assert rne16_scalar(hx(s)) == 0, s
        assert rne16_scalar(-hx(s)) == 0x8000, s
    for s in F["nonzero_inputs"]:
        assert rne16_scalar(hx(s)) == 0x0001, s


def test_golden_loss_scale_8_moves_range_into_fp16():
    F = facts()["loss_scale_8_shift"]
    lo, hi, S = hx(F["range_lo"]), hx(F["range_hi"]), F["scale"]
    rng = np.random.default_rng(1)
    g = (lo * np.exp2(rng.uniform(0, math.log2(hi / lo), 4096))).astype(np.float32)
    g = g[(g >= lo) & (g < hi)]
    unscaled = oracle.rne16(g)
    scaled = oracle.rne16(g * f32(S))
    assert np.all(scaled != 0)                 # every value survives under S = 8
    # ... and lands within half a unit of 2^-24 of its scaled value
    err = np.abs(oracle.widen16(scaled).astype(np.float64) - g.astype(np.float64) * S)
    assert np.all(err <= 2.0 ** -25)
    # without scaling the values at or below 2^-25 (the lower half of the
    # range in log scale) are lost
    assert np.all(unscaled[g <= 2.0 ** -25] == 0)
    assert np.mean(unscaled == 0) > 0.5
    # the step's underflow count sees the same thing
    r1 = oracle.check([unscaled], 1.0)
    r8 = oracle.check([scaled], S)
    assert r1.n_zero == int(np.sum(unscaled == 0)) and r8.n_zero == 0


def test_golden_swamping_fp16_vs_fp32():
    F = facts()
    w = hx(F["fp16_swamping_ratio"]["weight"])
    for u in F["fp16_swamping_ratio"]["lost_updates"]:
        assert rne16_scalar(float(f32(w) + f32(hx(u)))) == rne16_scalar(w), u
    for u in F["fp16_swamping_ratio"]["kept_updates"]:
        assert rne16_scalar(float(f32(w) + f32(hx(u)))) != rne16_scalar(w), u
    for u in F["fp32_swamping_ratio"]["lost_updates"]:
        assert f32(w) + f32(hx(u)) == f32(w), u
    for u in F["fp32_swamping_ratio"]["kept_updates"]:
        assert f32(w) + f32(hx(u)) != f32(w), u
    # the 2^13 precision ratio between the two accumulators
    ulp16 = widen_scalar(0x3C01) - 1.0
    ulp32 = float(np.spacing(f32(1.0)))
    assert ulp16 / ulp32 == 2.0 ** F["fp32_vs_fp16_precision"]["ratio_log2"]


def test_golden_fp32_master_keeps_update_at_ratio_below_2_24():
    # update u = 2^-23 via eta = 1, g = -u (exact FP16 subnormal at S = 1):
    # kept by the master; u = 2^-24 sits exactly at the 2^24 ratio (a tie,
    # to even) and is lost even in binary32.
    for u, expect in ((2.0 ** -23, 1.0 + 2.0 ** -23), (2.0 ** -24, 1.0)):
        st = one_tensor_state([1.0])
        g16 = oracle.rne16(np.array([-u], np.float32))
        assert widen_scalar(int(g16[0])) == -u
        oracle.step(st, [g16], 1.0, 1.0, 0.0, 0.0)
        assert float(st.master[0][0]) == expect


# ---------------------------------------------------------------------------
# P1 -- FP16 flush versus survive under S
# ---------------------------------------------------------------------------

def test_p1_flush_vs_survive():
    g_true = np.array([2.0 ** -26, 2.0 ** -25, 1.5 * 2.0 ** -25, 2.0 ** -20], np.float32)
    at1 = oracle.rne16(g_true)
    assert at1.tolist() == [0x0000, 0x0000, 0x0001, 0x0010]
    at1024 = oracle.rne16(g_true * f32(1024))
    assert at1024.tolist() == [0x0100, 0x0200, 0x0300, 0x1400]
    # at S = 2^10 every value is exact after unscaling
    assert np.array_equal(oracle.widen16(at1024) * f32(2.0 ** -10), g_true)
    r = oracle.check([at1], 1.0)
    assert (r.n_zero, r.n_subnormal, r.n_nonfinite, r.found_inf) == (2, 2, 0, 0)
    r = oracle.check([at1024], 1024.0)
    assert (r.n_zero, r.n_subnormal, r.n_nonfinite, r.found_inf) == (0, 3, 0, 0)


def test_counts_over_every_class():
    g = np.array([0x0000, 0x8000, 0x0001, 0x83FF, 0x03FF, 0x0400, 0x8400, 0x3C00,
                  0x7BFF, 0x7C00, 0xFC00, 0x7E00, 0x7C01, 0xFFFF, 0x0200], np.uint16)
    r = oracle.check([g[:7], g[7:]], 1.0)
    assert r.n_zero == 2
    assert r.n_subnormal == 4          # 0x0001 0x83FF 0x03FF 0x0200
    assert r.n_nonfinite == 5          # +inf -inf and three NaN patterns
    assert r.found_inf == 1


# ---------------------------------------------------------------------------
# P2 -- the master copy keeps what the FP16 weight loses
# ---------------------------------------------------------------------------

def test_p2_master_retains_small_update():
    g16 = oracle.rne16(np.array([-(2.0 ** -12)], np.float32))   # 0x8C00
    assert g16.tolist() == [0x8C00]
    st = one_tensor_state([1.0])
    ablation = one_tensor_state([1.0])
    masters, halves, stale = [], [], []
    for _ in range(4):
        r = oracle.step(st, [g16], 1.0, 1.0, 0.0, 0.0)
        oracle.step(ablation, [g16], 1.0, 1.0, 0.0, 0.0, flags=oracle.NO_MASTER)
        masters.append(float(st.master[0][0]))
        halves.append(int(st.w16[0][0]))
        stale.append(r["n_stale"])
        assert int(ablation.w16[0][0]) == 0x3C00      # FP16-only weight never moves
    assert masters == [1 + 2.0 ** -12, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -12, 1 + 2.0 ** -10]
    assert halves == [0x3C00, 0x3C00, 0x3C01, 0x3C01]   # step 2 is a tie -> even
    assert stale == [1, 1, 0, 1]


# ---------------------------------------------------------------------------
# P3 -- an overflowing step changes nothing and backs S off
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bad", [INF16, NINF16, NAN16, 0x7C01, 0xFE00])
def test_p3_overflow_skips_and_backs_off(bad):
    rng = np.random.default_rng(bad)
    sizes = [5, 33, 1, 17]
    st = oracle.State.from_master([rng.normal(0, 0.05, n).astype(np.float32) for n in sizes])
    st.momentum = [rng.normal(0, 1e-3, n).astype(np.float32) for n in sizes]
    st.clean_run = 3
    grads = [rng.integers(0, 0x7800, n).astype(np.uint16) for n in sizes]
    grads[2][0] = bad
    before = st.copy()
    cfg = oracle.scaler_cfg(growth_interval=4)
    r = oracle.step(st, grads, 2.0 ** 12, 0.01, 0.9, 1e-4, clip=1.0, cfg=cfg)
    assert r["found_inf"] == 1 and r["n_nonfinite"] == 1
    assert r["norm"] == math.inf and r["clip_coef"] == 1.0
    assert r["new_scale"] == 2.0 ** 11 and r["new_clean_run"] == 0
    for a, b in zip(st.master + st.momentum + st.w16, before.master + before.momentum + before.w16):
        assert a.tobytes() == b.tobytes()


# ---------------------------------------------------------------------------
# P4 -- the update is invariant to S when nothing overflows or underflows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("k", [1, 4, 9])
@pytest.mark.parametrize("clip_frac", [0.0, 0.5])
def test_p4_scale_invariance(k, clip_frac):
    rng = np.random.default_rng(100 + k)
    sizes = [64, 7, 300]
    exp_field = lambda n: rng.integers(1, 31 - k, n).astype(np.uint16)   # normal, room for k
    grads = [((rng.integers(0, 2, n) << 15) | (exp_field(n) << 10) | rng.integers(0, 1024, n))
             .astype(np.uint16) for n in sizes]
    scaled = [(g + np.uint16(k << 10)).astype(np.uint16) for g in grads]   # exactly g * 2^k
    assert np.array_equal(oracle.widen16(np.concatenate(scaled)),
                          oracle.widen16(np.concatenate(grads)) * f32(2.0 ** k))
    master = [rng.normal(0, 0.05, n).astype(np.float32) for n in sizes]
    a, b = oracle.State.from_master(master), oracle.State.from_master(master)
    S = 2.0 ** -6   # grads below 2^16 are unscaled to below 2^22
    clip = clip_frac * oracle.clip_coef(oracle.check(grads, S), 0.0).norm
    for _ in range(3):
        ra = oracle.step(a, grads, S, 0.01, 0.9, 1e-4, clip=clip)
        rb = oracle.step(b, scaled, S * 2.0 ** k, 0.01, 0.9, 1e-4, clip=clip)
        for key in ("found_inf", "clipped", "sumsq", "norm", "clip_coef", "n_zero",
                    "n_subnormal", "n_nonfinite", "n_stale"):
            assert ra[key] == rb[key], key
    if clip_frac:
        assert ra["clipped"] == 1
    for x, y in zip(a.master + a.momentum + a.w16, b.master + b.momentum + b.w16):
        assert x.tobytes() == y.tobytes()


# ---------------------------------------------------------------------------
# P5 -- brute force: every binary32 op as a correctly rounded binary64 op
# ---------------------------------------------------------------------------

def _bf_widen(h):
    return float(np.array([h], np.uint16).view(np.float16).astype(np.float64)[0])


def _bf_rne16(x):
    return int(np.array([x], np.float32).astype(np.float16).view(np.uint16)[0])


def brute_force_step(master, momentum, grads, S, lr, mom, wd, clip):
    """Plain Python restatement; binary64 has > 2*24+2 bits, so rounding the
    exact-enough binary64 result of +, *, / once to binary32 gives the
    correctly rounded binary32 result."""
    S, lr, mom, wd, clip = (float(f32(x)) for x in (S, lr, mom, wd, clip))
    inv = float(f32(1.0 / S))
    found, sumsq = False, 0.0
    for g in grads:
        for h in g:
            if (int(h) & 0x7FFF) >= 0x7C00:
                found = True
                continue
            x = float(f32(_bf_widen(h) * inv))
            sumsq += x * x
    if found:
        return None
    norm = math.sqrt(sumsq)
    clipped = clip > 0 and norm > clip
    coef = float(f32(clip / norm)) if clipped else 1.0
    new_w, new_v, new_h = [], [], []
    for g, w, v in zip(grads, master, momentum):
        W, V, H = [], [], []
        for h, wi, vi in zip(g, w.tolist(), v.tolist()):
            gi = float(f32(_bf_widen(h) * inv))
            if clipped:
                gi = float(f32(gi * coef))
            t = float(f32(wd * wi))
            d = float(f32(gi + t))
            u = float(f32(mom * vi))
            vn = float(f32(u + d))
            s = float(f32(lr * vn))
            wn = float(f32(wi - s))
            W.append(wn), V.append(vn), H.append(_bf_rne16(wn))
        new_w.append(np.array(W, np.float32))
        new_v.append(np.array(V, np.float32))
        new_h.append(np.array(H, np.uint16))
    return new_w, new_v, new_h, norm, coef


@pytest.mark.parametrize("seed", range(8))
def test_p5_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    sizes = list(rng.integers(1, 9, rng.integers(1, 4)))
    S = float(2.0 ** rng.integers(-3, 12)) if seed % 2 == 0 else float(rng.uniform(0.7, 3000))
    clip = [0.0, 1e-3, 10.0][seed % 3]
    master = [rng.normal(0, 0.05, n).astype(np.float32) for n in sizes]
    st = oracle.State.from_master(master)
    w, v = [m.copy() for m in master], [np.zeros(n, np.float32) for n in sizes]
    for step in range(4):
        grads = []
        for n in sizes:
            e = rng.integers(0, 30, n)
            g = (rng.integers(0, 2, n) << 15) | (e << 10) | rng.integers(0, 1024, n)
            g[rng.random(n) < 0.15] = 0
            grads.append(g.astype(np.uint16))
        r = oracle.step(st, grads, S, 0.01, 0.9, 1e-4, clip=clip)
        bf = brute_force_step(w, v, grads, S, 0.01, 0.9, 1e-4, clip)
        assert r["found_inf"] == 0 and bf is not None
        w, v, h, norm, coef = bf
        assert r["norm"] == norm and r["clip_coef"] == coef
        for a, b in zip(st.master + st.momentum + st.w16, w + v + h):
            assert a.tobytes() == b.tobytes()


# ---------------------------------------------------------------------------
# P7 -- exact recurrences (rational arithmetic) and closed forms
# ---------------------------------------------------------------------------

def _exact_f32(fr):
    x = f32(float(fr))
    return Fraction(float(x)) == fr


@pytest.mark.parametrize("mom,wd", [(Fraction(1, 2), Fraction(0)), (Fraction(1, 2), Fraction(1, 8)),
                                    (Fraction(0), Fraction(1, 2)), (Fraction(3, 4), Fraction(1, 16))])
def test_p7_exact_recurrence(mom, wd):
    """v_t = mu v_{t-1} + g + lambda w_{t-1};  w_t = w_{t-1} - eta v_t, in
    exact rationals; while every intermediate is a binary32 number the
    oracle must reproduce it bit for bit."""
    S, lr = Fraction(4), Fraction(1, 4)
    g16 = np.array([0x3E00, 0xBA00, 0x0000], np.uint16)          # 1.5, -0.75, 0
    g = [Fraction(_bf_widen(h)) / S for h in g16]
    w0 = [Fraction(1), Fraction(-2), Fraction(1, 2)]
    st = oracle.State.from_master([np.array([float(x) for x in w0], np.float32)])
    w, v = list(w0), [Fraction(0)] * 3
    exact_steps = 0
    for step in range(12):
        nv = [mom * v[i] + g[i] + wd * w[i] for i in range(3)]
        nw = [w[i] - lr * nv[i] for i in range(3)]
        inter = [wd * w[i] for i in range(3)] + [mom * v[i] for i in range(3)] + \
                [lr * nv[i] for i in range(3)] + [g[i] + wd * w[i] for i in range(3)] + nv + nw
        if not all(_exact_f32(x) for x in inter):
            break
        oracle.step(st, [g16], float(S), float(lr), float(mom), float(wd))
        w, v = nw, nv
        assert [Fraction(float(x)) for x in st.master[0]] == w
        assert [Fraction(float(x)) for x in st.momentum[0]] == v
        exact_steps += 1
    assert exact_steps >= 3


def test_p7_momentum_closed_form():
    """Constant gradient, lambda = 0: v_t = g (1 - mu^t) / (1 - mu) and
    w_t = w_0 - eta sum v_k; binary32 rounding keeps each within the bound
    t * 2 ulp."""
    mu, eta, g_true = 0.9, 0.01, 2.0 ** -8
    g16 = oracle.rne16(np.array([g_true * 128], np.float32))
    st = one_tensor_state([0.25])
    vsum = 0.0
    for t in range(1, 11):
        oracle.step(st, [g16], 128.0, eta, mu, 0.0)
        v_exact = g_true * (1 - float(f32(mu)) ** t) / (1 - float(f32(mu)))
        vsum += v_exact
        v = float(st.momentum[0][0])
        w = float(st.master[0][0])
        assert abs(v - v_exact) <= 2 * t * float(np.spacing(f32(v_exact)))
        assert abs(w - (0.25 - float(f32(eta)) * vsum)) <= 2 * t * float(np.spacing(f32(w)))


def test_p7_norm_closed_form():
    # n equal gradients c: norm = |c| sqrt(n); with c = 2^-3 and n = 4^5 it is 4
    g16 = oracle.rne16(np.full(1024, -(2.0 ** -3) * 64, np.float32))
    r = oracle.clip_coef(oracle.check([g16[:1000], g16[1000:]], 64.0), 0.0)
    assert r.norm == 4.0 and r.sumsq == 16.0 and r.clip_coef == 1.0


# ---------------------------------------------------------------------------
# P8 -- loss-scale state machine against hand tables
# ---------------------------------------------------------------------------

def test_p8_scaler_constant_scale_backs_off_only():
    cfg = oracle.scaler_cfg(growth_interval=0)
    overflow = [0, 0, 0, 0, 1, 0, 0, 0, 0, 0]
    expect_S = [1024, 1024, 1024, 1024, 512, 512, 512, 512, 512, 512]
    expect_c = [1, 2, 3, 4, 0, 1, 2, 3, 4, 5]
    S, c = 1024.0, 0
    for ov, es, ec in zip(overflow, expect_S, expect_c):
        S, c = oracle.scaler_next(cfg, ov, S, c)
        assert (S, c) == (es, ec)


def test_p8_scaler_dynamic_table():
    cfg = oracle.scaler_cfg(growth_interval=4)
    overflow = [0, 0, 0, 0, 0, 0, 1, 0, 0, 0, 0, 1, 1, 0]
    expect_S = [2 ** 16] * 3 + [2 ** 17] * 3 + [2 ** 16] * 4 + [2 ** 17, 2 ** 16, 2 ** 15, 2 ** 15]
    expect_c = [1, 2, 3, 0, 1, 2, 0, 1, 2, 3, 0, 0, 0, 1]
    S, c = float(2 ** 16), 0
    for ov, es, ec in zip(overflow, expect_S, expect_c):
        S, c = oracle.scaler_next(cfg, ov, S, c)
        assert (S, c) == (es, ec)


def test_p8_scaler_bounds():
    cfg = oracle.scaler_cfg(growth_interval=1, min_scale=2.0 ** -24, max_scale=2.0 ** 24)
    assert oracle.scaler_next(cfg, 1, 2.0 ** -24, 5) == (2.0 ** -24, 0)
    assert oracle.scaler_next(cfg, 0, 2.0 ** 24, 0) == (2.0 ** 24, 0)
    assert oracle.scaler_next(cfg, 0, 2.0 ** 23, 0) == (2.0 ** 24, 0)


def test_p8_skipped_step_through_the_step():
    cfg = oracle.scaler_cfg(growth_interval=0)
    st = one_tensor_state([0.5, 0.25])
    ok = np.array([0x3C00, 0x3C00], np.uint16)
    bad = np.array([0x3C00, INF16], np.uint16)
    S = 1024.0
    seen = []
    for t in range(1, 11):
        r = oracle.step(st, [bad if t == 5 else ok], S, 0.01, 0.9, 1e-4, cfg=cfg)
        S = r["new_scale"]
        seen.append(S)
    assert seen == [1024.0] * 4 + [512.0] * 6


# ---------------------------------------------------------------------------
# P9 -- global L2 clipping
# ---------------------------------------------------------------------------

def test_p9_clip():
    rng = np.random.default_rng(9)
    sizes = [100, 37]
    grads = [oracle.rne16(rng.normal(0, 0.1, n).astype(np.float32) * f32(256)) for n in sizes]
    norm = oracle.clip_coef(oracle.check(grads, 256.0), 0.0).norm
    master = [rng.normal(0, 0.05, n).astype(np.float32) for n in sizes]

    # norm <= clip: bitwise identical to no clipping
    a, b = oracle.State.from_master(master), oracle.State.from_master(master)
    oracle.step(a, grads, 256.0, 0.01, 0.9, 1e-4, clip=0.0)
    rb = oracle.step(b, grads, 256.0, 0.01, 0.9, 1e-4, clip=float(norm) * 1.01)
    assert rb["clipped"] == 0
    for x, y in zip(a.master + a.momentum + a.w16, b.master + b.momentum + b.w16):
        assert x.tobytes() == y.tobytes()

    # norm > clip: eta = 1, mu = 0, lambda = 0, w0 = 0 makes w1 = -clipped grad;
    # its L2 norm is the threshold
    clip = float(norm) / 3
    c = oracle.State.from_master([np.zeros(n, np.float32) for n in sizes])
    rc = oracle.step(c, grads, 256.0, 1.0, 0.0, 0.0, clip=clip)
    assert rc["clipped"] == 1 and rc["norm"] == norm
    gc = -np.concatenate(c.master).astype(np.float64)
    assert abs(math.sqrt(np.sum(gc * gc)) / f32(clip) - 1) < 1e-6
    # the clip multiplies the unscaled gradient, not the weight-decay term
    d = oracle.State.from_master([np.full(n, 0.5, np.float32) for n in sizes])
    oracle.step(d, grads, 256.0, 1.0, 0.0, 0.5, clip=clip)
    expect = [f32(0.5) - (f32(-x) + f32(0.25)) for x in c.master]
    for x, y in zip(d.master, expect):
        assert np.array_equal(x, np.asarray(y, np.float32))


# ---------------------------------------------------------------------------
# Gradient statistics of pass 1 and the direct choice of S
# ---------------------------------------------------------------------------

def test_stats_histogram_and_max_against_numpy():
    rng = np.random.default_rng(21)
    g = rng.integers(0, 1 << 16, 50_000).astype(np.uint16)
    g[:40] = [0, 0x8000, 0x0001, 0x7C00, 0xFC00, 0x7E00, 0x7BFF, 0xFBFF] * 5
    parts = [g[:7], g[7:30_000], g[30_000:]]
    r = oracle.check(parts, 2.0 ** 7)
    mag = g & 0x7FFF
    assert list(r.exp_hist) == np.bincount(mag >> 10, minlength=32).tolist()
    finite = mag[mag < 0x7C00]
    assert r.max_mag16 == finite.max() == 0x7BFF
    expect = np.float32(np.array([finite.max()], np.uint16).view(np.float16)[0]) * np.float32(2.0 ** -7)
    assert r.max_abs == expect
    # the maximum ignores inf/NaN and is found in any tensor of the list
    r2 = oracle.check([np.array([0x3C00, 0x7C00], np.uint16), np.array([0x4000], np.uint16)], 1.0)
    assert (r2.max_mag16, r2.max_abs) == (0x4000, 2.0)


def test_golden_direct_scale_formula():
    F = facts()["direct_scale_formula"]
    m = hx(F["max_abs_grad"])
    assert oracle.direct_scale(m, margin=1.0) == hx(F["scale"])
    assert oracle.direct_scale(m, margin=2.0) == hx(F["scale_with_margin"])
    assert oracle.direct_scale(0.0) == 0.0                      # no information
    assert oracle.direct_scale(2.0 ** -40, max_scale=2.0 ** 24) == 2.0 ** 24   # clamped
    assert oracle.direct_scale(2.0 ** 40, min_scale=2.0 ** -24) == 2.0 ** -24


@pytest.mark.parametrize("margin", [1.0, 2.0, 4.0])
def test_direct_scale_puts_the_largest_gradient_at_65504_over_margin(margin):
    rng = np.random.default_rng(int(margin))
    g_true = (rng.standard_normal(4096) * 1e-2).astype(np.float32)
    S = oracle.direct_scale(float(np.abs(g_true).max()), margin=margin)
    scaled = oracle.rne16(g_true * np.float32(S))
    assert np.all((scaled & 0x7FFF) < 0x7C00)                   # nothing overflows
    top = float(oracle.widen16(scaled[np.argmax(np.abs(g_true))])[0])
    assert abs(abs(top) - 65504.0 / margin) <= 32.0             # within half an ulp at 2^15


def test_direct_scaler_mode_through_the_step():
    """Direct mode: after a clean step S = 65504 / (margin * max|g_true|) of
    that step; an overflow backs off; all-zero gradients keep S."""
    cfg = oracle.scaler_cfg(mode=oracle.SCALER_DIRECT, direct_margin=2.0)
    st = one_tensor_state([0.5, -0.25, 1.0])
    S = 2.0 ** 10
    g_true = np.array([2.0 ** -9, -(2.0 ** -6), 3 * 2.0 ** -12], np.float32)
    r = oracle.step(st, [oracle.rne16(g_true * np.float32(S))], S, 0.01, 0.9, 0.0, cfg=cfg)
    assert r["max_abs"] == 2.0 ** -6
    assert r["new_scale"] == np.float32(65504.0 / (2.0 * 2.0 ** -6))
    S2 = r["new_scale"]
    bad = np.array([0x7C00, 0, 0], np.uint16)
    r = oracle.step(st, [bad], S2, 0.01, 0.9, 0.0, cfg=cfg)
    assert r["found_inf"] == 1 and r["new_scale"] == S2 * 0.5
    r = oracle.step(st, [np.zeros(3, np.uint16)], 64.0, 0.01, 0.9, 0.0, cfg=cfg)
    assert r["max_abs"] == 0.0 and r["new_scale"] == 64.0


# ---------------------------------------------------------------------------
# Nesterov momentum and Adagrad (the pages' speech models and bigLSTM)
# ---------------------------------------------------------------------------

def brute_force_update(w, v, g16, S, lr, mom, wd, opt, eps=1e-10):
    """Python restatement of one update, each binary32 op correctly rounded
    via binary64 (sqrt too: binary64 has more than 2*24+2 bits)."""
    S, lr, mom, wd, eps = (float(f32(x)) for x in (S, lr, mom, wd, eps))
    inv = float(f32(1.0 / S))
    W, V = [], []
    for h, wi, vi in zip(g16, w.tolist(), v.tolist()):
        g = float(f32(_bf_widen(h) * inv))
        d = float(f32(g + float(f32(wd * wi))))
        if opt == "adagrad":
            vn = float(f32(vi + float(f32(d * d))))
            den = float(f32(float(f32(math.sqrt(vn))) + eps))
            step = float(f32(d / den))
        else:
            vn = float(f32(float(f32(mom * vi)) + d))
            step = vn if opt == "momentum" else float(f32(d + float(f32(mom * vn))))
        W.append(float(f32(wi - float(f32(lr * step)))))
        V.append(vn)
    return np.array(W, np.float32), np.array(V, np.float32)


@pytest.mark.parametrize("opt,flag", [("nesterov", oracle.NESTEROV), ("adagrad", oracle.ADAGRAD),
                                      ("momentum", 0)])
def test_optimizers_brute_force(opt, flag):
    rng = np.random.default_rng(77)
    n = 64
    w = rng.normal(0, 0.05, n).astype(np.float32)
    st = oracle.State.from_master([w])
    bw, bv = w.copy(), np.zeros(n, np.float32)
    for step in range(5):
        g16 = ((rng.integers(0, 2, n) << 15) | (rng.integers(1, 29, n) << 10) |
               rng.integers(0, 1024, n)).astype(np.uint16)
        r = oracle.step(st, [g16], 2.0 ** 6, 0.01, 0.9, 1e-4, flags=flag)
        assert r["found_inf"] == 0
        bw, bv = brute_force_update(bw, bv, g16, 2.0 ** 6, 0.01, 0.9, 1e-4, opt)
        assert st.master[0].tobytes() == bw.tobytes(), (opt, step)
        assert st.momentum[0].tobytes() == bv.tobytes(), (opt, step)
        assert st.w16[0].tobytes() == oracle.rne16(bw).tobytes()


def test_nesterov_exact_recurrence():
    """v_t = mu v + d;  w_t = w - eta (d + mu v_t) in exact rationals while
    every intermediate is a binary32 number."""
    mu, lr, S = Fraction(1, 2), Fraction(1, 4), Fraction(2)
    g16 = np.array([0x3E00, 0xB800], np.uint16)                 # 1.5, -0.5
    g = [Fraction(_bf_widen(h)) / S for h in g16]
    w, v = [Fraction(1), Fraction(-3, 4)], [Fraction(0)] * 2
    st = oracle.State.from_master([np.array([float(x) for x in w], np.float32)])
    exact = 0
    for _ in range(10):
        nv = [mu * v[i] + g[i] for i in range(2)]
        stepv = [g[i] + mu * nv[i] for i in range(2)]
        nw = [w[i] - lr * stepv[i] for i in range(2)]
        if not all(_exact_f32(x) for x in nv + stepv + nw + [lr * s for s in stepv]):
            break
        oracle.step(st, [g16], float(S), float(lr), float(mu), 0.0, flags=oracle.NESTEROV)
        w, v = nw, nv
        assert [Fraction(float(x)) for x in st.master[0]] == w
        exact += 1
    assert exact >= 4


def test_adagrad_first_step_is_lr_times_sign():
    """With h0 = 0 and eps = 0 the first Adagrad step is exactly eta * sign(d)
    whatever the gradient's size; afterwards h holds the sum of squares."""
    g_true = np.array([3e-5, -7.0, 2.0 ** -20, -0.25], np.float32)
    g16 = oracle.rne16(g_true * f32(1024))
    st = oracle.State.from_master([np.full(4, 0.5, np.float32)])
    oracle.step(st, [g16], 1024.0, 0.125, 0.0, 0.0, flags=oracle.ADAGRAD, eps=0.0)
    assert st.master[0].tolist() == [0.5 - 0.125, 0.5 + 0.125, 0.5 - 0.125, 0.5 + 0.125]
    g = oracle.widen16(g16) * f32(2.0 ** -10)
    assert np.array_equal(st.momentum[0], g * g)
    oracle.step(st, [g16], 1024.0, 0.125, 0.0, 0.0, flags=oracle.ADAGRAD, eps=0.0)
    assert np.array_equal(st.momentum[0], g * g + g * g)


def test_adagrad_closed_form_constant_gradient():
    # constant g: h_t = t g^2, w_t = w0 - eta sum_k g / (sqrt(k) |g| + eps)
    g16 = np.array([0x2C00], np.uint16)                          # 2^-4
    st = oracle.State.from_master([np.array([1.0], np.float32)])
    w, eps, lr = 1.0, float(f32(1e-10)), float(f32(0.01))
    for t in range(1, 21):
        oracle.step(st, [g16], 1.0, 0.01, 0.0, 0.0, flags=oracle.ADAGRAD)
        w -= lr * 2.0 ** -4 / (math.sqrt(t) * 2.0 ** -4 + eps)
        assert abs(float(st.master[0][0]) - w) <= 4 * t * float(np.spacing(f32(w)))
    assert float(st.momentum[0][0]) == 20 * 2.0 ** -8
