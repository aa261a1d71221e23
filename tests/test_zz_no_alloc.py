"""The allocation-free entry point, mpt_check_flat_noalloc.

It exists for callers that cannot allocate device memory (a library living
inside a host program whose memory pool owns the device, or a step loop that
must never enter the CUDA allocator): it computes the overflow check and the
global gradient norm of one contiguous FP16 buffer with its scratch in a
fixed array inside the library.  Here it is called through the C ABI, and
every call's result is compared with the CPU oracle's check pass on the same
bits (found_inf and the non-finite count exact, the norm within 1e-5
relative, the clip coefficient within one binary32 ulp) and, for the first
calls, with the existing entry point, mpt_step, on the same gradients.  The
calls run back to back on the one shared scratch array, so what one call
leaves there cannot leak into the next unnoticed.

This file is collected last on purpose; it must pass alone in a fresh process
as well as after the other tests.
"""
import ctypes
import math

import numpy as np
import pytest

import loss_scaled_fp32_b200 as lsf


def test_noalloc_rejects_too_large_and_bad_arguments():
    L = lsf.lib()
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: rejected first
    out = ctypes.c_void_p(1 << 21)
    rc = L.mpt_check_flat_noalloc(fake, lsf.MPT_NOALLOC_MAX_ELEMS + 1, 1.0, 0.0, out, None)
    assert rc == lsf.MPT_ERR_TOO_LARGE
    assert b"2^30" in L.mpt_error_string(rc)
    assert L.mpt_check_flat_noalloc(fake, 0, 1.0, 0.0, out, None) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_check_flat_noalloc(None, 10, 1.0, 0.0, out, None) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_check_flat_noalloc(fake, 10, -1.0, 0.0, out, None) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_check_flat_noalloc(ctypes.c_void_p((1 << 20) + 1), 10, 1.0, 0.0, out,
                                    None) == lsf.MPT_ERR_INVALID_ARG


def _noalloc(g, scale, clip, out):
    import torch
    out.fill_(0xFF)                            # stale bytes must all be overwritten
    lsf.check_flat_noalloc(g, scale, clip, out)
    torch.cuda.synchronize()
    return lsf.CheckResult.from_buffer_copy(out.cpu().numpy().tobytes()).as_dict()


def _against_oracle(got, host_bits, scale, clip, what):
    import oracle
    ro = oracle.clip_coef(oracle.check([host_bits], scale), clip)
    assert got["found_inf"] == ro.found_inf, what
    assert got["n_nonfinite"] == ro.n_nonfinite, what
    assert got["clipped"] == ro.clipped, what
    if ro.found_inf:
        assert math.isinf(got["grad_norm"]) and got["clip_coef"] == 1.0, what
    else:
        assert abs(got["grad_norm"] - ro.norm) <= 1e-5 * ro.norm + 1e-300, (what, got, ro.norm)
        assert abs(np.float32(got["clip_coef"]) - np.float32(ro.clip_coef)) <= \
            np.spacing(np.float32(ro.clip_coef)), what
    return ro


def _grads(n, step, scale, law=("log2_normal", -14.0, 3.0)):
    import workloads as W
    from workloads.configs import Config, TensorSpec
    cfg = Config(name="flat", tensors=[TensorSpec("g", (n,), ("normal", 0.05))],
                 grad_law=law, scale0=scale, growth_interval=0, lr=0.01, momentum=0.9,
                 weight_decay=1e-4, clip=0.5, steps=3, seed=31)
    layout = W.GradLayout([n])
    return cfg, layout, W.make_grads(cfg, step, scale, layout, "cuda")


@pytest.mark.gpu
def test_noalloc_check_matches_oracle_and_mpt_step_on_consecutive_calls():
    import torch
    import workloads as W

    n = 3_000_017                              # 92 bins of 32768 and a ragged tail
    cfg, layout, _ = _grads(n, 1, 2.0 ** 12)
    opt = lsf.MPT([n], lsf.Config())
    for i, m in enumerate(W.make_master(cfg, "cuda")):
        opt.master(i).copy_(m)
    opt.refresh_half()
    out = torch.zeros(ctypes.sizeof(lsf.CheckResult), dtype=torch.uint8, device="cuda")

    calls = [(2.0 ** 12, 0.5, None),           # power-of-two S, clipping on
             (2.0 ** 12, 0.5, 0x7C00),         # an overflowing buffer
             (3000.0, 0.0, None),              # other S, no clipping
             (2.0 ** 12, 0.5, 0x7E00)]         # NaN, right after a clean call
    for k, (scale, clip, bad) in enumerate(calls, start=1):
        flat = W.make_grads(cfg, k, scale, layout, "cuda")
        if bad is not None:
            flat[n // 2] = bad
        g = layout.views(flat)[0]
        ref = opt.step([g], scale, cfg.lr, cfg.momentum, cfg.weight_decay, clip)
        got = _noalloc(g, scale, clip, out)
        host = g.cpu().numpy().view(np.uint16)
        _against_oracle(got, host, scale, clip, k)
        # the existing entry point on the same gradients agrees as well
        assert got["found_inf"] == ref["found_inf"] and got["clipped"] == ref["clipped"], k
        assert got["n_nonfinite"] == ref["n_nonfinite"], k
        if not ref["found_inf"]:
            assert abs(got["grad_norm"] - ref["grad_norm"]) <= 1e-5 * ref["grad_norm"], k
    opt.close()


@pytest.mark.gpu
def test_noalloc_check_unaligned_small_and_long_buffers():
    """Views 2 and 8 bytes past an aligned start (the load paths of a range
    that begins between 16-byte boundaries), a one-bin buffer (its only CTA
    is also the last one and writes the result), a single element, and a
    buffer of more than 2^26 elements (over 2048 bins, where the finish adds
    the partials eight loads at a time); each checked against the oracle,
    with and without an overflow, back to back on the shared scratch."""
    import torch

    out = torch.zeros(ctypes.sizeof(lsf.CheckResult), dtype=torch.uint8, device="cuda")
    _, _, flat = _grads(1_000_003, 2, 2.0 ** 10, law=("log2_uniform", -30.0, -4.0))
    cases = []
    for off in (1, 4, 3):
        cases.append(("offset %d" % off, flat[off:], 2.0 ** 10, 0.3))
    cases.append(("one bin", flat[5:1005], 2.0 ** 10, 0.01))
    cases.append(("one element", flat[7:8], 2.0 ** 10, 0.0))
    for what, g, scale, clip in cases:
        for bad in (None, 0x7C00):
            if bad is not None:
                saved = g[g.numel() - 1].item()
                g[g.numel() - 1] = bad
            got = _noalloc(g, scale, clip, out)
            _against_oracle(got, g.cpu().numpy().view(np.uint16), scale, clip, (what, bad))
            if bad is not None:
                assert got["found_inf"] == 1 and got["n_nonfinite"] == 1
                g[g.numel() - 1] = saved
    del flat

    n = 70_000_001                             # 2137 bins of 32768
    _, _, big = _grads(n, 3, 2.0 ** 8, law=("log2_uniform", -30.0, -6.0))
    host = big.cpu().numpy().view(np.uint16)
    for scale, clip in ((2.0 ** 8, 1.0), (1000.0, 0.0)):
        got = _noalloc(big, scale, clip, out)
        _against_oracle(got, host, scale, clip, ("long", scale))
    big[n - 2] = 0xFC00 - 65536             # -inf as int16 bits
    got = _noalloc(big, 2.0 ** 8, 1.0, out)
    assert got["found_inf"] == 1 and got["n_nonfinite"] == 1
