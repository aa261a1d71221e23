"""The allocation-free entry point, mpt_check_flat_noalloc.

It exists for callers that cannot allocate device memory (a library living
inside a host program whose memory pool owns the device, or a step loop that
must never enter the CUDA allocator): it computes the overflow check and the
global gradient norm of one contiguous FP16 buffer with its scratch in a
fixed array inside the library.  Here it is called through the C ABI and its
results are compared with those of the existing entry point, mpt_step, on the
same gradients, on consecutive calls (so that what one call leaves in the
shared scratch array cannot leak into the next).

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


@pytest.mark.gpu
def test_noalloc_check_matches_mpt_step_on_consecutive_calls():
    import torch
    import workloads as W
    from workloads.configs import Config, TensorSpec

    n = 3_000_017                              # 92 bins of 32768 and a ragged tail
    cfg = Config(name="flat", tensors=[TensorSpec("g", (n,), ("normal", 0.05))],
                 grad_law=("log2_normal", -14.0, 3.0), scale0=2.0 ** 12, growth_interval=0,
                 lr=0.01, momentum=0.9, weight_decay=1e-4, clip=0.5, steps=3, seed=31)
    layout = W.GradLayout([n])
    opt = lsf.MPT([n], lsf.Config())
    for i, m in enumerate(W.make_master(cfg, "cuda")):
        opt.master(i).copy_(m)
    opt.refresh_half()
    out = torch.zeros(ctypes.sizeof(lsf.CheckResult), dtype=torch.uint8, device="cuda")

    calls = [(2.0 ** 12, 0.5, None),           # power-of-two S, clipping on
             (2.0 ** 12, 0.5, 0x7C00),         # an overflowing buffer
             (3000.0, 0.0, None)]              # other S, no clipping
    for k, (scale, clip, bad) in enumerate(calls, start=1):
        flat = W.make_grads(cfg, k, scale, layout, "cuda")
        if bad is not None:
            flat[n // 2] = bad
        g = layout.views(flat)[0]
        ref = opt.step([g], scale, cfg.lr, cfg.momentum, cfg.weight_decay, clip)
        out.fill_(0xFF)                        # stale bytes must all be overwritten
        lsf.check_flat_noalloc(g, scale, clip, out)
        torch.cuda.synchronize()
        got = lsf.CheckResult.from_buffer_copy(out.cpu().numpy().tobytes()).as_dict()

        assert got["found_inf"] == ref["found_inf"], k
        assert got["n_nonfinite"] == ref["n_nonfinite"], k
        assert got["clipped"] == ref["clipped"], k
        if ref["found_inf"]:
            assert math.isinf(got["grad_norm"]) and got["clip_coef"] == 1.0
        else:
            assert abs(got["grad_norm"] - ref["grad_norm"]) <= 1e-5 * ref["grad_norm"], k
            assert abs(np.float32(got["clip_coef"]) - np.float32(ref["clip_coef"])) <= \
                np.spacing(np.float32(ref["clip_coef"])), k
    opt.close()
