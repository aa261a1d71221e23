"""CPU checks of the seeded workload generators (shared by both sides of the
parity tests, so they hold none of the step's arithmetic)."""
import numpy as np
import pytest
import torch

import workloads as W
from workloads.configs import EXPECTED_PARAMS, EXPECTED_TENSORS, miniature, truncated


@pytest.mark.parametrize("name", list(W.CONFIGS))
def test_workload_shapes(name):
    cfg = W.get(name)
    assert len(cfg.tensors) == EXPECTED_TENSORS[name]
    if name in EXPECTED_PARAMS:
        assert cfg.n_params == EXPECTED_PARAMS[name]
    assert all(s >= 1 for s in cfg.sizes)


def test_ragged_sizes_are_log_uniform():
    sizes = W.configs.ragged_sizes()
    assert sizes.min() >= 1 and sizes.max() < 2 ** 20
    assert abs(np.mean(sizes <= 64) - 0.30) < 0.02          # ln 64 / ln 2^20
    assert abs(np.mean(np.log(sizes)) / np.log(2.0 ** 20) - 0.5) < 0.02


def test_grads_are_deterministic_and_layout_independent():
    cfg = miniature("ragged20k")
    a = W.make_grads(cfg, 4, 2.0 ** 10, W.GradLayout(cfg.sizes), "cpu")
    b = W.make_grads(cfg, 4, 2.0 ** 10, W.GradLayout(cfg.sizes), "cpu")
    assert torch.equal(a, b)
    shifted = W.GradLayout(cfg.sizes, shifted=range(0, len(cfg.sizes), 2))
    c = W.make_grads(cfg, 4, 2.0 ** 10, shifted, "cpu")
    for x, y in zip(W.GradLayout(cfg.sizes).views(a), shifted.views(c)):
        assert torch.equal(x, y)
    other = W.make_grads(cfg, 5, 2.0 ** 10, W.GradLayout(cfg.sizes), "cpu")
    assert not torch.equal(a, other)


def test_layout_alignment():
    L = W.GradLayout([3, 17, 1, 40], shifted={2})
    assert [o % 16 for o in L.offsets] == [0, 0, 1, 0]
    assert L.total % 16 == 0 and L.total >= L.offsets[-1] + 40


def test_flat1m_law_and_injection():
    cfg = W.get("flat1m")
    L = W.GradLayout(cfg.sizes)
    h = W.make_grads(cfg, 1, cfg.scale0, L, "cpu").numpy().view(np.uint16)
    mag = h & 0x7FFF
    # |g_true| = 2^U, U in [-30, -6), times S = 2^10: exponents -20..3, so
    # about a quarter (-20..-15) are binary16 subnormals, none zero or inf
    assert abs(np.mean((mag > 0) & (mag < 0x400)) - 0.25) < 0.01
    assert np.all(mag > 0) and np.all(mag < 0x7C00)
    assert abs(np.mean(h >> 15) - 0.5) < 0.01
    h5 = W.make_grads(cfg, 5, cfg.scale0, L, "cpu").numpy().view(np.uint16)
    assert h5[cfg.seed % (1 << 20)] == 0x7C00 and np.sum((h5 & 0x7FFF) >= 0x7C00) == 1


def test_overflow_grows_with_scale():
    cfg = W.get("gpt2_medium")
    # P(|g_true * S| >= 2^16) from the table rises with S
    p = [1 - W.cdf_table(cfg.grad_law, 2.0 ** k)[-1] / 2 ** 62 for k in (14, 16, 18, 20)]
    assert p == sorted(p) and p[0] < 1e-12 < p[2]


def test_cdf_tables_are_monotone():
    for cfg in W.CONFIGS.values():
        t = W.cdf_table(cfg.grad_law, cfg.scale0)
        assert np.all(np.diff(t) >= 0) and t[0] >= 0 and t[-1] <= 2 ** 62


def test_master_init_laws():
    cfg = miniature("gpt2_medium")
    m = W.make_master(cfg, "cpu")
    for spec, w in zip(cfg.tensors, m):
        if spec.init[0] == "const":
            assert torch.all(w == spec.init[1])
        elif w.numel() > 10000:
            assert abs(w.double().std().item() / spec.init[1] - 1) < 0.02
            assert abs(w.double().mean().item()) < 0.02 * spec.init[1] * 5
    assert torch.equal(torch.cat(m), torch.cat(W.make_master(cfg, "cpu")))


def test_truncated_sample():
    cfg = truncated(W.get("gpt2_medium"), 1_000_000)
    assert cfg.n_params == 1_000_000 and len(cfg.tensors) == 1
