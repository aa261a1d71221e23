"""The sharded step on the GPU.

* Emulated ranks: W shard handles on one GPU, each run through the library's
  two phases (check pass -> 32-byte record; combine-and-finish + update) with
  the collectives done in-process (FP16 sum of the ranks' gradients in rank
  order; concatenation of the records).  Nothing waits on another kernel, so
  the ranks can share one GPU.  The shards must reproduce the oracle's step
  over the whole list.
* One real rank: ShardedMPT over a single-rank NCCL group on cuda:0 runs the
  production code path (reduce-scatter, record all-gather, FP16 all-gather).
"""
import math
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from loss_scaled_fp32_b200 import (MPT, MPT_FLAG_COUNT_STALE, MPT_FLAG_GRAD_STATS, MPT_PARTIAL_BYTES,
                                   MPT_SCALER_DIRECT, Config, shard_len)

pytestmark = pytest.mark.gpu


def _grads(rng, padded, total):
    e = rng.integers(0, 24, padded)
    g = ((rng.integers(0, 2, padded) << 15) | (e << 10) | rng.integers(0, 1024, padded)).astype(np.uint16)
    g[rng.random(padded) < 0.03] = 0
    g[total:] = 0
    return g


@pytest.mark.parametrize("world", [2, 3, 4])
def test_emulated_ranks_match_the_whole_step(world):
    total = 300_001
    n = shard_len(total, world)
    padded = n * world
    rng = np.random.default_rng(world)
    master = np.zeros(padded, np.float32)
    master[:total] = rng.normal(0, 0.05, total).astype(np.float32)
    cfg = Config(growth_interval=2)
    shards = []
    for r in range(world):
        h = MPT([n], cfg)
        h.master(0).copy_(torch.from_numpy(master[r * n:(r + 1) * n]))
        h.refresh_half()
        h.set_scaler_state(2.0 ** 12, 0)
        shards.append(h)
    state = oracle.State.from_master([master])
    ocfg = oracle.scaler_cfg(growth_interval=2)
    S = 2.0 ** 12
    records = torch.empty(world * MPT_PARTIAL_BYTES, dtype=torch.uint8, device="cuda")
    for step in range(6):
        local = [_grads(rng, padded, total) for _ in range(world)]
        if step == 3:
            local[world - 1][total - 1] = 0x7C00
        # reduce-scatter, emulated: FP16 sum in rank order
        acc = torch.from_numpy(local[0].view(np.float16).copy()).cuda()
        for g in local[1:]:
            acc = acc + torch.from_numpy(g.view(np.float16).copy()).cuda()
        summed = acc.view(torch.int16)
        for r, h in enumerate(shards):
            rec = h.step_partial([summed[r * n:(r + 1) * n]])
            records[r * MPT_PARTIAL_BYTES:(r + 1) * MPT_PARTIAL_BYTES].copy_(rec)
        for h in shards:
            h.step_finish(records, world, 0.01, 0.9, 1e-4, clip=0.5)
        res = [h.wait() for h in shards]
        host = summed.cpu().numpy().view(np.uint16)
        ro = oracle.step(state, [host], S, 0.01, 0.9, 1e-4, clip=0.5, cfg=ocfg)
        for r in res:
            assert r["found_inf"] == ro["found_inf"] and r["n_nonfinite"] == ro["n_nonfinite"]
            assert r["new_scale"] == ro["new_scale"] and r["clean_run"] == ro["new_clean_run"]
            for k in ("found_inf", "clipped", "new_scale", "clean_run", "grad_norm", "clip_coef",
                      "n_nonfinite"):
                assert r[k] == res[0][k], k                     # identical on every rank
        # the range counts come from each rank's check pass: per shard
        assert sum(r["n_zero"] for r in res) == ro["n_zero"]
        assert sum(r["n_subnormal"] for r in res) == ro["n_subnormal"]
        if not ro["found_inf"]:
            assert abs(res[0]["grad_norm"] - ro["norm"]) <= 1e-5 * ro["norm"]
        S = ro["new_scale"]
        exact = res[0]["clip_coef"] == ro["clip_coef"]
        for r, h in enumerate(shards):
            sl = slice(r * n, (r + 1) * n)
            for got, want in ((h.master(0), state.master[0][sl]), (h.momentum(0), state.momentum[0][sl])):
                g = got.cpu().numpy()
                if exact:
                    assert g.tobytes() == want.tobytes(), (step, r)
                else:
                    assert np.max(np.abs(g.view(np.int32).astype(np.int64) -
                                         want.view(np.int32).astype(np.int64))) <= 1
            hw = h.w16(0).cpu().numpy().view(np.uint16)
            if exact:
                assert hw.tobytes() == state.w16[0][sl].tobytes()
    for h in shards:
        h.close()


@pytest.mark.parametrize("n,chunk,flags,mode", [
    (3_000_017, 0, MPT_FLAG_COUNT_STALE, 0),                    # 733 check bins: one level
    (5_000_011, 2048, MPT_FLAG_GRAD_STATS, MPT_SCALER_DIRECT),  # 2 442 bins: two levels
])
def test_whole_step_and_one_rank_sharded_step_agree_bit_for_bit(n, chunk, flags, mode):
    """In a whole step every update CTA adds the check kernel's partials (CTA
    0 writes the result and the next S); in a one-rank sharded step the check
    kernel's last CTA adds them into the 32-byte record, and the update adds
    the one record.  Both add the same partials in the same order, so from the
    same state and gradients they must leave the same bits -- results, loss
    scale, histogram, stale counts, master, momentum and FP16 copy -- over
    clean, clipped and overflowing steps."""
    rng = np.random.default_rng(n)
    master = rng.normal(0, 0.05, n).astype(np.float32)
    cfg = Config(growth_interval=2, check_chunk_elems=chunk, flags=flags, scaler_mode=mode)
    a, b = MPT([n], cfg), MPT([n], cfg)
    for h in (a, b):
        h.master(0).copy_(torch.from_numpy(master))
        h.refresh_half()
        h.set_scaler_state(2.0 ** 12, 0)
    g = torch.empty(n, dtype=torch.int16, device="cuda")
    seen = set()
    for step in range(6):
        host = _grads(rng, n, n)
        if step == 3:
            host[n // 2] = 0x7C00
        g.copy_(torch.from_numpy(host.view(np.int16)))
        a.step_async([g], 0.01, 0.9, 1e-4, clip=0.5)
        ra = a.wait()
        rec = b.step_partial([g]).clone()
        b.step_finish(rec, 1, 0.01, 0.9, 1e-4, clip=0.5)
        rb = b.wait()
        assert ra == rb, step
        seen.add("overflow" if ra["found_inf"] else "clipped" if ra["clipped"] else "clean")
        assert torch.equal(a.master(0).view(torch.int32), b.master(0).view(torch.int32)), step
        assert torch.equal(a.momentum(0).view(torch.int32), b.momentum(0).view(torch.int32)), step
        assert torch.equal(a.w16(0), b.w16(0)), step
        if flags & MPT_FLAG_GRAD_STATS:
            assert a.grad_histogram() == b.grad_histogram(), step
        sa, sb = a.stats(), b.stats()
        for k in ("steps", "skipped", "n_fp16_stale_total"):
            assert sa[k] == sb[k], (step, k)
    assert {"overflow", "clipped"} <= seen
    if flags & MPT_FLAG_COUNT_STALE:
        assert a.stats()["n_fp16_stale_total"] > 0
    a.close()
    b.close()


def test_sharded_optimizer_single_rank_nccl():
    import torch.distributed as dist
    from loss_scaled_fp32_b200.sharded import ShardedMPT

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        total = 123_457
        opt = ShardedMPT(total, Config(growth_interval=3))
        rng = np.random.default_rng(5)
        master = rng.normal(0, 0.05, total).astype(np.float32)
        opt.load_master(torch.from_numpy(master).cuda())
        opt.set_scale(2.0 ** 10)
        state = oracle.State.from_master([np.concatenate([master, np.zeros(opt.padded - total, np.float32)])])
        ocfg = oracle.scaler_cfg(growth_interval=3)
        S = 2.0 ** 10
        for step in range(5):
            g = _grads(rng, opt.padded, total)
            w16 = opt.step(torch.from_numpy(g.view(np.float16).copy()).cuda(), 0.01, 0.9, 1e-4, clip=1.0)
            r = opt.wait()
            ro = oracle.step(state, [g], S, 0.01, 0.9, 1e-4, clip=1.0, cfg=ocfg)
            assert r["new_scale"] == ro["new_scale"] and r["found_inf"] == ro["found_inf"]
            S = ro["new_scale"]
            if r["clip_coef"] == ro["clip_coef"]:
                assert w16.cpu().numpy().view(np.uint16).tobytes() == state.w16[0][:total].tobytes()
                assert opt.opt.master(0).cpu().numpy().tobytes() == state.master[0].tobytes()
        opt.close()
    finally:
        dist.destroy_process_group()
