"""The sharded step's exchange on the CPU: two gloo ranks, each holding its
own FP16 gradients of a flat list, split the list into the library's equal
shards, sum the gradients across ranks, compute their shard's 32-byte record
(sum of squares, non-finite count, largest finite magnitude) with the oracle,
exchange the records with the same helper the sharded optimizer uses, and
combine them in rank order.  Both ranks must hold bit-identical totals, and
they must agree with the oracle's pass over the whole (summed) list."""
import os
import socket
import struct
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

TOTAL = 100_003
WORLD = 2
SCALE = 2.0 ** 10


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_grads(rank, padded, bad):
    rng = np.random.default_rng(100 + rank)
    e = rng.integers(0, 26, padded)
    g = ((rng.integers(0, 2, padded) << 15) | (e << 10) | rng.integers(0, 1024, padded)).astype(np.uint16)
    g[rng.random(padded) < 0.05] = 0
    g[TOTAL:] = 0                                   # padding: always zero
    if bad and rank == 1:
        g[TOTAL - 7] = 0x7C00
    return g


def _record(r):
    """The library's record layout: binary64 sumsq, u64 non-finite count,
    u32 max magnitude, u32 error bits, 8 bytes of padding."""
    return struct.pack("<dQII8x", r.sumsq, r.n_nonfinite, r.max_mag16, 0)


def _worker(rank, port, bad, out):
    sys.path.insert(0, ROOT)
    import oracle
    from loss_scaled_fp32_b200 import MPT_PARTIAL_BYTES, shard_len
    from loss_scaled_fp32_b200.sharded import exchange_records

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    shard = shard_len(TOTAL, WORLD)
    padded = shard * WORLD
    local = _local_grads(rank, padded, bad)
    # the gradient sum across ranks (FP16 arithmetic, as the collective does)
    summed = torch.from_numpy(local.view(np.float16).copy())
    dist.all_reduce(summed)
    mine = summed.numpy().view(np.uint16)[rank * shard:(rank + 1) * shard].copy()
    rec = torch.frombuffer(bytearray(_record(oracle.check([mine], SCALE))), dtype=torch.uint8)
    records = torch.empty(WORLD * MPT_PARTIAL_BYTES, dtype=torch.uint8)
    exchange_records(records, rec)
    sumsq, nf, mm = 0.0, 0, 0
    for r in range(WORLD):
        s, n, m, _ = struct.unpack("<dQII8x", records[r * 32:(r + 1) * 32].numpy().tobytes())
        sumsq += s
        nf += n
        mm = max(mm, m)
    whole = oracle.check([summed.numpy().view(np.uint16)], SCALE)
    out.put((rank, sumsq, nf, mm, whole.sumsq, whole.n_nonfinite, whole.max_mag16))
    dist.destroy_process_group()


@pytest.mark.parametrize("bad", [False, True])
def test_two_rank_record_exchange_matches_the_whole_list(bad):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, bad, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, s0, n0, m0, w_s, w_n, w_m), (_, s1, n1, m1, _, _, _) = res
    assert (s0, n0, m0) == (s1, n1, m1)                    # identical on every rank
    assert n0 == w_n == (1 if bad else 0)
    assert m0 == w_m
    assert abs(s0 - w_s) <= 1e-12 * w_s                     # order of the binary64 sum only


def test_shard_len():
    from loss_scaled_fp32_b200 import shard_len
    assert shard_len(100_003, 2) == 50_016
    assert shard_len(16, 8) == 16
    assert shard_len(1, 1) == 16
    for total, world in ((354_823_168, 8), (1_509_985_436, 4), (17, 3)):
        n = shard_len(total, world)
        assert n % 16 == 0 and n * world >= total and (n - 16) * world < total
