"""P6: the oracle's binary16 codec, exhaustively, against two independent
conversions: the x86 F16C instructions (all 2^32 binary32 inputs, in C) and
torch's CPU ``float32 -> float16`` conversion (all 2^32 inputs, chunked)."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))


def _has_f16c():
    try:
        with open("/proc/cpuinfo") as f:
            return " f16c" in f.read()
    except OSError:
        return False


@pytest.mark.skipif(not _has_f16c(), reason="host CPU lacks F16C")
def test_p6_codec_exhaustive_vs_f16c():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "codec_exhaustive")
        subprocess.run(["gcc", "-O2", "-fopenmp", "-mf16c", "-ffp-contract=off",
                        "-I", oracle_build.HERE,
                        os.path.join(HERE, "native", "codec_exhaustive.c"),
                        os.path.join(oracle_build.HERE, "oracle.c"), "-o", exe, "-lm"],
                       check=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0, out.stdout + out.stderr
        assert "narrow_mismatch 0 nan_mismatch 0 widen_mismatch 0" in out.stdout


def test_p6_widen_exhaustive_vs_numpy():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = oracle.widen16(h)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_p6_narrow_exhaustive_vs_torch():
    torch = pytest.importorskip("torch")
    from concurrent.futures import ThreadPoolExecutor

    chunk = 1 << 24
    base = np.arange(chunk, dtype=np.uint32)

    def one(c):
        x = (base + np.uint32(c * chunk)).view(np.float32)
        ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
        got = oracle.rne16(x)       # ctypes releases the GIL: chunks run in parallel
        nan = np.isnan(x)
        if nan.any():
            # NaN: only NaN-ness and sign are specified
            g, r = got[nan], ref[nan]
            if not (np.all(((g & 0x7C00) == 0x7C00) & ((g & 0x3FF) != 0))
                    and np.array_equal(g & 0x8000, r & 0x8000)):
                return c
        return None if np.array_equal(got[~nan], ref[~nan]) else c

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        bad = [c for c in ex.map(one, range(1 << 32 >> 24)) if c is not None]
    assert bad == []
