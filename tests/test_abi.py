"""CPU checks of the C-ABI library: it builds for sm_100a, loads, exports every
function ``include/mpt.h`` declares, and its host-side logic (defaults,
workspace sizing, argument validation, error strings) behaves, without any
compute call (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import loss_scaled_fp32_b200 as lsf
from loss_scaled_fp32_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mpt.h")


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^(?:int|const char\*)\s+(mpt_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mpt_create", "mpt_step", "mpt_stats", "mpt_workspace_bytes",
                     "mpt_tensor_views", "mpt_refresh_half", "mpt_get_scaler_state",
                     "mpt_set_scaler_state", "mpt_destroy", "mpt_error_string"):
        assert required in names


def test_library_builds_and_exports_every_declared_symbol():
    path = mbuild.build()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (mpt_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert missing == []
    L = lsf.lib()
    for n in declared_functions():
        assert hasattr(L, n)


def test_defaults_and_config_validation():
    c = lsf.Config()
    assert (c.backoff, c.growth, c.growth_interval) == (0.5, 2.0, 0)
    assert (c.min_scale, c.max_scale, c.flags) == (2.0 ** -24, 2.0 ** 24, 0)
    assert (c.check_chunk_elems, c.update_chunk_elems) == (0, 0)
    L = lsf.lib()
    sizes = (ctypes.c_int64 * 2)(10, 20)
    nb = ctypes.c_size_t()
    for bad in (dict(check_chunk_elems=1000), dict(check_chunk_elems=1 << 21),
                dict(update_chunk_elems=3000), dict(backoff=0.0),
                dict(backoff=1.5), dict(growth=0.5), dict(growth_interval=-1),
                dict(min_scale=0.0), dict(flags=0x100), dict(min_scale=4.0, max_scale=2.0)):
        assert L.mpt_workspace_bytes(sizes, 2, ctypes.byref(lsf.Config(**bad)),
                                     ctypes.byref(nb)) == lsf.MPT_ERR_INVALID_ARG, bad


def test_workspace_bytes():
    L = lsf.lib()

    def ws(sizes, **cfg):
        arr = (ctypes.c_int64 * len(sizes))(*sizes)
        nb = ctypes.c_size_t()
        rc = L.mpt_workspace_bytes(arr, len(sizes), ctypes.byref(lsf.Config(**cfg)) if cfg else None,
                                   ctypes.byref(nb))
        return rc, nb.value

    rc, b = ws([1_000_000])
    assert rc == 0
    assert b >= 10 * 1_000_000               # master + momentum + FP16 copy
    assert b < 10 * 1_000_000 + 64 * 1024
    rc, b2 = ws([1, 1, 1])                     # each tensor padded to 16 elements
    assert rc == 0 and b2 >= 10 * 48
    assert ws([5, 0])[0] == lsf.MPT_ERR_INVALID_ARG
    assert ws([-3])[0] == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_workspace_bytes(None, 1, None, ctypes.byref(ctypes.c_size_t())) == lsf.MPT_ERR_INVALID_ARG
    arr = (ctypes.c_int64 * 1)(5)
    assert L.mpt_workspace_bytes(arr, 0, None, ctypes.byref(ctypes.c_size_t())) == lsf.MPT_ERR_INVALID_ARG
    # smaller chunks mean more bins, hence more table bytes, never fewer
    assert ws([10_000_000], update_chunk_elems=2048)[1] > ws([10_000_000])[1]
    assert ws([10_000_000], check_chunk_elems=2048)[1] > ws([10_000_000])[1]


def test_default_check_bins_follow_the_list_size():
    """Default check bins: 64K elements, halved (to 2048 at least) while the
    list would give fewer than 592 bins.  Only the check table's size depends
    on the chunk, so the explicit chunk whose workspace equals the default's
    is the one the default chose; its neighbours differ by hundreds of bins,
    which the 256-byte region rounding cannot hide."""
    import workloads as W
    L = lsf.lib()

    def ws(sizes, **cfg):
        arr = (ctypes.c_int64 * len(sizes))(*sizes)
        nb = ctypes.c_size_t()
        assert L.mpt_workspace_bytes(arr, len(sizes), ctypes.byref(lsf.Config(**cfg)),
                                     ctypes.byref(nb)) == 0
        return nb.value

    cases = [([1 << 20], 2048),                    # 512 bins; the floor (4K would give 256)
             ([10_000_000], 16384),                # 611 bins; 32K would give 306
             ([38_700_000], 32768),                # 64K gives 591 < 592: halved
             ([38_900_000], 65536),                # 64K gives 594: kept
             (W.get("resnet50").sizes, 32768)]     # 780 bins of 32K; 64K would give 390
    for sizes, chunk in cases:
        assert ws(sizes) == ws(sizes, check_chunk_elems=chunk), (sizes[:2], chunk)
        for other in (chunk // 2, chunk * 2):
            if 2048 <= other <= 65536:
                assert ws(sizes, check_chunk_elems=other) != ws(sizes), (sizes[:2], other)
    assert ws([5000]) == ws([5000], check_chunk_elems=2048)   # nothing below 2048


def test_invalid_handles_and_arguments_return_codes():
    L = lsf.lib()
    r = lsf.StepResult()
    assert L.mpt_step(None, None, 1.0, 0.1, 0.9, 0.0, 0.0, None, ctypes.byref(r)) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_refresh_half(None, None) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_stats(None, ctypes.byref(lsf.Stats())) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_set_scaler_state(None, 1.0, 0) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_set_timing(None, 1) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_set_timing(None, -1) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_debug_fail_next_step(None) == lsf.MPT_ERR_INVALID_ARG
    assert L.mpt_destroy(None) == 0
    sizes = (ctypes.c_int64 * 1)(100)
    h = ctypes.c_void_p()
    # host memory is not a device workspace (and there may be no device at all)
    buf = ctypes.create_string_buffer(1 << 16)
    rc = L.mpt_create(sizes, 1, None, ctypes.c_void_p(ctypes.addressof(buf)), 1 << 16, ctypes.byref(h))
    assert rc in (lsf.MPT_ERR_WORKSPACE, lsf.MPT_ERR_CUDA) and not h.value
    # too small / misaligned workspace is rejected before any CUDA call
    rc = L.mpt_create(sizes, 1, None, ctypes.c_void_p(256), 16, ctypes.byref(h))
    assert rc == lsf.MPT_ERR_WORKSPACE
    rc = L.mpt_create(sizes, 1, None, ctypes.c_void_p(ctypes.addressof(buf) | 8), 1 << 16, ctypes.byref(h))
    assert rc == lsf.MPT_ERR_WORKSPACE


def test_error_strings():
    L = lsf.lib()
    for code in (0, -1, -2, -3, -4, -5, 17):
        s = L.mpt_error_string(code)
        assert isinstance(s, bytes) and len(s) > 0


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    import importlib
    monkeypatch.setattr(mbuild, "LIB", str(tmp_path / "absent" / "libmpt.so"))

    def no_nvcc():
        raise RuntimeError("nvcc not found: libmpt cannot be built")
    monkeypatch.setattr(mbuild, "nvcc", no_nvcc)
    monkeypatch.setattr(lsf, "_LIB", None)
    with pytest.raises(RuntimeError):
        lsf.lib()
    monkeypatch.setattr(lsf, "_LIB", None)

def test_plain_c_consumer_compiles_links_and_runs(tmp_path):
    """The header is strict C99 and the library links from C: a plain C
    program takes the address of every declared entry point and runs the
    calls that need no GPU (tests/native/abi_consumer.c)."""
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    lib_path = lsf.lib()._name
    lib_dir = os.path.dirname(lib_path)
    exe = str(tmp_path / "abi_consumer")
    build = subprocess.run(
        [gcc, "-std=c99", "-Wall", "-Wextra", "-Wpedantic", "-Werror",
         "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "native", "abi_consumer.c"),
         "-L", lib_dir, "-lmpt", "-Wl,-rpath," + lib_dir, "-o", exe],
        capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert "21 entry points" in run.stdout
