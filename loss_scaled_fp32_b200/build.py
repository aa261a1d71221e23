"""Build libmpt (the C-ABI CUDA library) in-tree for sm_100a.

    python -m loss_scaled_fp32_b200.build [--force]

The library links only the CUDA runtime (static); torch is not involved.
A SHA-256 stamp of the sources and flags next to the .so decides whether a
rebuild is needed.
"""
import hashlib
import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmpt.so")
STAMP = LIB + ".sha256"
SOURCES = [os.path.join(CSRC, f) for f in ("mpt.cu", "mpt_kernels.cuh", "mpt_internal.h")] + \
    [os.path.join(ROOT, "include", "mpt.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O2",
    "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    # every float operation of the step is written out explicitly; nothing may
    # be contracted, flushed or approximated behind its back
    "-fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xptxas", "-v",
]


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: libmpt cannot be built")


def _digest():
    h = hashlib.sha256()
    for p in SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()


def _code_only(text):
    """The source without its comments and with whitespace runs collapsed
    (the device sources hold no string literal with a comment marker)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_digest():
    """SHA-256 of the device code (comments and layout aside) and its flags,
    to tell whether a stored profile was taken on the kernels as they are
    now."""
    h = hashlib.sha256()
    for name in ("mpt_kernels.cuh", "mpt_internal.h"):
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()


def build(force=False, verbose=False):
    digest = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == digest:
                return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, os.path.join(CSRC, "mpt.cu"), "-o", tmp]
    out = subprocess.run(cmd, capture_output=True, text=True)
    if out.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + out.stdout + out.stderr)
    if verbose:
        sys.stderr.write(out.stderr)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(digest)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
