"""Build the CPU oracle (plain C) into ``oracle/liboracle.so``.

Test infrastructure: compiled by ``__graft_entry__.build()`` and on demand by
the test suite; the product library never links it.
"""
import hashlib
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["oracle.c", "oracle.h"]
LIB = os.path.join(HERE, "liboracle.so")
STAMP = LIB + ".sha256"

# Every float operation must round once to binary32: no contraction into FMA,
# no fast-math, SSE scalar arithmetic (the x86-64 default).
CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
          "-fno-unsafe-math-optimizations", "-fPIC", "-shared", "-Wall", "-Wextra"]


def _digest():
    h = hashlib.sha256()
    for name in SOURCES:
        with open(os.path.join(HERE, name), "rb") as f:
            h.update(f.read())
    h.update(" ".join(CFLAGS).encode())
    return h.hexdigest()


def build(force=False):
    digest = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == digest:
                return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, os.path.join(HERE, "oracle.c"), "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(digest)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
