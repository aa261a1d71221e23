"""Seeded input generators (counter-based, identical recipe on CPU and CUDA).

Every random number is a 32-bit integer hash of (seed, stream, element
index), computed with int64 torch arithmetic kept below 2^63 so that CPU and
CUDA give the same bits.  Gradients are drawn as binary16 *bit patterns*:

  1. the magnitude code k (0 .. 0x7C00) is found by comparing a 62-bit
     uniform integer with a cumulative table of the workload's |g_true * S|
     law, where code k stands for the interval [v_k, v_{k+1}) of magnitudes
     (floor quantisation onto the binary16 grid; v_0 = 0, v_0x7C00 = 2^16,
     so values below 2^-24 become 0 and values of 2^16 and more become inf);
  2. the sign is one more uniform bit.

No binary16 rounding routine is involved, so the generator shares none with
the oracle or the kernels.  Overflow therefore arises naturally when S grows,
as in real loss-scaled training.
"""
import math
from typing import Iterable, List, Sequence

import numpy as np
import torch

M32 = 0xFFFFFFFF
_MUL = 0x45D9F3B  # odd multiplier below 2^31: products stay below 2^63 in int64
_CHUNK = 1 << 25


def _hash32_t(x: torch.Tensor) -> torch.Tensor:
    """Integer mixing of 32-bit values held in int64 (shift-xor-multiply)."""
    x = x ^ (x >> 16)
    x = (x * _MUL) & M32
    x = x ^ (x >> 16)
    x = (x * _MUL) & M32
    x = x ^ (x >> 16)
    return x


def _hash32_py(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * _MUL) & M32
    x ^= x >> 16
    x = (x * _MUL) & M32
    x ^= x >> 16
    return x


def _stream_key(seed: int, stream: int, step: int) -> int:
    return _hash32_py(_hash32_py(_hash32_py(seed) ^ (stream * 0x9E3779B1 & M32)) + step)


def uniform_u32(seed: int, stream: int, step: int, idx: torch.Tensor) -> torch.Tensor:
    """32-bit uniform integers for element indices ``idx`` (int64, < 2^32)."""
    k = _stream_key(seed, stream, step)
    # the second round's key must not equal the first round of any small
    # index (a hash of k + 1 would cancel element 1 to exactly 0)
    k2 = _hash32_py((k * 0x9E3779B1 + 0x7F4A7C15) & M32)
    return _hash32_t(_hash32_t((idx + k) & M32) ^ k2)


# ---------------------------------------------------------------------------
# gradient magnitude tables
# ---------------------------------------------------------------------------

def fp16_magnitude_values() -> np.ndarray:
    """Value of every non-negative binary16 code 0 .. 0x7BFF (numpy's own
    conversion), followed by 2^16 as the upper edge of the last finite code."""
    v = np.arange(0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    return np.concatenate([v, [65536.0]])


def _law_sf(law, x: np.ndarray) -> np.ndarray:
    """P(|g_true| >= x) for the workload's gradient law, computed as an upper
    tail (erfc, not 1 - cdf) so that tiny overflow probabilities keep their
    precision."""
    kind = law[0]
    with np.errstate(divide="ignore"):
        lx = np.log2(x)
    if kind == "log2_uniform":
        lo, hi = law[1], law[2]
        return np.clip((hi - lx) / (hi - lo), 0.0, 1.0)
    if kind == "log2_normal":
        mean, std = law[1], law[2]
        z = (lx - mean) / (std * math.sqrt(2.0))
        return np.array([0.5 * math.erfc(t) if np.isfinite(t) else (1.0 if t < 0 else 0.0)
                         for t in z])
    if kind == "normal":
        std = law[1]
        return np.array([math.erfc(t / (std * math.sqrt(2.0))) for t in x])
    raise ValueError(law)


_TABLES = {}
Q_BITS = 62  # resolution of the uniform that selects a magnitude code


def cdf_table(law, scale: float) -> np.ndarray:
    """Thresholds T[k] = 2^62 - round(2^62 * P(|g_true * S| >= v_{k+1})),
    k = 0 .. 0x7BFF.  A 62-bit uniform q selects code #{k : T[k] <= q}
    (0x7C00 = inf), so code k has probability P(v_k <= |g_true S| < v_{k+1})
    to within 2^-62."""
    key = (tuple(law), float(scale))
    if key not in _TABLES:
        upper = fp16_magnitude_values()[1:] / float(scale)
        sf = _law_sf(law, upper)
        full = 1 << Q_BITS
        _TABLES[key] = np.array([full - int(round(p * full)) for p in sf], dtype=np.int64)
    return _TABLES[key]


# ---------------------------------------------------------------------------
# layouts
# ---------------------------------------------------------------------------

class GradLayout:
    """Where each gradient tensor sits in one flat binary16 buffer.

    Offsets are rounded up to ``align`` elements (16 elements = 32 bytes, as a
    framework's allocator would give); tensors listed in ``shifted`` start one
    element (2 bytes) later, to exercise unaligned gradient pointers."""

    def __init__(self, sizes: Sequence[int], align: int = 16, shifted: Iterable[int] = ()):
        shifted = set(shifted)
        self.sizes = [int(s) for s in sizes]
        self.offsets = []
        off = 0
        for i, s in enumerate(self.sizes):
            off = (off + align - 1) // align * align
            if i in shifted:
                off += 1
            self.offsets.append(off)
            off += s
        self.total = (off + align - 1) // align * align
        starts = np.cumsum([0] + self.sizes[:-1]).astype(np.int64)
        self.list_starts = [int(x) for x in starts]  # index of element 0 in the whole list

    def views(self, flat: torch.Tensor) -> List[torch.Tensor]:
        return [flat[o:o + s] for o, s in zip(self.offsets, self.sizes)]


# ---------------------------------------------------------------------------
# gradients and master weights
# ---------------------------------------------------------------------------

_GRAD_STREAM, _GRAD_STREAM2, _SIGN_STREAM = 11, 13, 12
_MASTER_STREAM_A, _MASTER_STREAM_B = 21, 22


def make_grads(cfg, step: int, scale: float, layout: GradLayout, device="cpu",
               out: torch.Tensor = None) -> torch.Tensor:
    """Binary16 bit patterns (int16 tensor, flat in ``layout``) of the scaled
    gradients of ``cfg`` at ``step`` (1-based) for loss scale ``scale``, with
    the workload's inf/NaN injections applied.  Element j of the whole list
    (tensors concatenated in order) is drawn from counter j, whatever the
    layout, so every layout of a workload carries the same values."""
    table = torch.from_numpy(cdf_table(cfg.grad_law, scale)).to(device)
    if out is None:
        out = torch.zeros(layout.total, dtype=torch.int16, device=device)
    starts = torch.tensor(layout.list_starts, dtype=torch.int64, device=device)
    delta = torch.tensor([o - s for o, s in zip(layout.offsets, layout.list_starts)],
                         dtype=torch.int64, device=device)
    total = sum(layout.sizes)
    for c0 in range(0, total, _CHUNK):
        n = min(_CHUNK, total - c0)
        idx = torch.arange(c0, c0 + n, dtype=torch.int64, device=device)
        q = ((uniform_u32(cfg.seed, _GRAD_STREAM, step, idx) >> 1) << 31) | \
            (uniform_u32(cfg.seed, _GRAD_STREAM2, step, idx) >> 1)
        code = torch.searchsorted(table, q, right=True)
        sign = (uniform_u32(cfg.seed, _SIGN_STREAM, step, idx) & 1) << 15
        bits = code | sign
        bits = (bits - ((bits >> 15) << 16)).to(torch.int16)
        if len(layout.sizes) == 1:
            out[layout.offsets[0] + c0: layout.offsets[0] + c0 + n] = bits
        else:
            t = torch.searchsorted(starts, idx, right=True) - 1
            out[idx + delta[t]] = bits
    for t, e, b in cfg.injections(step):
        if t < len(layout.sizes):
            out[layout.offsets[t] + e] = b - 65536 if b >= 32768 else b
    return out


def make_master(cfg, device="cpu") -> List[torch.Tensor]:
    """FP32 master weights, one tensor per list entry (views of one flat
    buffer): N(0, std) by Box-Muller on hashed uniforms of the element's index
    in the whole list, or constants (norm-layer gains 1, biases 0)."""
    sizes = [t.size for t in cfg.tensors]
    total = sum(sizes)
    starts = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)
    std = torch.tensor([float(t.init[1]) if t.init[0] == "normal" else 0.0 for t in cfg.tensors],
                       dtype=torch.float64, device=device)
    const = torch.tensor([float(t.init[1]) if t.init[0] == "const" else 0.0 for t in cfg.tensors],
                         dtype=torch.float32, device=device)
    is_const = torch.tensor([t.init[0] == "const" for t in cfg.tensors], device=device)
    starts_t = torch.from_numpy(starts).to(device)
    flat = torch.empty(total, dtype=torch.float32, device=device)
    for c0 in range(0, total, _CHUNK):
        n = min(_CHUNK, total - c0)
        idx = torch.arange(c0, c0 + n, dtype=torch.int64, device=device)
        t = torch.searchsorted(starts_t, idx, right=True) - 1
        u1 = (uniform_u32(cfg.seed, _MASTER_STREAM_A, 0, idx).double() + 1.0) / 4294967296.0
        u2 = uniform_u32(cfg.seed, _MASTER_STREAM_B, 0, idx).double() / 4294967296.0
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
        w = (z * std[t]).float()
        flat[c0:c0 + n] = torch.where(is_const[t], const[t], w)
    return [flat[int(s):int(s) + n] for s, n in zip(starts, sizes)]
