"""Parameter lists and hyperparameters of the five synthetic workloads.

The pages train CNNs and RNNs of more than 100 million parameters (ResNet-50
on ILSVRC, speech models of 115M-215M parameters, language models); these
lists stand in for them with the shapes of well-known architectures and
random-initialised weights.  No dataset or trained weight is involved.
"""
import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class TensorSpec:
    name: str
    shape: Tuple[int, ...]
    init: Tuple  # ("normal", std) | ("const", value)

    @property
    def size(self):
        return int(np.prod(self.shape, dtype=np.int64))


@dataclass
class Config:
    name: str
    tensors: List[TensorSpec]
    # |g_true| law: ("log2_uniform", lo, hi) | ("log2_normal", mean, std) | ("normal", std)
    grad_law: Tuple
    scale0: float
    growth_interval: int        # 0: constant S (still backs off on overflow)
    lr: float
    momentum: float
    weight_decay: float
    clip: float                 # <= 0: off
    steps: int
    seed: int
    backoff: float = 0.5
    growth: float = 2.0
    # step (1-based) -> list of (tensor index, element index, binary16 bits)
    injections: Callable = field(default=lambda step: [])

    @property
    def sizes(self):
        return [t.size for t in self.tensors]

    @property
    def n_params(self):
        return int(sum(self.sizes))


# ---------------------------------------------------------------------------
# shapes
# ---------------------------------------------------------------------------

def _resnet50():
    T = []

    def conv(name, cout, cin, k):
        T.append(TensorSpec(name, (cout, cin, k, k), ("normal", math.sqrt(2.0 / (cin * k * k)))))

    def bn(name, c):
        T.append(TensorSpec(name + ".weight", (c,), ("const", 1.0)))
        T.append(TensorSpec(name + ".bias", (c,), ("const", 0.0)))

    conv("conv1.weight", 64, 3, 7)
    bn("bn1", 64)
    cin = 64
    for stage, (blocks, width) in enumerate(zip([3, 4, 6, 3], [64, 128, 256, 512]), start=1):
        for b in range(blocks):
            p = f"layer{stage}.{b}"
            conv(p + ".conv1.weight", width, cin, 1)
            bn(p + ".bn1", width)
            conv(p + ".conv2.weight", width, width, 3)
            bn(p + ".bn2", width)
            conv(p + ".conv3.weight", width * 4, width, 1)
            bn(p + ".bn3", width * 4)
            if b == 0:
                conv(p + ".downsample.0.weight", width * 4, cin, 1)
                bn(p + ".downsample.1", width * 4)
            cin = width * 4
    T.append(TensorSpec("fc.weight", (1000, 2048), ("normal", math.sqrt(2.0 / 2048))))
    T.append(TensorSpec("fc.bias", (1000,), ("const", 0.0)))
    return T


def _gpt(layers, d, ffn, vocab, positions, std=0.02):
    T = [TensorSpec("wte", (vocab, d), ("normal", std)),
         TensorSpec("wpe", (positions, d), ("normal", std))]
    for i in range(layers):
        p = f"h.{i}"
        T += [TensorSpec(p + ".ln_1.weight", (d,), ("const", 1.0)),
              TensorSpec(p + ".ln_1.bias", (d,), ("const", 0.0)),
              TensorSpec(p + ".attn.c_attn.weight", (d, 3 * d), ("normal", std)),
              TensorSpec(p + ".attn.c_attn.bias", (3 * d,), ("const", 0.0)),
              TensorSpec(p + ".attn.c_proj.weight", (d, d), ("normal", std)),
              TensorSpec(p + ".attn.c_proj.bias", (d,), ("const", 0.0)),
              TensorSpec(p + ".ln_2.weight", (d,), ("const", 1.0)),
              TensorSpec(p + ".ln_2.bias", (d,), ("const", 0.0)),
              TensorSpec(p + ".mlp.c_fc.weight", (d, ffn), ("normal", std)),
              TensorSpec(p + ".mlp.c_fc.bias", (ffn,), ("const", 0.0)),
              TensorSpec(p + ".mlp.c_proj.weight", (ffn, d), ("normal", std)),
              TensorSpec(p + ".mlp.c_proj.bias", (d,), ("const", 0.0))]
    T += [TensorSpec("ln_f.weight", (d,), ("const", 1.0)),
          TensorSpec("ln_f.bias", (d,), ("const", 0.0))]
    return T


def ragged_sizes(n=20000, seed=20000, log_max=20):
    """Sizes floor(exp(U[0, ln 2^log_max))), at least 1 (log-uniform 1..2^20)."""
    rng = np.random.default_rng(seed)
    u = rng.uniform(0.0, log_max * math.log(2.0), n)
    return np.maximum(np.floor(np.exp(u)), 1).astype(np.int64)


def _ragged(n=20000, seed=20000):
    return [TensorSpec(f"t{i}", (int(s),), ("normal", 0.05))
            for i, s in enumerate(ragged_sizes(n, seed))]


# ---------------------------------------------------------------------------
# overflow injections
# ---------------------------------------------------------------------------

def _flat1m_injections(step, seed=1, n=1 << 20):
    # step 5: one gradient is +inf
    return [(0, seed % n, 0x7C00)] if step == 5 else []


def _ragged_injections_factory(sizes, seed, steps=200, count=20):
    rng = np.random.default_rng(seed + 7)
    chosen = rng.permutation(steps)[:count] + 1
    plan = {}
    patterns = [0x7C00, 0xFC00, 0x7E00]          # +inf, -inf, NaN
    for s in sorted(chosen.tolist()):
        t = int(rng.integers(0, len(sizes)))
        plan[s] = [(t, int(rng.integers(0, sizes[t])), patterns[int(rng.integers(0, 3))])]
    return lambda step: plan.get(step, [])


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

def _build():
    C = {}
    C["flat1m"] = Config(
        name="flat1m", tensors=[TensorSpec("w", (1 << 20,), ("normal", 0.05))],
        grad_law=("log2_uniform", -30.0, -6.0), scale0=1024.0, growth_interval=0,
        lr=0.01, momentum=0.9, weight_decay=1e-4, clip=0.0, steps=10, seed=1,
        injections=_flat1m_injections)
    C["resnet50"] = Config(
        name="resnet50", tensors=_resnet50(), grad_law=("log2_uniform", -28.0, -4.0),
        scale0=128.0, growth_interval=0, lr=0.01, momentum=0.9, weight_decay=1e-4,
        clip=0.0, steps=100, seed=2)
    C["gpt2_medium"] = Config(
        name="gpt2_medium", tensors=_gpt(24, 1024, 4096, 50257, 1024),
        grad_law=("log2_normal", -20.0, 3.0), scale0=2.0 ** 16, growth_interval=4,
        lr=0.01, momentum=0.9, weight_decay=0.01, clip=1.0, steps=50, seed=3)
    C["gpt_1p3b"] = Config(
        name="gpt_1p3b", tensors=_gpt(24, 2048, 8192, 50257, 2048),
        grad_law=("normal", 1e-3), scale0=2.0 ** 12, growth_interval=0,
        lr=0.01, momentum=0.9, weight_decay=0.01, clip=0.0, steps=20, seed=4)
    rag = _ragged()
    C["ragged20k"] = Config(
        name="ragged20k", tensors=rag, grad_law=("log2_uniform", -30.0, 0.0),
        scale0=2.0 ** 10, growth_interval=4, lr=0.01, momentum=0.9, weight_decay=1e-4,
        clip=0.0, steps=200, seed=5,
        injections=_ragged_injections_factory([t.size for t in rag], 5))
    return C


CONFIGS = _build()
EXPECTED_PARAMS = {"flat1m": 1 << 20, "resnet50": 25_557_032, "gpt2_medium": 354_823_168,
                   "gpt_1p3b": 1_315_723_264}
EXPECTED_TENSORS = {"flat1m": 1, "resnet50": 161, "gpt2_medium": 292, "gpt_1p3b": 292,
                    "ragged20k": 20000}


def get(name) -> Config:
    return CONFIGS[name]


def truncated(cfg: Config, max_params: int) -> Config:
    """The leading ``max_params`` parameters of a workload, in list order (the
    last tensor kept is cut short) -- the bounded sample the CPU baseline is
    timed on."""
    keep, total = [], 0
    for t in cfg.tensors:
        if total >= max_params:
            break
        take = min(t.size, max_params - total)
        keep.append(t if take == t.size else TensorSpec(t.name + "[:%d]" % take, (take,), t.init))
        total += take
    return Config(**{**cfg.__dict__, "tensors": keep, "name": cfg.name + "_lead%d" % total})


def miniature(name: str) -> Config:
    """The same workload with every dimension shrunk (same tensor count, same
    kinds of tensors, same laws and hyperparameters): small enough for the
    oracle to run many steps in seconds."""
    cfg = CONFIGS[name]
    if name == "gpt2_medium":
        tensors = _gpt(24, 128, 512, 5025, 128)
    elif name == "gpt_1p3b":
        tensors = _gpt(24, 256, 1024, 5025, 256)
    elif name == "ragged20k":
        tensors = [TensorSpec(f"t{i}", (int(s),), ("normal", 0.05))
                   for i, s in enumerate(ragged_sizes(n=3000, seed=11, log_max=14))]
    else:
        return cfg
    return Config(**{**cfg.__dict__, "tensors": tensors, "name": name + "_mini",
                     "injections": (lambda step: [])})
