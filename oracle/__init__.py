"""ctypes front end of the CPU oracle (``oracle/oracle.c``).

TEST INFRASTRUCTURE ONLY.  The oracle is the plain, slow, single-threaded
restatement of the loss-scaled FP32-master SGD-momentum step that the CUDA
library is checked against.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the product package
never does, and it has no CPU fallback through this module.

Arrays are numpy: FP16 data is carried as ``uint16`` bit patterns so that no
library conversion sits between the oracle and its inputs.
"""
import ctypes
import os
from dataclasses import dataclass, field
from typing import List

import numpy as np

from . import build as _build

_LIB = None

NO_MASTER = 1  # ORC_NO_MASTER: ablation mode, FP16 weights updated directly
NESTEROV = 2   # ORC_NESTEROV: Nesterov momentum
ADAGRAD = 4    # ORC_ADAGRAD: Adagrad (the momentum array holds sum of d^2)


SCALER_DYNAMIC, SCALER_DIRECT = 0, 1


class ScalerCfg(ctypes.Structure):
    _fields_ = [("backoff", ctypes.c_float), ("growth", ctypes.c_float),
                ("growth_interval", ctypes.c_int32), ("min_scale", ctypes.c_float),
                ("max_scale", ctypes.c_float), ("mode", ctypes.c_int32),
                ("direct_margin", ctypes.c_float)]


def scaler_cfg(backoff=0.5, growth=2.0, growth_interval=0, min_scale=2.0 ** -24,
               max_scale=2.0 ** 24, mode=SCALER_DYNAMIC, direct_margin=2.0):
    return ScalerCfg(backoff, growth, growth_interval, min_scale, max_scale, mode,
                     direct_margin)


class _Result(ctypes.Structure):
    _fields_ = [("found_inf", ctypes.c_int32), ("clipped", ctypes.c_int32),
                ("sumsq", ctypes.c_double), ("norm", ctypes.c_double),
                ("clip_coef", ctypes.c_float), ("n_zero", ctypes.c_uint64),
                ("n_subnormal", ctypes.c_uint64), ("n_nonfinite", ctypes.c_uint64),
                ("n_stale", ctypes.c_uint64), ("new_scale", ctypes.c_float),
                ("new_clean_run", ctypes.c_int32), ("max_mag16", ctypes.c_uint16),
                ("max_abs", ctypes.c_float), ("exp_hist", ctypes.c_uint64 * 32)]

    def as_dict(self):
        d = {name: getattr(self, name) for name, _ in self._fields_}
        d["exp_hist"] = list(self.exp_hist)
        return d


def lib():
    global _LIB
    if _LIB is None:
        # ORACLE_LIB lets the mutation test load a deliberately broken build
        # of the oracle and confirm that the pins reject it.
        path = os.environ.get("ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        vp, i64, i32, u32, f32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t)
        L.orc_rne16.argtypes, L.orc_rne16.restype = [f32], ctypes.c_uint16
        L.orc_widen16.argtypes, L.orc_widen16.restype = [ctypes.c_uint16], f32
        L.orc_rne16_array.argtypes, L.orc_rne16_array.restype = [vp, vp, sz], None
        L.orc_widen16_array.argtypes, L.orc_widen16_array.restype = [vp, vp, sz], None
        L.orc_check.argtypes = [vp, vp, i32, f32, ctypes.POINTER(_Result)]
        L.orc_check.restype = None
        L.orc_clip_coef.argtypes = [ctypes.POINTER(_Result), f32]
        L.orc_clip_coef.restype = None
        L.orc_update.argtypes = [i64, vp, vp, vp, vp, f32, i32, f32, f32, f32, f32, f32, u32]
        L.orc_update.restype = ctypes.c_uint64
        L.orc_scaler_next.argtypes = [ctypes.POINTER(ScalerCfg), i32, f32, f32,
                                      ctypes.POINTER(ctypes.c_int32)]
        L.orc_scaler_next.restype = f32
        L.orc_step.argtypes = [vp, vp, vp, vp, vp, i32, f32, f32, f32, f32, f32, f32,
                               ctypes.POINTER(ScalerCfg), ctypes.POINTER(ctypes.c_int32),
                               u32, ctypes.POINTER(_Result)]
        L.orc_step.restype = None
        L.orc_direct_scale.argtypes = [f32, f32, f32, f32]
        L.orc_direct_scale.restype = f32
        _LIB = L
    return _LIB


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _ptr_array(arrays):
    return (ctypes.c_void_p * len(arrays))(*[a.ctypes.data for a in arrays])


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


# ---- codec ------------------------------------------------------------------

def rne16(x):
    """binary32 -> binary16 bits (uint16), round to nearest even."""
    x = _c(np.asarray(x, dtype=np.float32), np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_rne16_array(_ptr(x), _ptr(out), x.size)
    return out


def widen16(h):
    """binary16 bits (uint16) -> binary32, exact."""
    h = _c(np.asarray(h, dtype=np.uint16), np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    lib().orc_widen16_array(_ptr(h), _ptr(out), h.size)
    return out


# ---- step -------------------------------------------------------------------

@dataclass
class State:
    """Per-tensor optimizer state: FP32 master, FP32 momentum, FP16 copy."""
    master: List[np.ndarray]
    momentum: List[np.ndarray]
    w16: List[np.ndarray]
    clean_run: int = 0
    scale_history: list = field(default_factory=list)

    @classmethod
    def from_master(cls, master):
        master = [np.ascontiguousarray(m, dtype=np.float32).copy() for m in master]
        return cls(master=master,
                   momentum=[np.zeros_like(m) for m in master],
                   w16=[rne16(m) for m in master])

    def copy(self):
        return State([m.copy() for m in self.master], [v.copy() for v in self.momentum],
                     [h.copy() for h in self.w16], self.clean_run, list(self.scale_history))


def check(grads, scale):
    """Pass 1 only: found_inf, counts and sumsq (no state needed)."""
    grads = [_c(g, np.uint16) for g in grads]
    sizes = np.array([g.size for g in grads], dtype=np.int64)
    r = _Result()
    lib().orc_check(_ptr_array(grads), _ptr(sizes), len(grads),
                    ctypes.c_float(np.float32(1.0) / np.float32(scale)), ctypes.byref(r))
    return r


def clip_coef(r, clip):
    lib().orc_clip_coef(ctypes.byref(r), clip)
    return r


def update(g16, w, v, w16, scale, clipped, coef, lr, momentum, weight_decay, flags=0,
           eps=1e-10):
    """Pass 2 on one set of elements (arrays are updated in place)."""
    g16 = _c(g16, np.uint16)
    for a, dt in ((w, np.float32), (v, np.float32), (w16, np.uint16)):
        assert a.flags.c_contiguous and a.dtype == dt
    inv = np.float32(1.0) / np.float32(scale)
    return lib().orc_update(g16.size, _ptr(g16), _ptr(w), _ptr(v), _ptr(w16), inv,
                            int(clipped), coef, lr, momentum, weight_decay, eps, flags)


def direct_scale(max_abs, margin=2.0, min_scale=2.0 ** -24, max_scale=2.0 ** 24):
    """S = 65504 / (margin * max|g|) (binary64, rounded to binary32, clamped)."""
    return lib().orc_direct_scale(max_abs, margin, min_scale, max_scale)


def scaler_next(cfg, found_inf, scale, clean_run, max_abs=0.0):
    c = ctypes.c_int32(clean_run)
    s = lib().orc_scaler_next(ctypes.byref(cfg), int(found_inf), max_abs, scale, ctypes.byref(c))
    return s, c.value


def step(state, grads, scale, lr, momentum, weight_decay, clip=0.0, cfg=None, flags=0,
         eps=1e-10):
    """One whole step; ``state`` is updated in place.  Returns the result dict."""
    cfg = cfg if cfg is not None else scaler_cfg()
    grads = [_c(g, np.uint16) for g in grads]
    n = len(grads)
    assert n == len(state.momentum)
    sizes = np.array([g.size for g in grads], dtype=np.int64)
    for g, v in zip(grads, state.momentum):
        assert g.size == v.size
    clean = ctypes.c_int32(state.clean_run)
    r = _Result()
    master = _ptr_array(state.master) if not (flags & NO_MASTER) else None
    lib().orc_step(_ptr_array(grads), master, _ptr_array(state.momentum),
                   _ptr_array(state.w16), _ptr(sizes), n, scale, lr, momentum,
                   weight_decay, clip, eps, ctypes.byref(cfg), ctypes.byref(clean), flags,
                   ctypes.byref(r))
    state.clean_run = clean.value
    state.scale_history.append(r.new_scale)
    return r.as_dict()
