"""Python binding of libmpt: the loss-scaled FP32-master optimizer step on B200.

Argument marshalling only (ctypes over the C ABI in ``include/mpt.h``): every
step of the path runs in the library's CUDA kernels.  PyTorch supplies the
device workspace and the stream.  There is no CPU fallback: if ``libmpt.so``
cannot be loaded (or built with nvcc), importing the library fails loudly.

    opt = MPT(sizes, Config(growth_interval=4))
    for i, w in enumerate(initial_weights):
        opt.master(i).copy_(w)
    opt.refresh_half()
    opt.set_scaler_state(2.0 ** 16)
    res = opt.step(grads, scale=opt.scale, lr=0.01, momentum=0.9,
                   weight_decay=1e-4, clip=1.0)
"""
import ctypes
import os

from . import build as _build

__all__ = ["MPT", "Config", "MptError", "lib", "grad_pointers", "check_flat_noalloc",
           "MPT_FLAG_CHECKED", "MPT_FLAG_COUNT_STALE", "MPT_FLAG_GRAD_STATS",
           "MPT_SCALER_DYNAMIC", "MPT_SCALER_DIRECT", "MPT_OPT_MOMENTUM", "MPT_OPT_NESTEROV",
           "MPT_OPT_ADAGRAD"]

MPT_FLAG_CHECKED = 0x1
MPT_FLAG_COUNT_STALE = 0x2
MPT_FLAG_GRAD_STATS = 0x4
MPT_SCALER_DYNAMIC = 0
MPT_SCALER_DIRECT = 1
MPT_OPT_MOMENTUM = 0
MPT_OPT_NESTEROV = 1
MPT_OPT_ADAGRAD = 2

MPT_OK = 0
MPT_ERR_INVALID_ARG = -1
MPT_ERR_WORKSPACE = -2
MPT_ERR_CUDA = -3
MPT_ERR_DEVICE_CHECK = -4
MPT_ERR_BROKEN = -5
MPT_ERR_TOO_LARGE = -6
MPT_NOALLOC_MAX_ELEMS = 1 << 30
MPT_PARTIAL_BYTES = 32


class MptError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {lib().mpt_error_string(code).decode()} ({code})")


class Config(ctypes.Structure):
    _fields_ = [("backoff", ctypes.c_float), ("growth", ctypes.c_float),
                ("growth_interval", ctypes.c_int32), ("min_scale", ctypes.c_float),
                ("max_scale", ctypes.c_float), ("flags", ctypes.c_uint32),
                ("check_chunk_elems", ctypes.c_int32), ("scaler_mode", ctypes.c_int32),
                ("direct_margin", ctypes.c_float), ("optimizer", ctypes.c_int32),
                ("eps", ctypes.c_float), ("update_chunk_elems", ctypes.c_int32)]

    def __init__(self, **kw):
        super().__init__()
        lib().mpt_config_init(ctypes.byref(self))
        for k, v in kw.items():
            if k not in dict(self._fields_):
                raise TypeError(f"unknown config field {k}")
            setattr(self, k, v)


class StepResult(ctypes.Structure):
    _fields_ = [("found_inf", ctypes.c_int32), ("clipped", ctypes.c_int32),
                ("new_scale", ctypes.c_float), ("clean_run", ctypes.c_int32),
                ("grad_norm", ctypes.c_double), ("clip_coef", ctypes.c_float),
                ("max_abs_grad", ctypes.c_float), ("n_zero", ctypes.c_uint64),
                ("n_subnormal", ctypes.c_uint64), ("n_nonfinite", ctypes.c_uint64),
                ("n_fp16_stale", ctypes.c_uint64)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class CheckResult(ctypes.Structure):
    """``mpt_check_result``: what mpt_check_flat_noalloc writes to device memory."""
    _fields_ = [("found_inf", ctypes.c_int32), ("clipped", ctypes.c_int32),
                ("grad_norm", ctypes.c_double), ("clip_coef", ctypes.c_float),
                ("reserved", ctypes.c_int32), ("n_nonfinite", ctypes.c_uint64)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_ if k != "reserved"}


class Stats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_uint64), ("skipped", ctypes.c_uint64),
                ("scale", ctypes.c_float), ("clean_run", ctypes.c_int32),
                ("last", StepResult), ("n_fp16_stale_total", ctypes.c_uint64),
                ("timed_steps", ctypes.c_uint64), ("check_ms_total", ctypes.c_double),
                ("update_ms_total", ctypes.c_double)]

    def as_dict(self):
        d = {k: getattr(self, k) for k, _ in self._fields_}
        d["last"] = self.last.as_dict()
        return d


_LIB = None


def lib():
    """Load (building with nvcc if needed) ``libmpt.so``; raises if impossible."""
    global _LIB
    if _LIB is None:
        path = _build.LIB
        if not os.path.exists(path) or os.environ.get("MPT_REBUILD"):
            path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        sig = {
            "mpt_config_init": [ctypes.POINTER(Config)],
            "mpt_workspace_bytes": [vp, i32, ctypes.POINTER(Config), ctypes.POINTER(ctypes.c_size_t)],
            "mpt_create": [vp, i32, ctypes.POINTER(Config), vp, ctypes.c_size_t, ctypes.POINTER(vp)],
            "mpt_tensor_views": [vp, i32, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp)],
            "mpt_refresh_half": [vp, vp],
            "mpt_step": [vp, vp, f32, f32, f32, f32, f32, vp, ctypes.POINTER(StepResult)],
            "mpt_stats": [vp, ctypes.POINTER(Stats)],
            "mpt_get_scaler_state": [vp, ctypes.POINTER(f32), ctypes.POINTER(i32)],
            "mpt_set_scaler_state": [vp, f32, i32],
            "mpt_set_timing": [vp, i32],
            "mpt_destroy": [vp],
            "mpt_check_flat_noalloc": [vp, ctypes.c_int64, f32, f32, vp, vp],
            "mpt_step_async": [vp, vp, f32, f32, f32, f32, vp],
            "mpt_wait": [vp, vp, ctypes.POINTER(StepResult)],
            "mpt_device_scale": [vp, ctypes.POINTER(vp)],
            "mpt_grad_histogram": [vp, ctypes.POINTER(ctypes.c_uint64 * 32)],
            "mpt_shard_len": [ctypes.c_int64, i32, ctypes.POINTER(ctypes.c_int64)],
            "mpt_step_partial": [vp, vp, vp, ctypes.POINTER(vp)],
            "mpt_step_finish": [vp, vp, i32, f32, f32, f32, f32, vp],
            "mpt_debug_fail_next_step": [vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.mpt_error_string.argtypes = [ctypes.c_int]
        L.mpt_error_string.restype = ctypes.c_char_p
        _LIB = L
    return _LIB


def _check(code, what):
    if code != MPT_OK:
        raise MptError(code, what)


def grad_pointers(tensors):
    """Host array of device pointers (build once, reuse across steps)."""
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def check_flat_noalloc(grads, scale, clip, out, stream=None):
    """Queue ``mpt_check_flat_noalloc`` on one contiguous FP16 CUDA tensor;
    ``out`` is a CUDA tensor of at least ``ctypes.sizeof(CheckResult)`` bytes
    that receives the result.  Returns without waiting."""
    if not grads.is_contiguous() or grads.element_size() != 2:
        raise ValueError("grads must be one contiguous 2-byte tensor")
    if out.numel() * out.element_size() < ctypes.sizeof(CheckResult):
        raise ValueError("out is too small for mpt_check_result")
    _check(lib().mpt_check_flat_noalloc(ctypes.c_void_p(grads.data_ptr()), grads.numel(),
                                        scale, clip, ctypes.c_void_p(out.data_ptr()),
                                        _stream_ptr(stream, grads.device)),
           "mpt_check_flat_noalloc")


def shard_len(total, world):
    """Elements per rank of the sharded step (``mpt_shard_len``)."""
    n = ctypes.c_int64()
    _check(lib().mpt_shard_len(int(total), int(world), ctypes.byref(n)), "mpt_shard_len")
    return n.value


def _stream_ptr(stream, device):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


class MPT:
    """One optimizer over a fixed list of tensor sizes (one CUDA device)."""

    def __init__(self, sizes, config=None, device=None):
        import torch
        self.sizes = [int(s) for s in sizes]
        self.n = len(self.sizes)
        self.config = config if config is not None else Config()
        self.device = torch.device(device if device is not None else "cuda", )
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self._sizes_c = (ctypes.c_int64 * self.n)(*self.sizes)
        nbytes = ctypes.c_size_t()
        _check(lib().mpt_workspace_bytes(self._sizes_c, self.n, ctypes.byref(self.config),
                                         ctypes.byref(nbytes)), "mpt_workspace_bytes")
        self.workspace_bytes = nbytes.value
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib().mpt_create(self._sizes_c, self.n, ctypes.byref(self.config),
                                    ctypes.c_void_p(self.workspace.data_ptr()),
                                    self.workspace_bytes, ctypes.byref(h)), "mpt_create")
        self._h = h
        self._views = [self._make_views(i) for i in range(self.n)]
        self._ptr_cache = None

    # -- state views ---------------------------------------------------------
    def _make_views(self, i):
        import torch
        m, v, w = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().mpt_tensor_views(self._h, i, ctypes.byref(m), ctypes.byref(v),
                                      ctypes.byref(w)), "mpt_tensor_views")
        base = self.workspace.data_ptr()
        n = self.sizes[i]
        ws = self.workspace
        return (ws[m.value - base: m.value - base + 4 * n].view(torch.float32),
                ws[v.value - base: v.value - base + 4 * n].view(torch.float32),
                ws[w.value - base: w.value - base + 2 * n].view(torch.float16))

    def master(self, i):
        return self._views[i][0]

    def momentum(self, i):
        return self._views[i][1]

    def w16(self, i):
        return self._views[i][2]

    # -- calls ---------------------------------------------------------------
    def refresh_half(self, stream=None):
        _check(lib().mpt_refresh_half(self._h, _stream_ptr(stream, self.device)),
               "mpt_refresh_half")

    def step(self, grads, scale, lr, momentum, weight_decay, clip=0.0, stream=None):
        """``grads``: list of FP16 (or int16 bit-pattern) CUDA tensors, or an
        array from :func:`grad_pointers`.  Returns the step result as a dict."""
        ptrs = self._ptrs(grads)
        r = StepResult()
        _check(lib().mpt_step(self._h, ptrs, scale, lr, momentum, weight_decay, clip,
                              _stream_ptr(stream, self.device), ctypes.byref(r)), "mpt_step")
        return r.as_dict()

    def _ptrs(self, grads):
        if isinstance(grads, ctypes.Array):
            return grads
        if len(grads) != self.n:
            raise ValueError(f"expected {self.n} gradient tensors, got {len(grads)}")
        for g, n in zip(grads, self.sizes):
            if g.numel() != n or g.element_size() != 2 or g.device != self.device:
                raise ValueError("gradient tensor does not match its size/dtype/device")
            if not g.is_contiguous():
                raise ValueError("gradient tensors must be contiguous")
        return grad_pointers(grads)

    def step_async(self, grads, lr, momentum, weight_decay, clip=0.0, stream=None):
        """Queue one step without waiting; S is the device scale state
        (:meth:`device_scale`).  Call :meth:`wait` for the result."""
        _check(lib().mpt_step_async(self._h, self._ptrs(grads), lr, momentum, weight_decay, clip,
                                    _stream_ptr(stream, self.device)), "mpt_step_async")

    def wait(self, stream=None):
        """Wait for the queued steps; returns the last step's result."""
        r = StepResult()
        _check(lib().mpt_wait(self._h, _stream_ptr(stream, self.device), ctypes.byref(r)),
               "mpt_wait")
        return r.as_dict()

    def device_scale(self):
        """A 1-element float32 CUDA tensor aliasing the device scale state."""
        p = ctypes.c_void_p()
        _check(lib().mpt_device_scale(self._h, ctypes.byref(p)), "mpt_device_scale")
        off = p.value - self.workspace.data_ptr()
        import torch
        return self.workspace[off:off + 4].view(torch.float32)

    def step_partial(self, grads, stream=None):
        """Sharded step, phase 2: queue the check pass; returns a 32-byte
        uint8 CUDA tensor aliasing this rank's record."""
        import torch
        p = ctypes.c_void_p()
        _check(lib().mpt_step_partial(self._h, self._ptrs(grads), _stream_ptr(stream, self.device),
                                      ctypes.byref(p)), "mpt_step_partial")
        off = p.value - self.workspace.data_ptr()
        return self.workspace[off:off + MPT_PARTIAL_BYTES]

    def step_finish(self, partials, world, lr, momentum, weight_decay, clip=0.0, stream=None):
        """Sharded step, phase 4: ``partials`` is a CUDA tensor holding the
        ``world`` records in rank order."""
        _check(lib().mpt_step_finish(self._h, ctypes.c_void_p(partials.data_ptr()), world, lr,
                                     momentum, weight_decay, clip,
                                     _stream_ptr(stream, self.device)), "mpt_step_finish")

    def grad_histogram(self):
        """Gradients of the last step per binary16 exponent field (32 bins)."""
        h = (ctypes.c_uint64 * 32)()
        _check(lib().mpt_grad_histogram(self._h, ctypes.byref(h)), "mpt_grad_histogram")
        return list(h)

    def stats(self):
        s = Stats()
        _check(lib().mpt_stats(self._h, ctypes.byref(s)), "mpt_stats")
        return s.as_dict()

    @property
    def scale(self):
        return self.scaler_state()[0]

    def scaler_state(self):
        s, c = ctypes.c_float(), ctypes.c_int32()
        _check(lib().mpt_get_scaler_state(self._h, ctypes.byref(s), ctypes.byref(c)),
               "mpt_get_scaler_state")
        return s.value, c.value

    def set_scaler_state(self, scale, clean_run=0):
        _check(lib().mpt_set_scaler_state(self._h, scale, clean_run), "mpt_set_scaler_state")

    def set_timing(self, every=1):
        """Time the two kernels of every ``every``-th following step (0 or
        False: off; True or 1: every step)."""
        _check(lib().mpt_set_timing(self._h, int(every)), "mpt_set_timing")

    def debug_fail_next_step(self):
        """Test hook: the next step fails like a failed kernel launch and the
        handle becomes unusable (``mpt_debug_fail_next_step``)."""
        _check(lib().mpt_debug_fail_next_step(self._h), "mpt_debug_fail_next_step")

    def close(self):
        if getattr(self, "_h", None):
            lib().mpt_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
