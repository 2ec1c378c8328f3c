"""Python binding of the InfLLM block-memory sparse attention layer (libinfllm.so, sm_100a).

Argument marshalling only: every step of the layer runs in the CUDA kernels behind the C ABI
declared in include/infllm.h.  There is no CPU fallback: if the shared library is missing or
cannot be loaded, importing the binding's entry points raises.

    layer = InfLLMLayer(n_q_heads=32, n_kv_heads=8, head_dim=128, n_sink=128, window=4096,
                        unit_size=128, n_reps=4, top_k=16, max_chunk=512, max_tokens=131072,
                        rope_base=1e6, dtype="bf16")
    layer.append_chunk(q, k, v)      # torch CUDA tensors [n, H, d]
    out = layer.attend_chunk(q)      # [n, Hq, d]
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["InfLLMLayer", "InfLLMError", "load_library", "library_path", "Config", "Stats", "STATUS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libinfllm.so")

STATUS = {0: "OK", 1: "EINVAL", 2: "ECAPACITY", 3: "ESTATE", 4: "ECUDA", 5: "EDEVICE"}
DTYPES = {"f32": 0, "bf16": 1}
SCORE_MODES = {"reps": 0, "repsum": 1, "meankey": 2}


class InfLLMError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")


class Config(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("n_sink", ctypes.c_int32), ("window", ctypes.c_int32), ("unit_size", ctypes.c_int32),
                ("n_reps", ctypes.c_int32), ("top_k", ctypes.c_int32), ("max_chunk", ctypes.c_int32),
                ("max_tokens", ctypes.c_int64), ("rope_base", ctypes.c_double), ("dtype", ctypes.c_int32),
                ("score_mode", ctypes.c_int32)]


class Stats(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int64), ("units_with_reps", ctypes.c_int64), ("n_mem", ctypes.c_int32),
                ("n_selected", ctypes.c_int32), ("window_base", ctypes.c_int64), ("active_tokens", ctypes.c_int64),
                ("kernel_launches", ctypes.c_int64), ("attend_path", ctypes.c_int32), ("score_mode", ctypes.c_int32),
                ("ms_append", ctypes.c_double), ("ms_reps", ctypes.c_double), ("ms_prep", ctypes.c_double),
                ("ms_select", ctypes.c_double), ("ms_attend", ctypes.c_double), ("ms_decode", ctypes.c_double),
                ("n_append", ctypes.c_int64), ("n_reps", ctypes.c_int64), ("n_prep", ctypes.c_int64),
                ("n_select", ctypes.c_int64), ("n_attend", ctypes.c_int64), ("n_decode", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


# every entry point of include/infllm.h: name -> (restype, argtypes)
_P = ctypes.c_void_p
SIGNATURES = {
    "infllm_create": (ctypes.c_int, [ctypes.POINTER(Config), _P, ctypes.POINTER(_P)]),
    "infllm_destroy": (ctypes.c_int, [_P]),
    "infllm_reset": (ctypes.c_int, [_P]),
    "infllm_append_chunk": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int32]),
    "infllm_attend_chunk": (ctypes.c_int, [_P, _P, ctypes.c_int32, _P]),
    "infllm_decode_step": (ctypes.c_int, [_P, _P, _P, _P, _P]),
    "infllm_prefill": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int64, ctypes.c_int32, _P]),
    "infllm_set_launch_chaining": (ctypes.c_int, [_P, ctypes.c_int32]),
    "infllm_set_prefill_lookup": (ctypes.c_int, [_P, ctypes.c_int32]),
    "infllm_get_selection": (ctypes.c_int, [_P, _P]),
    "infllm_get_unit_scores": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]),
    "infllm_get_reps": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P]),
    "infllm_get_stats": (ctypes.c_int, [_P, ctypes.POINTER(Stats)]),
    "infllm_set_profiling": (ctypes.c_int, [_P, ctypes.c_int32]),
    "infllm_set_score_mode": (ctypes.c_int, [_P, ctypes.c_int32]),
    "infllm_select_units_noalloc": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                                    ctypes.c_int32, ctypes.c_int32, _P, _P, _P]),
    "infllm_last_error": (ctypes.c_char_p, [_P]),
    "infllm_version": (ctypes.c_char_p, []),
}

_lib = None


def load_library(path: str | None = None):
    """Load libinfllm.so (built in-tree by block_memory_sparse_b200/build.py).  Raises if absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or library_path
    if not os.path.exists(p):
        raise ImportError(f"libinfllm.so not found at {p}: build it with `python -m block_memory_sparse_b200.build` "
                          "(there is no CPU fallback)")
    L = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = L
    return L


def _torch():
    import torch
    return torch


def _dev_ptr(x, dtype, shape, what):
    torch = _torch()
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError(f"{what}: expected a CUDA tensor")
    if x.dtype != dtype or not x.is_contiguous() or tuple(x.shape) != tuple(shape):
        raise ValueError(f"{what}: expected contiguous {dtype} {tuple(shape)}, got {x.dtype} {tuple(x.shape)}")
    return ctypes.c_void_p(x.data_ptr())


class InfLLMLayer:
    """One InfLLM attention layer's context memory on the current CUDA device."""

    def __init__(self, *, n_q_heads, n_kv_heads, head_dim, n_sink, window, unit_size, n_reps, top_k, max_chunk,
                 max_tokens, rope_base, dtype="bf16", score_mode="reps", stream=None):
        torch = _torch()
        self.L = load_library()
        self.cfg = Config(n_q_heads, n_kv_heads, head_dim, n_sink, window, unit_size, n_reps, top_k, max_chunk,
                          max_tokens, float(rope_base), DTYPES[dtype], SCORE_MODES[score_mode])
        self.dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        if stream is None:
            stream = torch.cuda.current_stream()
        self.stream = stream
        h = _P()
        st = self.L.infllm_create(ctypes.byref(self.cfg), _P(stream.cuda_stream), ctypes.byref(h))
        if st != 0:
            raise InfLLMError(st, "infllm_create", "invalid configuration or allocation failure")
        self.h = h
        self._n_pending = None

    @classmethod
    def from_workload(cls, w, max_tokens=None, max_chunk=None, score_mode="reps", stream=None):
        cfg = w.as_config()
        return cls(**cfg, max_chunk=max_chunk or max(w.chunk, w.build_chunk, 1),
                   max_tokens=max_tokens or w.total_tokens, score_mode=score_mode, stream=stream)

    def _check(self, st, where):
        if st != 0:
            raise InfLLMError(st, where, self.L.infllm_last_error(self.h).decode())

    @property
    def Hq(self):
        return self.cfg.n_q_heads

    @property
    def Hkv(self):
        return self.cfg.n_kv_heads

    @property
    def d(self):
        return self.cfg.head_dim

    def append_chunk(self, q, k, v):
        n = q.shape[0]
        qp = _dev_ptr(q, self.dtype, (n, self.Hq, self.d), "q")
        kp = _dev_ptr(k, self.dtype, (n, self.Hkv, self.d), "k")
        vp = _dev_ptr(v, self.dtype, (n, self.Hkv, self.d), "v")
        self._check(self.L.infllm_append_chunk(self.h, qp, kp, vp, n), "infllm_append_chunk")

    def attend_chunk(self, q, out=None):
        torch = _torch()
        n = q.shape[0]
        qp = _dev_ptr(q, self.dtype, (n, self.Hq, self.d), "q")
        if out is None:
            out = torch.empty((n, self.Hq, self.d), dtype=self.dtype, device=q.device)
        op = _dev_ptr(out, self.dtype, (n, self.Hq, self.d), "out")
        self._check(self.L.infllm_attend_chunk(self.h, qp, n, op), "infllm_attend_chunk")
        return out

    def prefill(self, q, k, v, chunk, out=None):
        """Whole prompt in chunks of `chunk` tokens (append + attend per chunk, one C call)."""
        torch = _torch()
        n = q.shape[0]
        qp = _dev_ptr(q, self.dtype, (n, self.Hq, self.d), "q")
        kp = _dev_ptr(k, self.dtype, (n, self.Hkv, self.d), "k")
        vp = _dev_ptr(v, self.dtype, (n, self.Hkv, self.d), "v")
        if out is None:
            out = torch.empty((n, self.Hq, self.d), dtype=self.dtype, device=q.device)
        op = _dev_ptr(out, self.dtype, (n, self.Hq, self.d), "out")
        self._check(self.L.infllm_prefill(self.h, qp, kp, vp, n, int(chunk), op), "infllm_prefill")
        return out

    def set_prefill_lookup(self, on: bool):
        """off: chunks attend to sinks + window only (representatives still built); decode looks up."""
        self._check(self.L.infllm_set_prefill_lookup(self.h, 1 if on else 0), "infllm_set_prefill_lookup")

    def set_launch_chaining(self, on: bool):
        self._check(self.L.infllm_set_launch_chaining(self.h, 1 if on else 0), "infllm_set_launch_chaining")

    def decode_step(self, q, k, v, out=None):
        torch = _torch()
        qp = _dev_ptr(q, self.dtype, (1, self.Hq, self.d), "q")
        kp = _dev_ptr(k, self.dtype, (1, self.Hkv, self.d), "k")
        vp = _dev_ptr(v, self.dtype, (1, self.Hkv, self.d), "v")
        if out is None:
            out = torch.empty((1, self.Hq, self.d), dtype=self.dtype, device=q.device)
        op = _dev_ptr(out, self.dtype, (1, self.Hq, self.d), "out")
        self._check(self.L.infllm_decode_step(self.h, qp, kp, vp, op), "infllm_decode_step")
        return out

    def selection(self):
        import numpy as np
        buf = np.full((self.Hkv, max(1, self.cfg.top_k)), -1, dtype=np.int32)
        self._check(self.L.infllm_get_selection(self.h, buf.ctypes.data), "infllm_get_selection")
        return buf[:, :self.cfg.top_k]

    def unit_scores(self):
        import numpy as np
        n = ctypes.c_int32(0)
        self._check(self.L.infllm_get_unit_scores(self.h, None, 0, ctypes.byref(n)), "infllm_get_unit_scores")
        buf = np.zeros((self.Hkv, n.value), dtype=np.float32)
        self._check(self.L.infllm_get_unit_scores(self.h, buf.ctypes.data, n.value, ctypes.byref(n)),
                    "infllm_get_unit_scores")
        return buf

    def reps(self, unit_begin, n_units):
        import numpy as np
        buf = np.zeros((self.Hkv, n_units, self.cfg.n_reps), dtype=np.int32)
        self._check(self.L.infllm_get_reps(self.h, unit_begin, n_units, buf.ctypes.data), "infllm_get_reps")
        return buf

    def stats(self) -> dict:
        s = Stats()
        self._check(self.L.infllm_get_stats(self.h, ctypes.byref(s)), "infllm_get_stats")
        return s.as_dict()

    PROFILE = {"all": 1, "append": 2, "reps": 4, "prep": 8, "select": 16, "attend": 32, "decode": 64}

    def set_profiling(self, on):
        """on: bool (all kernel classes / off) or an iterable of class names (see PROFILE)."""
        if isinstance(on, bool) or on is None:
            mask = 1 if on else 0
        else:
            mask = 0
            for name in on:
                mask |= self.PROFILE[name]
        self._check(self.L.infllm_set_profiling(self.h, mask), "infllm_set_profiling")

    def set_score_mode(self, mode: str):
        self._check(self.L.infllm_set_score_mode(self.h, SCORE_MODES[mode]), "infllm_set_score_mode")

    def reset(self):
        self._check(self.L.infllm_reset(self.h), "infllm_reset")

    def close(self):
        if getattr(self, "h", None):
            self.L.infllm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
