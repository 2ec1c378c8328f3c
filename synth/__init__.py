"""Seeded synthetic inputs for the InfLLM block-memory attention layer.

This module is shared by the CPU oracle and the CUDA path and holds none of
the attention method's arithmetic: it produces Q/K/V token streams from
(seed, tensor id, token range) with a counter-based generator (``synth.c``),
so any chunk of any workload can be regenerated independently.

Tensors are laid out ``[tokens][heads][head_dim]``; bf16 data is returned as
``uint16`` bit patterns (numpy has no bfloat16), float32 data as ``float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .workloads import ALL, SMALL, WORKLOADS, Workload, chunk_bounds, gen_chunk, needle_info  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "synth.c")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, OpenMP, strict IEEE)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            L.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p,
                                       ctypes.c_int32, ctypes.c_void_p]
            L.synth_normal.restype = None
            L.synth_normal_flat.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_void_p]
            L.synth_normal_flat.restype = None
            L.synth_philox4x32_10.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
            L.synth_philox4x32_10.restype = None
            L.synth_round_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
            L.synth_round_bf16.restype = None
            _lib = L
    return _lib


def normal(seed: int, tensor_id: int, t0: int, n_tok: int, n_head: int, dim: int, *, dtype: str = "f32",
           scale: float = 1.0, bias: np.ndarray | None = None, out: np.ndarray | None = None) -> np.ndarray:
    """Normal deviates for tokens [t0, t0+n_tok) of one tensor, shape [n_tok, n_head, dim].

    ``bias`` (float32 [n_head, dim]) is added in float32 before rounding.
    dtype "f32" returns float32, "bf16" returns uint16 bf16 bit patterns.
    """
    npdt = np.float32 if dtype == "f32" else np.uint16
    if out is None:
        out = np.empty((n_tok, n_head, dim), dtype=npdt)
    assert out.dtype == npdt and out.flags.c_contiguous and out.size == n_tok * n_head * dim
    b = None
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
        assert bias.shape == (n_head, dim)
        b = bias.ctypes.data
    lib().synth_normal(seed, tensor_id, t0, n_tok, n_head, dim, float(scale), b,
                       0 if dtype == "f32" else 1, out.ctypes.data)
    return out


def normal_flat(seed: int, tensor_id: int, e0: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal_flat(seed, tensor_id, e0, n, out.ctypes.data)
    return out


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    o = np.empty(4, dtype=np.uint32)
    lib().synth_philox4x32_10(c.ctypes.data, k.ctypes.data, o.ctypes.data)
    return o


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits (round to nearest even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = np.empty(x.shape, dtype=np.uint16)
    lib().synth_round_bf16(x.ctypes.data, x.size, o.ctypes.data)
    return o


def bf16_to_f64(u: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float64 values."""
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of a generated array (float32 or bf16 bits) to float64."""
    if a.dtype == np.uint16:
        return bf16_to_f64(a)
    return np.asarray(a, dtype=np.float64)
