"""Oracle for the CQS attention path: test infrastructure only.

Only the test suite, the package's smoke check and the benchmark's
CPU-baseline / reference legs import this package.  The product library
never does, and this package imports nothing from the product.

  * ``attention_rows``  - fp64 exact softmax attention (C, OpenMP) for chosen
    query rows, from ``oracle_attention.c``.
  * ``attention_probs`` - the full weight matrix for tiny problems.
  * ``cqs_ref``         - plain-Python CQS Divide reference (difference sets,
    subsequences, masks, recursion, decomposed fp64 simulation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle_attention.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FP32 = 0
BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc + OpenMP (no GPU needed)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_attention_probs.restype = ctypes.c_int
        lib.oracle_attention_probs.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _as_stored(x):
    """Return (contiguous numpy array of the stored bits, dtype tag).

    Accepts numpy float32 arrays, or torch CPU tensors of float32/bfloat16
    (bf16 is passed as its raw 16-bit patterns, widened exactly in C)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), FP32
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, FP32
    raise TypeError(f"unsupported dtype {x.dtype}")


def num_threads() -> int:
    return _load().oracle_num_threads()


def attention_rows(q, k, v, rows=None, causal=False, scale=None):
    """fp64 attention for query rows ``rows`` (default: all), every head.

    q, k, v: [N, H, d] fp32 or bf16.  Returns (out [R, H, d] float64,
    lse [R, H] float64, natural log)."""
    lib = _load()
    qa, tq = _as_stored(q)
    ka, tk = _as_stored(k)
    va, tv = _as_stored(v)
    if not (tq == tk == tv):
        raise TypeError("q, k, v must share a dtype")
    N, H, d = qa.shape
    if ka.shape != (N, H, d) or va.shape != (N, H, d):
        raise ValueError("q, k, v must all be [N, H, d]")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((rows.size, H, d), dtype=np.float64)
    lse = np.empty((rows.size, H), dtype=np.float64)
    rc = lib.oracle_attention_rows(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, tq,
                                   N, H, d, int(bool(causal)), float(scale),
                                   rows.ctypes.data, rows.size,
                                   out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attention_rows rejected its arguments")
    return out, lse


def attention_probs(q, k, causal=False, scale=None):
    """Softmax weights [H, N, N] (fp64) for tiny problems."""
    lib = _load()
    qa, tq = _as_stored(q)
    ka, tk = _as_stored(k)
    if tq != tk:
        raise TypeError("q, k must share a dtype")
    N, H, d = qa.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    probs = np.empty((H, N, N), dtype=np.float64)
    rc = lib.oracle_attention_probs(qa.ctypes.data, ka.ctypes.data, tq, N, H, d,
                                    int(bool(causal)), float(scale), probs.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attention_probs rejected its arguments")
    return probs
