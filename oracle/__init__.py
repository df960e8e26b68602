"""Oracle for the CQS attention path: test infrastructure only.

Only the test suite, the package's smoke check and the benchmark's
CPU-baseline / reference legs import this package.  The product library
never does, and this package imports nothing from the product.

  * ``attention_rows``  - fp64 exact softmax attention (C, OpenMP) for chosen
    query rows, from ``oracle_attention.c``.
  * ``attention_probs`` - the full weight matrix for tiny problems.
  * ``attention_backward_dq`` / ``attention_backward_dkdv`` - fp64 gradients
    of the same definition for chosen query / key rows.
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
        for name in ("oracle_attention_backward_dq", "oracle_attention_backward_dkdv"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
        lib.oracle_attention_backward_dq.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_attention_backward_dkdv.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
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


def _four(q, k, v, dout):
    qa, tq = _as_stored(q)
    ka, tk = _as_stored(k)
    va, tv = _as_stored(v)
    da, td = _as_stored(dout)
    if not (tq == tk == tv == td):
        raise TypeError("q, k, v, dout must share a dtype")
    N, H, d = qa.shape
    for x in (ka, va, da):
        if x.shape != (N, H, d):
            raise ValueError("q, k, v, dout must all be [N, H, d]")
    return qa, ka, va, da, tq, N, H, d


def attention_backward_dq(q, k, v, dout, rows=None, causal=False, scale=None):
    """fp64 dq for query rows ``rows`` (default all), every head, given the
    output gradient ``dout``.  Returns (dq [R, H, d], lse [R, H], D [R, H])
    with D_i = <dout_i, out_i>."""
    lib = _load()
    qa, ka, va, da, t, N, H, d = _four(q, k, v, dout)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    rows = np.arange(N, dtype=np.int64) if rows is None else rows
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dq = np.empty((rows.size, H, d), dtype=np.float64)
    lse = np.empty((rows.size, H), dtype=np.float64)
    D = np.empty((rows.size, H), dtype=np.float64)
    rc = lib.oracle_attention_backward_dq(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data,
                                          t, N, H, d, int(bool(causal)), float(scale),
                                          rows.ctypes.data, rows.size, dq.ctypes.data,
                                          lse.ctypes.data, D.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attention_backward_dq rejected its arguments")
    return dq, lse, D


def attention_backward_dkdv(q, k, v, dout, keys=None, causal=False, scale=None):
    """fp64 dk, dv for key rows ``keys`` (default all), every head.
    Returns (dk [K, H, d], dv [K, H, d]).  Costs O(N^2 H d)."""
    lib = _load()
    qa, ka, va, da, t, N, H, d = _four(q, k, v, dout)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    keys = np.arange(N, dtype=np.int64) if keys is None else keys
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
    dk = np.empty((keys.size, H, d), dtype=np.float64)
    dv = np.empty((keys.size, H, d), dtype=np.float64)
    rc = lib.oracle_attention_backward_dkdv(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data,
                                            t, N, H, d, int(bool(causal)), float(scale),
                                            keys.ctypes.data, keys.size, dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attention_backward_dkdv rejected its arguments")
    return dk, dv
