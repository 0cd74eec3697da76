"""Masked softmax attention in fp64 (test infrastructure; see package doc).

Follows the attention equation of "DiT as Real-Time Rerenderer" (papernotes
note, Method > Key Designs 2):

    Attn(Q, K, V) = softmax(Q K^T / sqrt(d) + M) V,
    M_ij = 0 if floor(j/k) <= floor(i/k) else -inf,

d the head dimension, k the spatial tokens per latent frame, i / j logical
token positions.  The arithmetic runs in the C library ``rtr_oracle.c``
(plain per-row loops in double precision); this module only marshals arrays.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None


def library_path() -> str:
    return _build.LIB


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.rtr_oracle_visible.restype = ctypes.c_int
        lib.rtr_oracle_visible.argtypes = [ctypes.c_int64] * 3
        p = ctypes.c_void_p
        lib.rtr_oracle_attention.restype = ctypes.c_int
        lib.rtr_oracle_attention.argtypes = [
            p, p, ctypes.c_int64, p, p, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_double, p,
            ctypes.c_int]
        lib.rtr_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses by default."""
    return int(_load().rtr_oracle_max_threads())


def visible(i: int, j: int, k: int) -> bool:
    """The mask M: logical query position i sees logical key position j."""
    return bool(_load().rtr_oracle_visible(int(i), int(j), int(k)))


def decode(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of stored input bits.

    ``dtype`` "bf16": ``raw`` holds bfloat16 bit patterns as uint16; a
    bfloat16 is the upper half of an IEEE binary32, so shifting the pattern
    into the high 16 bits gives the same number as a float32.  "f32": float32.
    """
    if dtype == "bf16":
        raw = np.ascontiguousarray(raw, dtype=np.uint16)
        return (raw.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "f32":
        return np.ascontiguousarray(raw, dtype=np.float32).astype(np.float64)
    raise ValueError("dtype must be 'bf16' or 'f32'")


def attention(q, q_pos, k, v, k_per_frame, causal=True, scale=None,
              nthreads=0) -> np.ndarray:
    """softmax(q k^T * scale + M) v for the given query rows, in fp64.

    q: [nq, H, d]; q_pos: [nq] logical positions of the query rows;
    k, v: [nk, H, d] with key j at logical position j.  ``causal=False``
    drops M (every key visible).  ``scale`` defaults to 1/sqrt(d).
    Returns [nq, H, d] float64.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    q_pos = np.ascontiguousarray(q_pos, dtype=np.int64)
    nq, H, d = q.shape
    nk = k.shape[0]
    assert k.shape == (nk, H, d) and v.shape == (nk, H, d)
    assert q_pos.shape == (nq,)
    if nq and q_pos.min() < 0:
        raise ValueError("positions must be non-negative")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((nq, H, d), dtype=np.float64)
    if nq == 0:
        return out
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    failed = _load().rtr_oracle_attention(ptr(q), ptr(q_pos), nq, ptr(k), ptr(v), nk,
                                          H, d, int(k_per_frame), 1 if causal else 0,
                                          float(scale), ptr(out), int(nthreads))
    if failed:
        raise MemoryError("oracle attention: row buffers could not be allocated")
    return out


def prefill(q, k, v, k_per_frame, rows=None, scale=None, nthreads=0):
    """Block-causal attention over one whole sequence [n, H, d].

    Token i of the sequence sits at logical position i, so its frame is
    floor(i/k).  ``rows`` selects query rows (default: all); the result has
    one row per selected query.
    """
    q = np.asarray(q)
    n = q.shape[0]
    rows = np.arange(n, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    return attention(q[rows], rows, k, v, k_per_frame, True, scale, nthreads)
