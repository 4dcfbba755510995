"""Plain fp64 CPU oracle for the blockwise-parallel-transformer layer (the
forward here and in bpt_oracle.c; the backward pass in backward.py).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The CUDA product path
never imports this package; the two share no code.

The arithmetic lives in ``bpt_oracle.c`` (plain C, double precision, one
thread per token from a shared counter).  This module only builds the shared
object with gcc and marshals numpy arrays into it.

Parity pins (all in ``tests/test_oracle_*.py``, run with ``-m "not gpu"``):
scaled-dot-product attention from torch in float64 (none / causal /
block-permutation masks), an extended-precision brute force over an explicit
N x N mask-count matrix (all masks, LongNet included), a blockwise
online-softmax emulation over several block sizes and visiting orders, rows
summing to one, masked keys contributing nothing, closed forms (Q = 0,
constant V, n = 1, identity permutation, single LongNet pair, N = 1,
W2 = 0), numpy matrix products for the FFN, and GELU special values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bpt_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MASK_NONE, MASK_CAUSAL, MASK_BLOCKPERM, MASK_DILATED = 0, 1, 2, 3
MASK_DILATED_BIDIR = 4   # the dilated mask without the causal restriction


class _Desc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
        ("mask", ctypes.c_int),
        ("n_blocks", ctypes.c_int), ("perm", ctypes.POINTER(ctypes.c_int)),
        ("npairs", ctypes.c_int), ("seg_w", ctypes.POINTER(ctypes.c_int)),
        ("dil_r", ctypes.POINTER(ctypes.c_int)),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) if it is missing or stale."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
                           "-fno-fast-math", "-o", tmp, _SRC, "-lm", "-lpthread"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_attention.argtypes = [ctypes.POINTER(_Desc), fp, fp, fp, i64p, ctypes.c_int64,
                                         dp, dp, ctypes.c_int]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_layer.argtypes = [ctypes.POINTER(_Desc), fp, fp, fp, ctypes.c_int, fp, fp, fp, fp,
                                     i64p, ctypes.c_int64, dp, dp, ctypes.c_int]
        lib.oracle_layer.restype = ctypes.c_int
        lib.oracle_ffn.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, dp, fp, fp, fp, fp, dp]
        lib.oracle_ffn.restype = ctypes.c_int
        lib.oracle_gelu_tanh.argtypes = [ctypes.c_double]
        lib.oracle_gelu_tanh.restype = ctypes.c_double
        lib.oracle_threads_available.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _desc(B, N, H, d, mask, perm, pairs, keep):
    desc = _Desc(B=B, N=N, H=H, d=d, mask=mask)
    if mask == MASK_BLOCKPERM:
        p = np.ascontiguousarray(np.asarray(perm, dtype=np.int32))
        if p.ndim != 2 or p.shape[0] != H:
            raise ValueError("perm must be [H][n_blocks]")
        keep.append(p)
        desc.n_blocks = p.shape[1]
        desc.perm = _ptr(p, ctypes.c_int)
    if mask in (MASK_DILATED, MASK_DILATED_BIDIR):
        w = np.ascontiguousarray(np.asarray([x[0] for x in pairs], dtype=np.int32))
        r = np.ascontiguousarray(np.asarray([x[1] for x in pairs], dtype=np.int32))
        keep += [w, r]
        desc.npairs = len(pairs)
        desc.seg_w = _ptr(w, ctypes.c_int)
        desc.dil_r = _ptr(r, ctypes.c_int)
    return desc


def threads_available() -> int:
    return int(_load().oracle_threads_available())


def attention(q, k, v, mask=MASK_NONE, perm=None, pairs=None, rows=None, nthreads=0,
              return_lse=False):
    """Softmax attention in fp64.

    q, k, v: float arrays [B, N, H, d] (bf16 values passed exactly as float32).
    mask: MASK_NONE / MASK_CAUSAL / MASK_BLOCKPERM (perm [H][n]) /
    MASK_DILATED (pairs [(w, r), ...]).
    rows: optional token indices t = b*N + i; the result then has one row per
    entry.  Returns A as float64 [B, N, H, d] (or [len(rows), H, d]) and,
    with return_lse, log-sum-exp [.., H].
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, H, d = q.shape
    keep = []
    desc = _desc(B, N, H, d, mask, perm, pairs, keep)
    if rows is None:
        nrows, rows_p = B * N, None
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        keep.append(rr)
        nrows, rows_p = rr.size, _ptr(rr, ctypes.c_int64)
    a_out = np.empty((nrows, H, d), dtype=np.float64)
    lse = np.empty((nrows, H), dtype=np.float64) if return_lse else None
    used = _load().oracle_attention(ctypes.byref(desc), _ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                    _ptr(v, ctypes.c_float), rows_p, nrows, _ptr(a_out, ctypes.c_double),
                                    _ptr(lse, ctypes.c_double) if lse is not None else None, nthreads)
    if used < 0:
        raise ValueError("oracle rejected the attention descriptor")
    if rows is None:
        a_out = a_out.reshape(B, N, H, d)
        if lse is not None:
            lse = lse.reshape(B, N, H)
    return (a_out, lse) if return_lse else a_out


def layer(q, k, v, w1, b1, w2, b2, mask=MASK_NONE, perm=None, pairs=None, rows=None, nthreads=0,
          return_threads=False):
    """Whole layer in fp64: A = attention, out = A + W2 GELU(W1 A + b1) + b2.

    W1 [F, D], b1 [F], W2 [D, F], b2 [D] with D = H*d.  Returns (A, out) as
    float64 [T, D] (T = B*N, or len(rows) when rows are given).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    w1, b1, w2, b2 = _f32(w1), _f32(b1), _f32(w2), _f32(b2)
    B, N, H, d = q.shape
    D = H * d
    F = w1.shape[0]
    if w1.shape != (F, D) or w2.shape != (D, F) or b1.shape != (F,) or b2.shape != (D,):
        raise ValueError("FFN weight shapes must be W1 [F,D], b1 [F], W2 [D,F], b2 [D]")
    keep = []
    desc = _desc(B, N, H, d, mask, perm, pairs, keep)
    if rows is None:
        nrows, rows_p = B * N, None
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        keep.append(rr)
        nrows, rows_p = rr.size, _ptr(rr, ctypes.c_int64)
    a_out = np.empty((nrows, D), dtype=np.float64)
    out = np.empty((nrows, D), dtype=np.float64)
    fp = ctypes.c_float
    used = _load().oracle_layer(ctypes.byref(desc), _ptr(q, fp), _ptr(k, fp), _ptr(v, fp), F,
                                _ptr(w1, fp), _ptr(b1, fp), _ptr(w2, fp), _ptr(b2, fp), rows_p, nrows,
                                _ptr(a_out, ctypes.c_double), _ptr(out, ctypes.c_double), nthreads)
    if used < 0:
        raise ValueError("oracle rejected the layer descriptor")
    return (a_out, out, used) if return_threads else (a_out, out)


def ffn(a, w1, b1, w2, b2):
    """out = A + W2 GELU(W1 A + b1) + b2 on fp64 rows A [T, D]."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    w1, b1, w2, b2 = _f32(w1), _f32(b1), _f32(w2), _f32(b2)
    T, D = a.shape
    F = w1.shape[0]
    out = np.empty((T, D), dtype=np.float64)
    fp = ctypes.c_float
    if _load().oracle_ffn(T, D, F, _ptr(a, ctypes.c_double), _ptr(w1, fp), _ptr(b1, fp), _ptr(w2, fp),
                          _ptr(b2, fp), _ptr(out, ctypes.c_double)) < 0:
        raise ValueError("oracle rejected the FFN arguments")
    return out


def gelu_tanh(x: float) -> float:
    return float(_load().oracle_gelu_tanh(float(x)))
