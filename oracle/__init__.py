"""ctypes front-end for the fp64 CPU oracle in ``hsa_oracle.c``.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The CUDA library never imports it.

Every array is passed as a C-contiguous numpy array; float inputs are float64
(the exact values the GPU sees, e.g. bf16 widened to fp64), the pooled chunk
keys are float32 (their stored precision is part of the definition).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libhsa_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        i, i64, p = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
        L.or_pool.argtypes = [i, i, i, i, i, p, p]
        L.or_select.argtypes = [i, i, i, i, i, i, p, p, p, i64, p, p, p, p]
        L.or_fwd.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p, i64, p, p, p, p]
        L.or_attend.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p, i64, p, p]
        L.or_decode.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p, p, p, p]
        L.or_bwd.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p, p, p, p, p, p, p]
        for f in (L.or_pool, L.or_select, L.or_fwd, L.or_attend, L.or_decode, L.or_bwd):
            f.restype = ctypes.c_int
        L.or_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"oracle {name} failed with code {rc}")


def num_threads() -> int:
    return int(lib().or_num_threads())


def pool(k: np.ndarray, S: int) -> np.ndarray:
    """k [B, h_kv, L, d] -> kbar [B, h_kv, L//S, d] float32."""
    k = _f64(k)
    B, h_kv, L, d = k.shape
    kbar = np.zeros((B, h_kv, L // S, d), dtype=np.float32)
    _check(lib().or_pool(B, h_kv, L, d, S, _ptr(k), _ptr(kbar)), "pool")
    return kbar


def select(q_slc: np.ndarray, kbar: np.ndarray, S: int, K: int, rows=None):
    """q_slc [B, L, h_kv, d], kbar [B, h_kv, n_c, d] float32.

    Returns idx [n, h_kv, K] int32, w, s [n, h_kv, K] float64 and
    gap [n, h_kv] (score gap between the K-th and (K+1)-th best chunk; +inf
    when no more than K chunks are eligible).  ``rows`` are flat b*L+t indices
    (default: all rows in order, n = B*L).
    """
    q_slc = _f64(q_slc)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, L, h_kv, d = q_slc.shape
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = B * L if rows_a is None else rows_a.shape[0]
    idx = np.zeros((n, h_kv, K), dtype=np.int32)
    w = np.zeros((n, h_kv, K))
    s = np.zeros((n, h_kv, K))
    gap = np.zeros((n, h_kv))
    _check(lib().or_select(B, L, h_kv, d, S, K, _ptr(q_slc), _ptr(kbar), _ptr(rows_a), n,
                           _ptr(idx), _ptr(w), _ptr(s), _ptr(gap)), "select")
    return idx, w, s, gap


def fwd(q, k, v, q_slc, kbar, S: int, K: int, rows=None):
    """Forward pass.  Returns o [n, h_q, d], lse [n, h_q, K], idx, w [n, h_kv, K]."""
    q, k, v, q_slc = _f64(q), _f64(k), _f64(v), _f64(q_slc)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, L, h_q, d = q.shape
    h_kv = k.shape[1]
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = B * L if rows_a is None else rows_a.shape[0]
    o = np.zeros((n, h_q, d))
    lse = np.zeros((n, h_q, K))
    idx = np.zeros((n, h_kv, K), dtype=np.int32)
    w = np.zeros((n, h_kv, K))
    _check(lib().or_fwd(B, L, h_q, h_kv, d, S, K, _ptr(q), _ptr(k), _ptr(v), _ptr(q_slc),
                        _ptr(kbar), _ptr(rows_a), n, _ptr(o), _ptr(lse), _ptr(idx), _ptr(w)), "fwd")
    return o, lse, idx, w


def attend(q, k, v, idx, w, S: int, rows=None):
    """Attention and fusion for a given selection idx, w [n, h_kv, K] (one
    entry per listed row).  Returns o [n, h_q, d], lse [n, h_q, K]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, h_q, d = q.shape
    h_kv, K = k.shape[1], idx.shape[-1]
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = B * L if rows_a is None else rows_a.shape[0]
    idx = np.ascontiguousarray(np.asarray(idx).reshape(n, h_kv, K), dtype=np.int32)
    w = _f64(np.asarray(w).reshape(n, h_kv, K))
    o = np.zeros((n, h_q, d))
    lse = np.zeros((n, h_q, K))
    _check(lib().or_attend(B, L, h_q, h_kv, d, S, K, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(w),
                           _ptr(rows_a), n, _ptr(o), _ptr(lse)), "attend")
    return o, lse


def decode(q, q_slc, k_cache, v_cache, kbar, S: int, K: int):
    """One decode step.  q [B, h_q, d], q_slc [B, h_kv, d], caches [B, h_kv, P, d].

    Returns o [B, h_q, d], idx, w [B, h_kv, K] and gap [B, h_kv].
    """
    q, q_slc, k_cache, v_cache = _f64(q), _f64(q_slc), _f64(k_cache), _f64(v_cache)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, h_q, d = q.shape
    h_kv, P = k_cache.shape[1], k_cache.shape[2]
    o = np.zeros((B, h_q, d))
    idx = np.zeros((B, h_kv, K), dtype=np.int32)
    w = np.zeros((B, h_kv, K))
    gap = np.zeros((B, h_kv))
    _check(lib().or_decode(B, P, h_q, h_kv, d, S, K, _ptr(q), _ptr(q_slc), _ptr(k_cache),
                           _ptr(v_cache), _ptr(kbar), _ptr(o), _ptr(idx), _ptr(w), _ptr(gap)),
           "decode")
    return o, idx, w, gap


def bwd(q, k, v, q_slc, kbar, dO, S: int, K: int, tok_mask=None):
    """Backward pass.  Returns dq, dk, dv, dq_slc, dkbar (float64).

    ``tok_mask`` [B, L] (bool) restricts which tokens contribute; gradients of
    the chunks selected only by masked-in tokens are then complete.
    """
    q, k, v, q_slc, dO = _f64(q), _f64(k), _f64(v), _f64(q_slc), _f64(dO)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, L, h_q, d = q.shape
    h_kv = k.shape[1]
    m = None if tok_mask is None else np.ascontiguousarray(tok_mask, dtype=np.uint8)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dq_slc = np.zeros_like(q_slc)
    dkbar = np.zeros((B, h_kv, L // S, d))
    _check(lib().or_bwd(B, L, h_q, h_kv, d, S, K, _ptr(q), _ptr(k), _ptr(v), _ptr(q_slc),
                        _ptr(kbar), _ptr(dO), _ptr(m), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dq_slc),
                        _ptr(dkbar)), "bwd")
    return dq, dk, dv, dq_slc, dkbar
