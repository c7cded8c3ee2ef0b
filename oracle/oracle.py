"""ctypes front end of the HiLS CPU oracle.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
use this module.  It builds ``libhils_oracle.so`` from ``hils_oracle.c`` with
gcc and exposes the oracle's entry points on numpy arrays.  It imports
nothing from the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "hils_oracle.c")
LIB = os.path.join(_HERE, "libhils_oracle.so")

_lib = None


class OCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "chunk_size", "top_k", "calib_rank",
        "dtype")]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-shared", "-fPIC", "-o", LIB, SRC, "-lm"])
    return LIB


def lib():
    """Load the oracle.  HILS_ORACLE_LIB names another build of hils_oracle.c to
    load instead; the mutation test uses it to run the pins on planted bugs."""
    global _lib
    if _lib is None:
        path = os.environ.get("HILS_ORACLE_LIB")
        if not path:
            path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oracle_hils_rows.restype = ctypes.c_int
        L.oracle_hils_rows.argtypes = [ctypes.POINTER(OCfg), ctypes.c_int64, P, P, P, P, P, P,
                                       P, P, ctypes.c_int32, P, P, P, P, P, P, P]
        L.oracle_scores_rows.restype = ctypes.c_int
        L.oracle_scores_rows.argtypes = [ctypes.POINTER(OCfg), ctypes.c_int64, P, P, P, P, P, P,
                                         P, ctypes.c_int32, ctypes.c_int32, P]
        L.oracle_topk_rows.restype = ctypes.c_int
        L.oracle_topk_rows.argtypes = [ctypes.c_int64, P, ctypes.c_int32, P, ctypes.c_int32,
                                       ctypes.c_int32, P, P, P]
        L.oracle_calibrate.restype = None
        L.oracle_calibrate.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_set_threads.restype = ctypes.c_int
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 = leave as is); returns the count in use."""
    return lib().oracle_set_threads(int(n))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def cfg(batch, n_q_heads, n_kv_heads, head_dim, chunk_size, top_k, calib_rank, dtype):
    return OCfg(batch, n_q_heads, n_kv_heads, head_dim, chunk_size, top_k, calib_rank, dtype)


def _qstore(q_rows, dtype):
    return _c(q_rows, np.float32 if dtype == 0 else np.uint16)


def calibrate(q, A, B):
    """q~ = q + (qA)B of one float64 vector."""
    q = _c(q, np.float64)
    A = _c(A, np.float32)
    B = _c(B, np.float32)
    d, r = A.shape
    out = np.zeros(d, dtype=np.float64)
    lib().oracle_calibrate(_p(q), _p(A), _p(B), d, r, _p(out))
    return out


def hils_rows(c: OCfg, q_rows, row_b, row_h, row_pos, A, B, pages, block_table, landmarks,
              forced_idx=None):
    """Run the oracle on explicit rows.  Returns dict(out, idx, w, sel_scores, gap);
    ``out`` is None when ``pages`` is None (selection only)."""
    n = len(row_b)
    d, k = c.head_dim, c.top_k
    q_rows = _qstore(q_rows, c.dtype).reshape(n, d)
    row_b = _c(row_b, np.int32)
    row_h = _c(row_h, np.int32)
    row_pos = _c(row_pos, np.int64)
    A = _c(A, np.float32)
    B = _c(B, np.float32)
    bt = _c(block_table, np.int32)
    max_chunks = bt.shape[-1]
    lm = _qstore(landmarks, c.dtype)
    pg = None if pages is None else _qstore(pages, c.dtype)
    fi = None if forced_idx is None else _c(forced_idx, np.int32).reshape(n, k)
    out = np.zeros((n, d), dtype=np.float64) if pg is not None else None
    idx = np.zeros((n, k), dtype=np.int32)
    w = np.zeros((n, k), dtype=np.float64)
    ss = np.zeros((n, k), dtype=np.float64)
    gap = np.zeros(n, dtype=np.float64)
    rc = lib().oracle_hils_rows(ctypes.byref(c), n, _p(q_rows), _p(row_b), _p(row_h),
                                _p(row_pos), _p(A), _p(B), _p(pg), _p(bt), max_chunks, _p(lm),
                                _p(fi), _p(out), _p(idx), _p(w), _p(ss), _p(gap))
    if rc != 0:
        raise ValueError("oracle_hils_rows: bad arguments")
    return {"out": out, "idx": idx, "w": w, "sel_scores": ss, "gap": gap}


def scores_rows(c: OCfg, q_rows, row_b, row_h, row_pos, A, B, landmarks, max_chunks, n_cols):
    n = len(row_b)
    q_rows = _qstore(q_rows, c.dtype).reshape(n, c.head_dim)
    out = np.zeros((n, n_cols), dtype=np.float64)
    rc = lib().oracle_scores_rows(ctypes.byref(c), n, _p(q_rows), _p(_c(row_b, np.int32)),
                                  _p(_c(row_h, np.int32)), _p(_c(row_pos, np.int64)),
                                  _p(_c(A, np.float32)), _p(_c(B, np.float32)),
                                  _p(_qstore(landmarks, c.dtype)), int(max_chunks), int(n_cols),
                                  _p(out))
    if rc != 0:
        raise ValueError("oracle_scores_rows: bad arguments")
    return out


def topk_rows(scores, row_pos, chunk_size, k):
    s = _c(scores, np.float64)
    n, n_cols = s.shape
    idx = np.zeros((n, k), dtype=np.int32)
    w = np.zeros((n, k), dtype=np.float64)
    gap = np.zeros(n, dtype=np.float64)
    rc = lib().oracle_topk_rows(n, _p(s), n_cols, _p(_c(row_pos, np.int64)), chunk_size, k,
                                _p(idx), _p(w), _p(gap))
    if rc != 0:
        raise ValueError("oracle_topk_rows: bad arguments")
    return idx, w, gap
