"""fp64 CPU oracle of the HySparse2 hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package. It shares no code with ``long_context_mqa_b200`` (neither imports the other);
both consume the bf16 inputs produced by ``synth``.

The arithmetic lives in ``hs2_oracle.c`` (plain loops, double precision, libm exp/log),
compiled on first use with gcc into ``liboracle.so`` next to it. See that file's header
for what is computed and which passages of the pages each function follows.

Arrays: bf16 tensors are passed as numpy ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

ERRORS = {1: "invalid argument", 2: "index out of range / empty selection", 3: "out of memory"}


def build(force: bool = False) -> str:
    """Compile hs2_oracle.c into liboracle.so (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i, d, i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
            lib.oracle_full_attn_select.argtypes = [P, P, P, i, i, i, i, i, d, i, i, P, i64, P, P, P, P, i]
            lib.oracle_sparse_attn.argtypes = [P, P, P, P, i, i, i, i, i, i, d, P, i64, P, P, i]
            lib.oracle_bridge_kv_proj.argtypes = [P, i, i, P, i, i, P, i64, P, i]
            for f in (lib.oracle_full_attn_select, lib.oracle_sparse_attn, lib.oracle_bridge_kv_proj):
                f.restype = ctypes.c_int
            lib.oracle_default_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs must be uint16 bit patterns")
    return a


def _rows(rows, total):
    if rows is None:
        return None, total
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    return r, r.size


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what}: {ERRORS.get(rc, rc)}")


def full_attn_select(q, k, v, scale, window, topk, rows=None, want_score=False, threads=0):
    """Causal MQA attention + selection. q: [B,Lq,H,d], k/v: [B,Lk,d] (bf16 bits).

    rows: flattened query rows (b*Lq + i) to compute, default all.
    Returns dict(out [n,H,d] f64, lse [n,H] f64, idx [n,window+topk] i32 ascending -1 padded,
    score [n,Lk] f64 if want_score).
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Lq, H, d = q.shape
    Bk, Lk, dk = k.shape
    assert Bk == B and dk == d and v.shape == k.shape
    r, n = _rows(rows, B * Lq)
    out = np.empty((n, H, d), np.float64)
    lse = np.empty((n, H), np.float64)
    idx = np.empty((n, window + topk), np.int32)
    score = np.empty((n, Lk), np.float64) if want_score else None
    rc = _load().oracle_full_attn_select(_ptr(q), _ptr(k), _ptr(v), B, Lq, Lk, H, d, float(scale), window, topk,
                                         _ptr(r), n, _ptr(out), _ptr(lse), _ptr(idx), _ptr(score), threads)
    _check(rc, "full_attn_select")
    res = {"out": out, "lse": lse, "idx": idx}
    if want_score:
        res["score"] = score
    return res


def sparse_attn(q, k, v, idx, scale, rows=None, threads=0):
    """Sparse attention over idx[b,i,:] (-1 = empty). Returns dict(out [n,H,d], lse [n,H])."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    B, Lq, H, d = q.shape
    _, Lk, _ = k.shape
    assert idx.shape[:2] == (B, Lq)
    S = idx.shape[2]
    r, n = _rows(rows, B * Lq)
    out = np.empty((n, H, d), np.float64)
    lse = np.empty((n, H), np.float64)
    rc = _load().oracle_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), B, Lq, Lk, H, d, S, float(scale), _ptr(r),
                                    n, _ptr(out), _ptr(lse), threads)
    _check(rc, "sparse_attn")
    return {"out": out, "lse": lse}


def bridge_kv_proj(h, w, rows=None, threads=0):
    """KV Bridging. h: [T, hidden], w: [n, 2, hidden, d] -> KV [n, 2, n_rows, d] (f64)."""
    h, w = _u16(h), _u16(w)
    T, hidden = h.shape
    n_layers, two, hw, d = w.shape
    assert two == 2 and hw == hidden
    r, n = _rows(rows, T)
    kv = np.empty((n_layers, 2, n, d), np.float64)
    rc = _load().oracle_bridge_kv_proj(_ptr(h), T, hidden, _ptr(w), n_layers, d, _ptr(r), n, _ptr(kv), threads)
    _check(rc, "bridge_kv_proj")
    return kv
