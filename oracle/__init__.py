"""fp64 CPU oracle of the HySparse2 hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package. It shares no code with ``long_context_mqa_b200`` (neither imports the other);
both consume the bf16 inputs produced by ``synth``.

The arithmetic lives in ``hs2_oracle.c`` (plain loops, double precision, libm exp/log),
compiled on first use with gcc into ``liboracle.so`` next to it. See that file's header
for what is computed and which passages of the pages each function follows.

Arrays: bf16 tensors are passed as numpy ``uint16`` bit patterns.

An FP8 (e4m3) K/V cache is read through ``e4m3_to_bf16``: the codes are decoded from the OCP
8-bit floating-point definition (numpy, below) and multiplied by the tensor's power-of-two
scale; every such value is exactly a bf16 value, so the functions above then run unchanged on
the cache the kernels read.
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
            lib.oracle_attn_bwd.argtypes = [P, P, P, P, P, i, i, i, i, i, i, d, P, i64, P, P, P, i]
            for f in (lib.oracle_full_attn_select, lib.oracle_sparse_attn, lib.oracle_bridge_kv_proj,
                      lib.oracle_attn_bwd):
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


def e4m3_values() -> np.ndarray:
    """The value of each of the 256 e4m3 codes (float64; NaN for 0x7F and 0xFF).

    Code bits s eeee mmm: exponent field e with bias 7; e == 0 encodes the subnormals
    m/8 * 2^-6, otherwise (1 + m/8) * 2^(e - 7); no infinities, and s 1111 111 is NaN.
    """
    c = np.arange(256)
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.power(2.0, e - 7.0))
    val = np.where(s == 1, -mag, mag)
    val[(c & 0x7F) == 0x7F] = np.nan
    return val


def e4m3_to_bf16(codes, scale: float) -> np.ndarray:
    """bf16 bit patterns of code value * scale (scale a power of two; exact, else ValueError)."""
    m, _ = np.frexp(scale)
    if not (scale > 0 and m == 0.5):
        raise ValueError("the e4m3 scale must be a positive power of two")
    x = e4m3_values()[np.asarray(codes, dtype=np.uint8)] * scale
    if np.isnan(x).any():
        raise ValueError("NaN code in the e4m3 cache")
    f = x.astype(np.float32)
    u = f.view(np.uint32)
    if np.any(f.astype(np.float64) != x) or np.any(u & np.uint32(0xFFFF)):
        raise ValueError("dequantised value is not a bf16 value")
    return (u >> np.uint32(16)).astype(np.uint16)


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


def block_scores(score_row, t, block=64):
    """Score of every block meeting 0..t: the sum of its tokens' scores at or before t (the
    reading of the HySparse block score stated in block_select)."""
    score_row = np.asarray(score_row, dtype=np.float64)
    nb = t // block + 1
    return np.array([score_row[j * block:min((j + 1) * block, t + 1)].sum() for j in range(nb)])


def block_select(score_row, t, block=64, n_blocks=16):
    """The HySparse (v1) selection of one query at position t: the n_blocks blocks of `block`
    consecutive tokens with the largest block score, ties to the lower block; returns the chosen
    blocks' tokens at or before t, ascending (every token 0..t when at most n_blocks blocks exist).

    The pages give the selection's shape (1,024 global tokens chosen in 64-token blocks, beside a
    separate 128-token sliding-window branch fused by a gate: arex-research.com, section "外层 KV
    Bridging，内层 KV Reuse", the paragraph on the two changes from HySparse) but not the block
    score. Reading taken: a block's score is the sum of the token scores (the full layer's
    head-summed attention probabilities) of its tokens at or before t; every block that starts at
    or before t is a candidate (the window branch is separate, so recent blocks compete too).
    score_row: [>= t + 1] float64 token scores.
    """
    nb = t // block + 1                       # blocks meeting 0..t
    if nb <= n_blocks:
        return np.arange(t + 1, dtype=np.int64)
    bs = block_scores(score_row, t, block)
    order = sorted(range(nb), key=lambda j: (-bs[j], j))
    chosen = sorted(order[:n_blocks])
    return np.concatenate([np.arange(j * block, min((j + 1) * block, t + 1)) for j in chosen]).astype(np.int64)


def sparse_attn_v1(q, k, v, block_idx, gate, scale, window=128, threads=0):
    """HySparse (v1) sparse layer: softmax attention over the selected blocks' tokens and over the
    last `window` tokens (the sliding-window branch), fused per (query, head) as
    gate * blocks + (1 - gate) * window (same page and section as block_select; the gate is a
    learned function of the hidden state that the pages do not specify, so it is an input here).
    q: [B,Lq,H,d], k/v: [B,Lk,d] (bf16 bits); block_idx: [B,Lq,S] token indices (-1 = empty);
    gate: [B,Lq,H] in [0, 1]. Returns dict(out [B*Lq,H,d] f64)."""
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    gate = np.asarray(gate, dtype=np.float64).reshape(B * Lq, H)
    win = np.full((B, Lq, window), -1, np.int32)
    for i in range(Lq):
        t = Lk - Lq + i
        lo = max(0, t - window + 1)
        win[:, i, :t - lo + 1] = np.arange(lo, t + 1, dtype=np.int32)
    ob = sparse_attn(q, k, v, block_idx, scale, threads=threads)["out"]
    ow = sparse_attn(q, k, v, win, scale, threads=threads)["out"]
    return {"out": gate[:, :, None] * ob + (1.0 - gate[:, :, None]) * ow}


def attn_bwd(q, k, v, do, scale, idx=None, rows=None, want_kv=True, threads=0):
    """Gradients of causal MQA attention (idx None: query i at t = Lk - Lq + i reads keys 0..t)
    or of sparse attention over idx [B,Lq,S] (-1 = empty), for the output gradient do
    [B,Lq,H,d] (bf16 bits like q). Returns dict(dq [n,H,d] f64 for `rows` (default all),
    dk, dv [B,Lk,d] f64 when want_kv (then rows must be None))."""
    q, k, v, do = _u16(q), _u16(k), _u16(v), _u16(do)
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    assert do.shape == q.shape and k.shape == (B, Lk, d) and v.shape == k.shape
    if want_kv and rows is not None:
        raise ValueError("dk, dv need every row")
    S = 0
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        assert idx.shape[:2] == (B, Lq)
        S = idx.shape[2]
    r, n = _rows(rows, B * Lq)
    dq = np.empty((n, H, d), np.float64)
    dk = np.empty((B, Lk, d), np.float64) if want_kv else None
    dv = np.empty((B, Lk, d), np.float64) if want_kv else None
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(idx), B, Lq, Lk, H, d, S, float(scale),
                                 _ptr(r), n, _ptr(dq), _ptr(dk), _ptr(dv), threads)
    _check(rc, "attn_bwd")
    res = {"dq": dq}
    if want_kv:
        res["dk"], res["dv"] = dk, dv
    return res


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
