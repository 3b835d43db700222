"""hs2 -- B200-native (sm_100a) hot path of HySparse2 token-level hybrid sparse attention.

Thin Python binding of the C-ABI library ``libhs2.so`` (declared in ``include/hs2.h``):
argument marshalling only, every step of the computation runs in the library's CUDA
kernels. PyTorch provides device memory and streams. There is no CPU fallback: importing
this package fails loudly if the library cannot be loaded.

    out, lse, idx = full_attn_select(q, k, v)            # full layer + indexer
    out2 = sparse_attn(q2, k, v, idx)                     # a sparse layer (KV Reuse)
    kv = bridge_kv_proj(h, w)                             # KV Bridging projection

Tensors: q [B, Lq, H, d] bf16, k/v [B, Lk, d] bf16 (one K/V head), idx [B, Lq, S] int32,
h [T, hidden] bf16, w [n_layers, 2, hidden, d] bf16 -> kv [n_layers, 2, T, d] bf16.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

WINDOW = 128
TOPK = 1024

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libhs2.so")

STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported shape or device", 3: "workspace missing or too small",
    4: "CUDA error", 5: "device-side wait timed out", 6: "device-side index out of range",
}
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_DEVICE_BOUNDS = range(7)


class HS2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)} (status {code})")
        self.code = code


def _load_library() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        from . import _build
        _build.build()
    lib = ctypes.CDLL(_LIB_PATH)
    P, i32, f32, sz, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_longlong
    lib.hs2_abi_version.restype = i32
    lib.hs2_status_string.argtypes = [i32]
    lib.hs2_status_string.restype = ctypes.c_char_p
    lib.hs2_full_attn_select_workspace_bytes.argtypes = [i32] * 7
    lib.hs2_full_attn_select_workspace_bytes.restype = sz
    lib.hs2_full_attn_select.argtypes = [P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, P, P, P, P, sz, P]
    lib.hs2_full_attn_select.restype = i32
    lib.hs2_full_attn_select_ragged_workspace_bytes.argtypes = [i32, P, i32, i32, i32, i32, i32]
    lib.hs2_full_attn_select_ragged_workspace_bytes.restype = sz
    lib.hs2_full_attn_select_ragged.argtypes = [P, P, P, i32, P, i32, i32, i32, f32, i32, i32, P, P, P, P, sz, P]
    lib.hs2_full_attn_select_ragged.restype = i32
    lib.hs2_full_attn_select_paged_workspace_bytes.argtypes = [i32, P, i32, i32, i32, i32, i32]
    lib.hs2_full_attn_select_paged_workspace_bytes.restype = sz
    lib.hs2_full_attn_select_paged.argtypes = [P, P, P, i32, P, i32, i32, P, i32, i32, f32, i32, i32, P, P, P, P, sz, P]
    lib.hs2_full_attn_select_paged.restype = i32
    lib.hs2_sparse_attn_paged.argtypes = [P, P, P, i32, P, i32, P, i32, i32, i32, i32, i32, f32, P, P, P, sz, P]
    lib.hs2_sparse_attn_paged.restype = i32
    lib.hs2_sparse_attn_workspace_bytes.argtypes = [i32] * 6
    lib.hs2_sparse_attn_workspace_bytes.restype = sz
    lib.hs2_sparse_attn.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, f32, P, P, P, sz, P]
    lib.hs2_sparse_attn.restype = i32
    lib.hs2_full_attn_select_fp8kv_workspace_bytes.argtypes = [i32, P, i32, i32, i32, i32, i32]
    lib.hs2_full_attn_select_fp8kv_workspace_bytes.restype = sz
    lib.hs2_full_attn_select_fp8kv.argtypes = [P, P, P, f32, f32, i32, P, i32, P, i32, i32, i32, i32, f32, i32, i32,
                                               P, P, P, P, sz, P]
    lib.hs2_full_attn_select_fp8kv.restype = i32
    lib.hs2_full_attn_select_prefill_fp8kv_workspace_bytes.argtypes = [i32] * 7
    lib.hs2_full_attn_select_prefill_fp8kv_workspace_bytes.restype = sz
    lib.hs2_full_attn_select_prefill_fp8kv.argtypes = [P, P, P, f32, f32, i32, i32, i32, i32, i32, f32, i32, i32, P, P,
                                                       P, P, sz, P]
    lib.hs2_full_attn_select_prefill_fp8kv.restype = i32
    lib.hs2_sparse_attn_fp8kv.argtypes = [P, P, P, f32, f32, P, i32, i32, i32, P, i32, i32, i32, i32, i32, f32, P, P,
                                          P, sz, P]
    lib.hs2_sparse_attn_fp8kv.restype = i32
    lib.hs2_selftest_e4m3.argtypes = [P, P, P, i32, P]
    lib.hs2_selftest_e4m3.restype = i32
    lib.hs2_full_attn_select_v1_workspace_bytes.argtypes = [i32] * 7
    lib.hs2_full_attn_select_v1_workspace_bytes.restype = sz
    lib.hs2_full_attn_select_v1.argtypes = [P, P, P, i32, i32, i32, i32, f32, i32, i32, i32, P, P, P, P, sz, P]
    lib.hs2_full_attn_select_v1.restype = i32
    lib.hs2_sparse_attn_v1.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, P, P, sz, P]
    lib.hs2_sparse_attn_v1.restype = i32
    lib.hs2_attn_bwd_workspace_bytes.argtypes = [i32] * 5
    lib.hs2_attn_bwd_workspace_bytes.restype = sz
    lib.hs2_full_attn_bwd.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, P, P, P, P, sz, P]
    lib.hs2_full_attn_bwd.restype = i32
    lib.hs2_sparse_attn_bwd.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, P, P, P, P, sz, P]
    lib.hs2_sparse_attn_bwd.restype = i32
    lib.hs2_bridge_kv_proj_workspace_bytes.argtypes = [i32] * 4
    lib.hs2_bridge_kv_proj_workspace_bytes.restype = sz
    lib.hs2_bridge_kv_proj.argtypes = [P, i32, i32, P, i32, i32, P, P, sz, P]
    lib.hs2_bridge_kv_proj.restype = i32
    lib.hs2_read_device_status.argtypes = [P, P]
    lib.hs2_read_device_status.restype = i32
    lib.hs2_clear_device_status.argtypes = [P, P]
    lib.hs2_clear_device_status.restype = i32
    lib.hs2_set_wait_limit_ns.argtypes = [ll]
    lib.hs2_set_wait_limit_ns.restype = None
    lib.hs2_selftest_wait_timeout.argtypes = [P, sz, ll, P]
    lib.hs2_selftest_wait_timeout.restype = i32
    lib.hs2_selftest_exp2.argtypes = [P, P, P, i32, P]
    lib.hs2_selftest_exp2.restype = i32
    lib.hs2_kernel_launches.restype = ctypes.c_ulonglong
    lib.hs2_profile_enable.argtypes = [ctypes.c_char_p]
    lib.hs2_profile_enable.restype = None
    lib.hs2_profile_read.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
    lib.hs2_profile_read.restype = i32
    return lib


lib = _load_library()
LIBRARY_PATH = _LIB_PATH
ABI_VERSION = lib.hs2_abi_version()


def _load_marshalling():
    """The C++ module that checks torch tensors and calls hs2_full_attn_select / hs2_sparse_attn
    (bind/hs2_torch.cpp; a few microseconds of host time per call instead of the ctypes path's
    tens). None when it is not built, and the ctypes path below serves every call."""
    import importlib.util
    import sysconfig
    path = os.path.join(_PKG, "_hs2_torch" + sysconfig.get_config_var("EXT_SUFFIX"))
    if not os.path.exists(path):
        return None
    spec = importlib.util.spec_from_file_location(__name__ + "._hs2_torch", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    addr = lambda f: ctypes.cast(f, ctypes.c_void_p).value
    mod.set_entries(addr(lib.hs2_full_attn_select), addr(lib.hs2_sparse_attn))
    return mod


_fast = _load_marshalling()

_ws_lock = threading.Lock()
_ws_cache: dict = {}


def _workspace(nbytes: int, device: torch.device, key: str) -> torch.Tensor:
    """Cached per-(device, op) workspace; pass your own for concurrent streams."""
    with _ws_lock:
        k = (device, key)
        ws = _ws_cache.get(k)
        if ws is None or ws.numel() < nbytes:
            ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            _ws_cache[k] = ws
        return ws


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_ptr(stream, t: torch.Tensor | None = None) -> int:
    """The cudaStream_t of `stream`, else of the current stream of t's device (read without
    building a Stream object: this is on every call's path)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None and t is not None:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream().cuda_stream


def _check(code: int, what: str):
    if code != OK:
        raise HS2Error(code, what)


def _need(t: torch.Tensor, name: str, dtype, dim: int):
    if t.dtype is dtype and t.is_cuda and t.dim() == dim and t.is_contiguous():
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got shape {tuple(t.shape)}")
    raise ValueError(f"{name} must be contiguous")


def full_attn_select_workspace_bytes(B, Lq, Lk, H, d, window=WINDOW, topk=TOPK) -> int:
    return int(lib.hs2_full_attn_select_workspace_bytes(B, Lq, Lk, H, d, window, topk))


def sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S) -> int:
    return int(lib.hs2_sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S))


def bridge_kv_proj_workspace_bytes(T, hidden, n_layers, d) -> int:
    return int(lib.hs2_bridge_kv_proj_workspace_bytes(T, hidden, n_layers, d))


def full_attn_select(q, k, v, *, scale=None, window=WINDOW, topk=TOPK, out=None, lse=None, idx=None,
                     workspace=None, stream=None):
    """Causal MQA attention that also selects tokens (hs2_full_attn_select).

    Returns (out [B,Lq,H,d] bf16, lse [B,Lq,H] fp32 natural log, idx [B,Lq,window+topk] int32).
    """
    if _fast is not None and out is not None and lse is not None and idx is not None and workspace is not None:
        # every buffer given (a decode loop): checks and call in C++
        sc = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
        st = _stream_ptr(stream, q) if q.is_cuda else 0  # (a host tensor fails the checks in C++)
        _check(_fast.full_attn_select(q, k, v, sc, window, topk, out, lse, idx, workspace, st),
               "hs2_full_attn_select")
        return out, lse, idx
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    if tuple(k.shape) != (B, Lk, d) or tuple(v.shape) != (B, Lk, d):
        raise ValueError("k and v must be [B, Lk, d] matching q")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    S = window + topk
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Lq, H), dtype=torch.float32, device=q.device) if lse is None else lse
    idx = torch.empty((B, Lq, S), dtype=torch.int32, device=q.device) if idx is None else idx
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(idx, "idx", torch.int32, 3)
    ws = workspace if workspace is not None else _workspace(
        full_attn_select_workspace_bytes(B, Lq, Lk, H, d, window, topk), q.device, "full")
    code = lib.hs2_full_attn_select(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Lq, Lk, H, d, scale, window, topk,
                                    out.data_ptr(), lse.data_ptr(), idx.data_ptr(), ws.data_ptr(), ws.nbytes,
                                    _stream_ptr(stream, q))
    _check(code, "hs2_full_attn_select")
    return out, lse, idx


V1_BLOCK = 64
V1_BLOCKS = 16


def full_attn_select_v1_workspace_bytes(B, Lk, H, d, window=WINDOW, block=V1_BLOCK, n_blocks=V1_BLOCKS) -> int:
    return int(lib.hs2_full_attn_select_v1_workspace_bytes(B, Lk, H, d, window, block, n_blocks))


def full_attn_select_v1(q, k, v, *, scale=None, window=WINDOW, block=V1_BLOCK, n_blocks=V1_BLOCKS, out=None,
                        lse=None, idx=None, workspace=None, stream=None):
    """Decode full layer with HySparse (v1) block selection (hs2_full_attn_select_v1).

    q [B,1,H,d]; k, v [B,Lk,d]. Returns (out [B,1,H,d] bf16, lse [B,1,H] fp32, idx
    [B,1,n_blocks*block+window] int32: the chosen blocks' tokens, then the window).
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    if Lq != 1 or tuple(k.shape) != (B, Lk, d) or tuple(v.shape) != (B, Lk, d):
        raise ValueError("q must be [B,1,H,d] and k, v [B,Lk,d]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    S = n_blocks * block + window
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, 1, H), dtype=torch.float32, device=q.device) if lse is None else lse
    idx = torch.empty((B, 1, S), dtype=torch.int32, device=q.device) if idx is None else idx
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(idx, "idx", torch.int32, 3)
    nbytes = full_attn_select_v1_workspace_bytes(B, Lk, H, d, window, block, n_blocks)
    ws = _workspace(nbytes, q.device, "full_v1") if workspace is None else workspace
    code = lib.hs2_full_attn_select_v1(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Lk, H, d, scale, window, block,
                                       n_blocks, out.data_ptr(), lse.data_ptr(), idx.data_ptr(), ws.data_ptr(),
                                       ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_full_attn_select_v1")
    return out, lse, idx


def sparse_attn_v1(q, k, v, idx, gate, *, branch=V1_BLOCK * V1_BLOCKS, scale=None, out=None, workspace=None,
                   stream=None):
    """Sparse layer of the v1 design (hs2_sparse_attn_v1): gate * attention over idx slots
    [0, branch) + (1 - gate) * attention over slots [branch, S). gate [B,Lq,H] fp32."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(idx, "idx", torch.int32, 3)
    _need(gate, "gate", torch.float32, 3)
    B, Lq, H, d = q.shape
    Lk, S = k.shape[1], idx.shape[2]
    if tuple(idx.shape[:2]) != (B, Lq) or tuple(gate.shape) != (B, Lq, H):
        raise ValueError("idx must be [B,Lq,S] and gate [B,Lq,H]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", torch.bfloat16, 4)
    nbytes = sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S)
    ws = _workspace(nbytes, q.device, "sparse") if workspace is None else workspace
    code = lib.hs2_sparse_attn_v1(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), gate.data_ptr(), B, Lq,
                                  Lk, H, d, S, branch, scale, out.data_ptr(), ws.data_ptr(),
                                  ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_sparse_attn_v1")
    return out


def attn_bwd_workspace_bytes(B, Lq, Lk, H, d) -> int:
    return int(lib.hs2_attn_bwd_workspace_bytes(B, Lq, Lk, H, d))


def _bwd_outputs(q, k, dq, dk, dv):
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.zeros((B, Lk, d), dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.zeros((B, Lk, d), dtype=torch.float32, device=q.device) if dv is None else dv
    _need(dq, "dq", torch.bfloat16, 4)
    _need(dk, "dk", torch.float32, 3)
    _need(dv, "dv", torch.float32, 3)
    return dq, dk, dv


def full_attn_bwd(q, k, v, out, lse, do, *, scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward of the full layer's causal attention (hs2_full_attn_bwd).

    out, lse: the forward's outputs for q, k, v; do: [B,Lq,H,d] bf16 upstream gradient.
    Returns (dq [B,Lq,H,d] bf16, dk, dv [B,Lk,d] fp32). dk and dv are ADDED into when given
    (zeros otherwise): the layers of a block share K and V.
    """
    for t, n in ((q, "q"), (out, "out"), (do, "do")):
        _need(t, n, torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(lse, "lse", torch.float32, 3)
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq, dk, dv = _bwd_outputs(q, k, dq, dk, dv)
    nbytes = attn_bwd_workspace_bytes(B, Lq, Lk, H, d)
    ws = _workspace(nbytes, q.device, "bwd") if workspace is None else workspace
    code = lib.hs2_full_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), B, Lq, Lk, H, d, scale, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                 ws.data_ptr(), ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_full_attn_bwd")
    return dq, dk, dv


def sparse_attn_bwd(q, k, v, idx, out, lse, do, *, scale=None, dq=None, dk=None, dv=None, workspace=None,
                    stream=None):
    """Backward of a sparse layer over the selected tokens (hs2_sparse_attn_bwd); out and lse
    are the forward sparse layer's (sparse_attn with want_lse=True). Returns (dq, dk, dv) as
    full_attn_bwd, dk and dv accumulated."""
    for t, n in ((q, "q"), (out, "out"), (do, "do")):
        _need(t, n, torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(lse, "lse", torch.float32, 3)
    _need(idx, "idx", torch.int32, 3)
    B, Lq, H, d = q.shape
    Lk, S = k.shape[1], idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq, dk, dv = _bwd_outputs(q, k, dq, dk, dv)
    nbytes = attn_bwd_workspace_bytes(B, Lq, Lk, H, d)
    ws = _workspace(nbytes, q.device, "bwd") if workspace is None else workspace
    code = lib.hs2_sparse_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), do.data_ptr(), B, Lq, Lk, H, d, S, scale, dq.data_ptr(),
                                   dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                                   _stream_ptr(stream))
    _check(code, "hs2_sparse_attn_bwd")
    return dq, dk, dv


def _lens_array(lens, B, Lk):
    arr = (ctypes.c_int32 * B)(*[int(x) for x in lens])
    if len(lens) != B or any(not (1 <= int(x) <= Lk) for x in lens):
        raise ValueError(f"lens must hold B={B} lengths in [1, {Lk}]")
    return arr


def full_attn_select_ragged_workspace_bytes(lens, Lk, H, d, window=WINDOW, topk=TOPK) -> int:
    B = len(lens)
    return int(lib.hs2_full_attn_select_ragged_workspace_bytes(B, _lens_array(lens, B, Lk), Lk, H, d, window, topk))


def full_attn_select_ragged(q, k, v, lens, *, scale=None, window=WINDOW, topk=TOPK, out=None, lse=None, idx=None,
                            workspace=None, stream=None):
    """Decode over sequences of different cache lengths (hs2_full_attn_select_ragged).

    q [B,1,H,d]; k, v [B,Lk,d] with sequence b's cache in its first lens[b] rows; lens: B host
    integers. Returns (out [B,1,H,d] bf16, lse [B,1,H] fp32, idx [B,1,window+topk] int32).
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    if Lq != 1 or tuple(k.shape) != (B, Lk, d) or tuple(v.shape) != (B, Lk, d):
        raise ValueError("q must be [B,1,H,d] and k, v [B,Lk,d]")
    lens_c = _lens_array(list(lens), B, Lk)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    S = window + topk
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, 1, H), dtype=torch.float32, device=q.device) if lse is None else lse
    idx = torch.empty((B, 1, S), dtype=torch.int32, device=q.device) if idx is None else idx
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(idx, "idx", torch.int32, 3)
    nbytes = int(lib.hs2_full_attn_select_ragged_workspace_bytes(B, lens_c, Lk, H, d, window, topk))
    ws = _workspace(nbytes, q.device, "full") if workspace is None else workspace
    code = lib.hs2_full_attn_select_ragged(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, lens_c, Lk, H, d, scale, window,
                                           topk, out.data_ptr(), lse.data_ptr(), idx.data_ptr(), ws.data_ptr(),
                                           ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_full_attn_select_ragged")
    return out, lse, idx


def full_attn_select_paged_workspace_bytes(lens, max_pages, H, d, window=WINDOW, topk=TOPK) -> int:
    B = len(lens)
    return int(lib.hs2_full_attn_select_paged_workspace_bytes(B, _lens_array(lens, B, max_pages * 128), max_pages, H, d,
                                                              window, topk))


def full_attn_select_paged(q, k_pages, v_pages, page_table, lens, *, scale=None, window=WINDOW, topk=TOPK, out=None,
                           lse=None, idx=None, workspace=None, stream=None):
    """Decode over a paged cache (hs2_full_attn_select_paged).

    q [B,1,H,d]; k_pages, v_pages [n_pages,128,d]; page_table [B,max_pages] int32 on the device;
    lens: B host integers. Returns (out, lse, idx) as full_attn_select_ragged.
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k_pages, "k_pages", torch.bfloat16, 3)
    _need(v_pages, "v_pages", torch.bfloat16, 3)
    _need(page_table, "page_table", torch.int32, 2)
    B, Lq, H, d = q.shape
    n_pages = k_pages.shape[0]
    max_pages = page_table.shape[1]
    if Lq != 1 or tuple(k_pages.shape) != (n_pages, 128, d) or v_pages.shape != k_pages.shape or page_table.shape[0] != B:
        raise ValueError("q [B,1,H,d], k_pages/v_pages [n_pages,128,d], page_table [B,max_pages]")
    lens_c = _lens_array(list(lens), B, max_pages * 128)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    S = window + topk
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, 1, H), dtype=torch.float32, device=q.device) if lse is None else lse
    idx = torch.empty((B, 1, S), dtype=torch.int32, device=q.device) if idx is None else idx
    nbytes = int(lib.hs2_full_attn_select_paged_workspace_bytes(B, lens_c, max_pages, H, d, window, topk))
    ws = _workspace(nbytes, q.device, "full") if workspace is None else workspace
    code = lib.hs2_full_attn_select_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), n_pages,
                                          page_table.data_ptr(), max_pages, B, lens_c, H, d, scale, window, topk,
                                          out.data_ptr(), lse.data_ptr(), idx.data_ptr(), ws.data_ptr(),
                                          ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_full_attn_select_paged")
    return out, lse, idx


def sparse_attn_paged(q, k_pages, v_pages, page_table, idx, *, scale=None, out=None, workspace=None, stream=None):
    """Sparse attention over a paged cache (hs2_sparse_attn_paged); idx [B,Lq,S] token positions."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_pages, "k_pages", torch.bfloat16, 3)
    _need(v_pages, "v_pages", torch.bfloat16, 3)
    _need(page_table, "page_table", torch.int32, 2)
    _need(idx, "idx", torch.int32, 3)
    B, Lq, H, d = q.shape
    S = idx.shape[2]
    n_pages, max_pages = k_pages.shape[0], page_table.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    nbytes = sparse_attn_workspace_bytes(B, Lq, max_pages * 128, H, d, S)
    ws = _workspace(nbytes, q.device, "sparse") if workspace is None else workspace
    code = lib.hs2_sparse_attn_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), n_pages,
                                     page_table.data_ptr(), max_pages, idx.data_ptr(), B, Lq, H, d, S, scale,
                                     out.data_ptr(), None, ws.data_ptr(), ws.nbytes,
                                     _stream_ptr(stream, ws))
    _check(code, "hs2_sparse_attn_paged")
    return out


def _fp8_cache(k8, v8, page_table, B, d):
    """(Lk, max_pages, n_pages) of an e4m3 cache: [B,Lk,d] rows, or pools [n_pages,128,d] + table."""
    _need(k8, "k8", torch.uint8, 3)
    _need(v8, "v8", torch.uint8, 3)
    if v8.shape != k8.shape or k8.shape[2] != d:
        raise ValueError("k8 and v8 must have the same shape [.., .., d]")
    if page_table is None:
        if k8.shape[0] != B:
            raise ValueError("k8, v8 must be [B, Lk, d]")
        return k8.shape[1], 0, 0
    _need(page_table, "page_table", torch.int32, 2)
    if k8.shape[1] != 128 or page_table.shape[0] != B:
        raise ValueError("paged: k8, v8 [n_pages, 128, d], page_table [B, max_pages]")
    return page_table.shape[1] * 128, page_table.shape[1], k8.shape[0]


def full_attn_select_fp8kv_workspace_bytes(B, lens, Lk, H, d, window=WINDOW, topk=TOPK) -> int:
    lens_c = _lens_array(list(lens), B, Lk) if lens is not None else None
    return int(lib.hs2_full_attn_select_fp8kv_workspace_bytes(B, lens_c, Lk, H, d, window, topk))


def full_attn_select_fp8kv(q, k8, v8, k_scale, v_scale, *, lens=None, page_table=None, scale=None, window=WINDOW,
                           topk=TOPK, out=None, lse=None, idx=None, workspace=None, stream=None):
    """Decode step over an e4m3 K/V cache (hs2_full_attn_select_fp8kv).

    q [B,1,H,d] bf16; k8, v8 uint8 e4m3 codes [B,Lk,d] (or page pools [n_pages,128,d] with
    page_table [B,max_pages] int32 on the device); the cache is k_scale * k8, v_scale * v8;
    lens: B host integers or None (every sequence full). Returns (out, lse, idx) as
    full_attn_select_ragged.
    """
    _need(q, "q", torch.bfloat16, 4)
    B, Lq, H, d = q.shape
    if Lq != 1:
        raise ValueError("q must be [B, 1, H, d]")
    Lk, max_pages, n_pages = _fp8_cache(k8, v8, page_table, B, d)
    lens_c = _lens_array(list(lens), B, Lk) if lens is not None else None
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    S = window + topk
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, 1, H), dtype=torch.float32, device=q.device) if lse is None else lse
    idx = torch.empty((B, 1, S), dtype=torch.int32, device=q.device) if idx is None else idx
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(idx, "idx", torch.int32, 3)
    nbytes = int(lib.hs2_full_attn_select_fp8kv_workspace_bytes(B, lens_c, Lk, H, d, window, topk))
    ws = _workspace(nbytes, q.device, "full") if workspace is None else workspace
    code = lib.hs2_full_attn_select_fp8kv(q.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(k_scale), float(v_scale), B,
                                          lens_c, Lk, page_table.data_ptr() if page_table is not None else None,
                                          max_pages, n_pages, H, d, scale, window, topk, out.data_ptr(),
                                          lse.data_ptr(), idx.data_ptr(), ws.data_ptr(),
                                          ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_full_attn_select_fp8kv")
    return out, lse, idx


def full_attn_select_prefill_fp8kv(q, k8, v8, k_scale, v_scale, *, scale=None, window=WINDOW, topk=TOPK, out=None,
                                   lse=None, idx=None, workspace=None, stream=None):
    """Full attention + selection of Lq queries over an e4m3 K/V cache [B,Lk,d]
    (hs2_full_attn_select_prefill_fp8kv): a whole prompt (Lq == Lk), a chunk (Lq < Lk) or one
    decode query. Returns (out, lse, idx) as full_attn_select."""
    _need(q, "q", torch.bfloat16, 4)
    B, Lq, H, d = q.shape
    Lk, _, _ = _fp8_cache(k8, v8, None, B, d)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    S = window + topk
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Lq, H), dtype=torch.float32, device=q.device) if lse is None else lse
    idx = torch.empty((B, Lq, S), dtype=torch.int32, device=q.device) if idx is None else idx
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(idx, "idx", torch.int32, 3)
    nbytes = int(lib.hs2_full_attn_select_prefill_fp8kv_workspace_bytes(B, Lq, Lk, H, d, window, topk))
    ws = _workspace(nbytes, q.device, "full") if workspace is None else workspace
    code = lib.hs2_full_attn_select_prefill_fp8kv(q.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(k_scale),
                                                  float(v_scale), B, Lq, Lk, H, d, scale, window, topk, out.data_ptr(),
                                                  lse.data_ptr(), idx.data_ptr(), ws.data_ptr(),
                                                  ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_full_attn_select_prefill_fp8kv")
    return out, lse, idx


def sparse_attn_fp8kv(q, k8, v8, k_scale, v_scale, idx, *, page_table=None, scale=None, out=None, lse=None,
                      want_lse=False, workspace=None, stream=None):
    """Sparse attention over an e4m3 K/V cache (hs2_sparse_attn_fp8kv); arguments as
    full_attn_select_fp8kv and sparse_attn. Returns out, or (out, lse) when want_lse or lse is given."""
    _need(q, "q", torch.bfloat16, 4)
    _need(idx, "idx", torch.int32, 3)
    B, Lq, H, d = q.shape
    Lk, max_pages, n_pages = _fp8_cache(k8, v8, page_table, B, d)
    S = idx.shape[2]
    if tuple(idx.shape[:2]) != (B, Lq):
        raise ValueError("idx must be [B, Lq, S]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", torch.bfloat16, 4)
    if want_lse and lse is None:
        lse = torch.empty((B, Lq, H), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
    nbytes = sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S)
    ws = _workspace(nbytes, q.device, "sparse") if workspace is None else workspace
    code = lib.hs2_sparse_attn_fp8kv(q.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(k_scale), float(v_scale),
                                     idx.data_ptr(), B, Lq, Lk, page_table.data_ptr() if page_table is not None else None,
                                     max_pages, n_pages, H, d, S, scale, out.data_ptr(),
                                     lse.data_ptr() if lse is not None else None, ws.data_ptr(),
                                     ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_sparse_attn_fp8kv")
    return (out, lse) if lse is not None else out


def sparse_attn(q, k, v, idx, *, scale=None, out=None, lse=None, want_lse=False, workspace=None, stream=None):
    """Sparse attention of one sparse layer over the reused K/V and indices (hs2_sparse_attn).

    Returns out [B,Lq,H,d] bf16, or (out, lse) when want_lse or lse is given.
    """
    if _fast is not None and out is not None and workspace is not None and (lse is not None or not want_lse):
        # every buffer given (a decode loop): checks and call in C++
        sc = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
        st = _stream_ptr(stream, q) if q.is_cuda else 0  # (a host tensor fails the checks in C++)
        _check(_fast.sparse_attn(q, k, v, idx, sc, out, lse, workspace, st), "hs2_sparse_attn")
        return (out, lse) if lse is not None else out
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(idx, "idx", torch.int32, 3)
    B, Lq, H, d = q.shape
    Lk = k.shape[1]
    S = idx.shape[2]
    if tuple(idx.shape[:2]) != (B, Lq):
        raise ValueError("idx must be [B, Lq, S]")
    if tuple(k.shape) != (B, Lk, d) or tuple(v.shape) != (B, Lk, d):
        raise ValueError("k and v must be [B, Lk, d] matching q")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", torch.bfloat16, 4)
    if want_lse and lse is None:
        lse = torch.empty((B, Lq, H), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
    ws = workspace if workspace is not None else _workspace(
        sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S), q.device, "sparse")
    code = lib.hs2_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), B, Lq, Lk, H, d, S, scale,
                               out.data_ptr(), lse.data_ptr() if lse is not None else None, ws.data_ptr(),
                               ws.nbytes, _stream_ptr(stream, q))
    _check(code, "hs2_sparse_attn")
    return (out, lse) if lse is not None else out


def bridge_kv_proj(h, w, *, out=None, workspace=None, stream=None):
    """KV Bridging: kv[l, 0] = h @ w[l, 0], kv[l, 1] = h @ w[l, 1] (hs2_bridge_kv_proj)."""
    _need(h, "h", torch.bfloat16, 2)
    _need(w, "w", torch.bfloat16, 4)
    T, hidden = h.shape
    n, two, hw, d = w.shape
    if two != 2 or hw != hidden:
        raise ValueError("w must be [n_layers, 2, hidden, d]")
    out = torch.empty((n, 2, T, d), dtype=torch.bfloat16, device=h.device) if out is None else out
    _need(out, "out", torch.bfloat16, 4)
    nbytes = bridge_kv_proj_workspace_bytes(T, hidden, n, d)
    ws = _workspace(nbytes, h.device, "bridge") if workspace is None else workspace
    code = lib.hs2_bridge_kv_proj(h.data_ptr(), T, hidden, w.data_ptr(), n, d, out.data_ptr(), ws.data_ptr(),
                                  ws.nbytes, _stream_ptr(stream, ws))
    _check(code, "hs2_bridge_kv_proj")
    return out


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Waits for the stream and returns the status word of `workspace` (0 = ok)."""
    return int(lib.hs2_read_device_status(workspace.data_ptr(), _stream_ptr(stream)))


def clear_device_status(workspace: torch.Tensor, stream=None) -> None:
    _check(lib.hs2_clear_device_status(workspace.data_ptr(), _stream_ptr(stream)), "hs2_clear_device_status")


def cached_workspace(key: str, device=None):
    """The workspace the convenience calls used for `key` ("full", "sparse", "bridge")."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return _ws_cache.get((device, key))


def set_wait_limit_ns(ns: int) -> None:
    lib.hs2_set_wait_limit_ns(int(ns))


def selftest_wait_timeout(workspace: torch.Tensor, limit_ns: int, stream=None) -> None:
    _check(lib.hs2_selftest_wait_timeout(workspace.data_ptr(), workspace.numel(), int(limit_ns), _stream_ptr(stream)),
           "hs2_selftest_wait_timeout")


def selftest_exp2(x: torch.Tensor, stream=None):
    """(software 2^x, MUFU 2^x) of the device float32 tensor x (even length), see hs2.h."""
    _need(x, "x", torch.float32, 1)
    ys, ym = torch.empty_like(x), torch.empty_like(x)
    _check(lib.hs2_selftest_exp2(x.data_ptr(), ys.data_ptr(), ym.data_ptr(), x.numel(), _stream_ptr(stream)),
           "hs2_selftest_exp2")
    return ys, ym


def selftest_e4m3(x: torch.Tensor, stream=None):
    """(f16 bits, bf16 bits) as int16 tensors: the device widening of the e4m3 codes x (uint8,
    even length) that the FP8-cache kernels use, see hs2.h."""
    _need(x, "x", torch.uint8, 1)
    yh = torch.empty(x.numel(), dtype=torch.int16, device=x.device)
    yb = torch.empty_like(yh)
    _check(lib.hs2_selftest_e4m3(x.data_ptr(), yh.data_ptr(), yb.data_ptr(), x.numel(), _stream_ptr(stream)),
           "hs2_selftest_e4m3")
    return yh, yb


def kernel_launches() -> int:
    """CUDA kernels this library launched since it was loaded."""
    return int(lib.hs2_kernel_launches())


def profile_enable(kernel: str | None) -> None:
    """None: off; "*": time every kernel; otherwise time only the named kernel."""
    lib.hs2_profile_enable(kernel.encode() if kernel is not None else None)


def profile_read(kernel: str) -> tuple[float, int]:
    """(summed milliseconds, launches) of the recorded launches of `kernel`; forgets them."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_longlong(0)
    if lib.hs2_profile_read(kernel.encode(), ctypes.byref(ms), ctypes.byref(n)) != 0:
        raise HS2Error(ERR_CUDA, "hs2_profile_read")
    return ms.value, n.value
