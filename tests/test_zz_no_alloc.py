"""hs2_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.

Such callers (for example a plugin whose enqueue hook runs inside an inference runtime that
forbids device allocation there and provides no scratch buffer) use this entry point, which
keeps its scratch in a 4 KiB array inside the library instead of a caller workspace. These
tests call it through the C ABI and require the same results as hs2_sparse_attn (which is
given its own workspace), on two calls in a row, including shapes whose rows split over a
cluster; the fp64 oracle's results on the same indices; that an index outside the cache is
reported by hs2_sparse_attn_noalloc_status and that the next valid call reports nothing; and
that every supported shape's workspace fits the scratch, while an invalid shape is refused
before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_out_close, bf16_to_f64, to_torch_bf16

pytestmark = pytest.mark.gpu


def _entry():
    import long_context_mqa_b200 as hs2
    lib = ctypes.CDLL(hs2.LIBRARY_PATH)
    f = lib.hs2_sparse_attn_noalloc
    P, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, i, i, i, i, i, i, ctypes.c_float, P, P, P]
    f.restype = i
    return hs2, f


def _status():
    import long_context_mqa_b200 as hs2
    lib = ctypes.CDLL(hs2.LIBRARY_PATH)
    f = lib.hs2_sparse_attn_noalloc_status
    f.argtypes = [ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f(torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    hs2, f = _entry()
    B, Lk, S = 6, 7000, 1152
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    k, v = to_torch_bf16(g.k), to_torch_bf16(g.v)
    _, _, idx = hs2.full_attn_select(to_torch_bf16(g.q), k, v, scale=g.wl.scale)
    stream = torch.cuda.current_stream().cuda_stream
    for layer in range(2):  # two calls in a row, each with its own sparse-layer queries
        q = to_torch_bf16(g.q_sparse(layer))
        ws = torch.zeros(hs2.sparse_attn_workspace_bytes(B, 1, Lk, 64, 128, S), dtype=torch.uint8, device="cuda")
        ref, ref_lse = hs2.sparse_attn(q, k, v, idx, scale=g.wl.scale, want_lse=True, workspace=ws)
        out = torch.empty_like(q)
        lse = torch.empty_like(ref_lse)
        rc = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), B, 1, Lk, 64, 128, S, g.wl.scale,
               out.data_ptr(), lse.data_ptr(), stream)
        assert rc == 0, hs2.STATUS.get(rc, rc)
        assert _status() == 0
        torch.cuda.synchronize()
        assert_out_close(bf16_to_f64(out), bf16_to_f64(ref), f"no-alloc vs workspace entry point, call {layer}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=0, atol=2e-3)


def test_noalloc_matches_oracle_and_reports_a_bad_index():
    hs2, f = _entry()
    B, Lk, S = 3, 2500, 1152
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    k, v = to_torch_bf16(g.k), to_torch_bf16(g.v)
    _, _, idx = hs2.full_attn_select(to_torch_bf16(g.q), k, v, scale=g.wl.scale)
    stream = torch.cuda.current_stream().cuda_stream
    qs = g.q_sparse(1)
    q = to_torch_bf16(qs)
    out = torch.empty_like(q)
    lse = torch.empty((B, 1, 64), dtype=torch.float32, device="cuda")
    rc = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), B, 1, Lk, 64, 128, S, g.wl.scale,
           out.data_ptr(), lse.data_ptr(), stream)
    assert rc == 0 and _status() == 0
    idx_np = idx.cpu().numpy()
    ref = oracle.sparse_attn(qs, g.k, g.v, idx_np, g.wl.scale)
    assert_out_close(bf16_to_f64(out).reshape(ref["out"].shape), ref["out"], "no-alloc vs oracle")
    assert np.abs(lse.double().cpu().numpy().reshape(ref["lse"].shape) - ref["lse"]).max() < 2e-3
    # an entry equal to Lk (outside the cache) is skipped and reported, not read
    bad = idx_np.copy()
    bad[1, 0, 5] = Lk
    bad_t = torch.from_numpy(bad).cuda()
    rc = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), bad_t.data_ptr(), B, 1, Lk, 64, 128, S, g.wl.scale,
           out.data_ptr(), None, stream)
    assert rc == 0 and _status() == hs2.ERR_DEVICE_BOUNDS
    # the next call clears the word before its kernels run
    rc = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), B, 1, Lk, 64, 128, S, g.wl.scale,
           out.data_ptr(), None, stream)
    assert rc == 0 and _status() == 0
    torch.cuda.synchronize()
    assert_out_close(bf16_to_f64(out).reshape(ref["out"].shape), ref["out"], "no-alloc after a reported call")


def test_noalloc_scratch_covers_every_shape_and_refuses_invalid_ones():
    hs2, f = _entry()
    # split rows merge in distributed shared memory: only the status word is needed
    for B, Lq, S in [(1, 1, 128), (8, 1, 1152), (100, 1, 1152), (147, 1, 2048), (1, 32768, 1152)]:
        assert 0 < hs2.sparse_attn_workspace_bytes(B, Lq, 8, 64, 128, S) <= 4096
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = f(x.data_ptr(), x.data_ptr(), x.data_ptr(), i.data_ptr(), 0, 1, 8, 64, 128, 1152, 0.1, x.data_ptr(), None,
           torch.cuda.current_stream().cuda_stream)
    assert rc == hs2.ERR_INVALID_ARG
