"""hs2_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.

Such callers (for example a plugin whose enqueue hook runs inside an inference runtime that
forbids device allocation there and provides no scratch buffer) use this entry point, which
keeps its scratch in a 4 KiB array inside the library instead of a caller workspace. These
tests call it through the C ABI and require the same results as hs2_sparse_attn (which is
given its own workspace), on two calls in a row, including shapes whose rows split over a
cluster; and that every supported shape's workspace fits the scratch, while an invalid shape
is refused before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

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
        torch.cuda.synchronize()
        assert_out_close(bf16_to_f64(out), bf16_to_f64(ref), f"no-alloc vs workspace entry point, call {layer}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=0, atol=2e-3)


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
