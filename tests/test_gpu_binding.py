"""The binding's two call paths give the same results: with every buffer given (checks in the C++
marshalling module) and with buffers allocated by the binding (checks in Python, ctypes call)."""
import numpy as np
import pytest
import torch

import synth
from parity import to_torch_bf16

pytestmark = pytest.mark.gpu


def test_marshalling_paths_agree():
    import long_context_mqa_b200 as hs2
    assert hs2._fast is not None
    wl = synth.small("decode_32k", B=3, Lk=5000)
    g = synth.SyntheticInputs(wl)
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    qs = to_torch_bf16(g.q_sparse(0))
    S = wl.window + wl.topk
    # allocated by the binding: the Python path
    out0, lse0, idx0 = hs2.full_attn_select(q, k, v, scale=wl.scale)
    sp0, splse0 = hs2.sparse_attn(qs, k, v, idx0, scale=wl.scale, want_lse=True)
    # every buffer given: the C++ path
    out1, lse1 = torch.empty_like(out0), torch.empty_like(lse0)
    idx1 = torch.empty_like(idx0)
    ws = torch.zeros(hs2.full_attn_select_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d), dtype=torch.uint8, device="cuda")
    hs2.full_attn_select(q, k, v, scale=wl.scale, out=out1, lse=lse1, idx=idx1, workspace=ws)
    sp1, splse1 = torch.empty_like(sp0), torch.empty_like(splse0)
    wss = torch.zeros(hs2.sparse_attn_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d, S), dtype=torch.uint8, device="cuda")
    hs2.sparse_attn(qs, k, v, idx1, scale=wl.scale, out=sp1, lse=splse1, workspace=wss)
    torch.cuda.synchronize()
    assert hs2.read_device_status(ws) == 0 and hs2.read_device_status(wss) == 0
    assert torch.equal(idx0, idx1)
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)
    assert torch.equal(sp0, sp1) and torch.equal(splse0, splse1)
    # argument errors on the C++ path are ValueError, like the Python path's
    with pytest.raises(ValueError):
        hs2.sparse_attn(qs, k, v, idx1[:, :, :100].contiguous().float(), scale=wl.scale, out=sp1, workspace=wss)
