"""GPU parity of the HySparse (v1) variant against the fp64 oracle: the block-level selection
(hs2_full_attn_select_v1) and the gated two-branch sparse layer (hs2_sparse_attn_v1).

The selection is checked block by block (oracle.block_select on the oracle's own token scores;
swaps only between blocks whose oracle scores differ by <= 1e-5 relative), the window slots
exactly, the full layer's output and lse as for the token-level path, and the sparse layer
against oracle.sparse_attn_v1 on the GPU's own blocks with random gates.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_out_close, bf16_to_f64, check_block_selection, to_torch_bf16

pytestmark = pytest.mark.gpu

BLOCK, NBLK, W = 64, 16, 128


@pytest.fixture(scope="module")
def hs2():
    import long_context_mqa_b200 as m
    assert torch.cuda.is_available()
    return m


def _check_v1(hs2, g, k=None):
    wl = g.wl
    kb = g.k if k is None else k
    q_t, k_t, v_t = to_torch_bf16(g.q), to_torch_bf16(kb), to_torch_bf16(g.v)
    ws = torch.zeros(hs2.full_attn_select_v1_workspace_bytes(wl.B, wl.Lk, wl.H, wl.d), dtype=torch.uint8,
                     device="cuda")
    out, lse, idx = hs2.full_attn_select_v1(q_t, k_t, v_t, scale=wl.scale, workspace=ws)
    torch.cuda.synchronize()
    assert hs2.read_device_status(ws) == 0
    ora = oracle.full_attn_select(g.q, kb, g.v, wl.scale, W, NBLK * BLOCK, want_score=True)
    assert_out_close(bf16_to_f64(out).reshape(ora["out"].shape), ora["out"], "v1 full attention")
    assert np.abs(lse.double().cpu().numpy().reshape(ora["lse"].shape) - ora["lse"]).max() < 2e-3
    gi = idx.cpu().numpy().reshape(wl.B, -1)
    t = wl.Lk - 1
    swaps = 0
    for b in range(wl.B):
        toks = oracle.block_select(ora["score"][b], t, BLOCK, NBLK)
        bs = oracle.block_scores(ora["score"][b], t, BLOCK)
        st = check_block_selection(gi[b], toks, bs, t, BLOCK, NBLK, W)
        assert st.ok(), (b, st.failures)
        swaps += st.swaps
    return out, idx, swaps


@pytest.mark.parametrize("B,Lk", [(3, 5000), (2, 700), (2, 1025), (1, 1), (4, 1088), (2, 20000)])
def test_v1_selection_small(hs2, B, Lk):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    _check_v1(hs2, g)


def test_v1_all_ties_prefer_lower_blocks(hs2):
    """K = 0: every token of the row scores H / (t + 1), every full block the same: the lowest
    16 blocks are chosen (and the last, partial block scores less)."""
    g = synth.SyntheticInputs(synth.small("decode_32k", B=2, Lk=3000))
    k0 = np.zeros_like(g.k)
    _, idx, _ = _check_v1(hs2, g, k=k0)
    gi = idx.cpu().numpy().reshape(2, -1)
    assert np.array_equal(gi[:, :NBLK * BLOCK], np.tile(np.arange(NBLK * BLOCK), (2, 1)))


@pytest.mark.parametrize("name", ["decode_32k", "decode_256k"])
def test_v1_full_size(hs2, name):
    g = synth.SyntheticInputs(synth.WORKLOADS[name])
    _, _, swaps = _check_v1(hs2, g)
    print(f"{name} v1 block selection: swaps {swaps}")


def _gate(B, H, seed):
    return np.random.default_rng(seed).uniform(0.0, 1.0, size=(B, 1, H))


@pytest.mark.parametrize("B,Lk", [(3, 5000), (2, 700), (8, 40000)])
def test_v1_sparse_layer_matches_oracle(hs2, B, Lk):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    wl = g.wl
    k_t, v_t = to_torch_bf16(g.k), to_torch_bf16(g.v)
    _, _, idx = hs2.full_attn_select_v1(to_torch_bf16(g.q), k_t, v_t, scale=wl.scale)
    gi = idx.cpu().numpy()
    for layer in range(2):
        qs = g.q_sparse(layer)
        gate = _gate(B, wl.H, 10 + layer)
        gate_t = torch.from_numpy(gate.astype(np.float32)).cuda()
        ws = torch.zeros(hs2.sparse_attn_workspace_bytes(B, 1, Lk, wl.H, wl.d, idx.shape[2]), dtype=torch.uint8,
                         device="cuda")
        out = hs2.sparse_attn_v1(to_torch_bf16(qs), k_t, v_t, idx, gate_t, scale=wl.scale, workspace=ws)
        torch.cuda.synchronize()
        assert hs2.read_device_status(ws) == 0
        ref = oracle.sparse_attn_v1(qs, g.k, g.v, np.ascontiguousarray(gi[:, :, :NBLK * BLOCK]), gate, wl.scale,
                                    window=W)["out"]
        assert_out_close(bf16_to_f64(out).reshape(ref.shape), ref, f"v1 sparse layer {layer}")


def test_v1_sparse_gate_limits(hs2):
    """gate 1: plain sparse attention over the block slots; gate 0: over the window slots."""
    B, Lk = 2, 6000
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    wl = g.wl
    k_t, v_t = to_torch_bf16(g.k), to_torch_bf16(g.v)
    _, _, idx = hs2.full_attn_select_v1(to_torch_bf16(g.q), k_t, v_t, scale=wl.scale)
    q = to_torch_bf16(g.q_sparse(0))
    nbs = NBLK * BLOCK
    for gv, sl in ((1.0, slice(0, nbs)), (0.0, slice(nbs, nbs + W))):
        gate = torch.full((B, 1, wl.H), gv, dtype=torch.float32, device="cuda")
        out = hs2.sparse_attn_v1(q, k_t, v_t, idx, gate, scale=wl.scale)
        part = idx[:, :, sl].contiguous()
        ref = hs2.sparse_attn(q, k_t, v_t, part, scale=wl.scale)
        torch.cuda.synchronize()
        assert_out_close(bf16_to_f64(out), bf16_to_f64(ref), f"gate {gv}", max_abs=1e-2, rel_l2=2e-3)


def test_v1_rejects_bad_arguments(hs2):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=1, Lk=600))
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    idx = torch.zeros((1, 1, 1152), dtype=torch.int32, device="cuda")
    gate = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(hs2.HS2Error):
        hs2.sparse_attn_v1(q, k, v, idx, gate, branch=1000)  # not a multiple of 128
    with pytest.raises(hs2.HS2Error):
        hs2.full_attn_select_v1(q, k, v, block=32)           # blocks of 64 tokens only
