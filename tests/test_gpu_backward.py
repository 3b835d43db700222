"""GPU parity of the backward pass (hs2_full_attn_bwd, hs2_sparse_attn_bwd) against the fp64
oracle (oracle.attn_bwd), on the seeded workloads' inputs with a seeded N(0, 1) upstream gradient.

Tolerance (derived from the arithmetic): every MMA operand the kernels form on chip (dS, and P
for dV) is rounded to bf16 once (relative 2^-9), dQ is rounded to bf16 on output (2^-9), and
sums accumulate in fp32. Two such roundings bound the relative error of a sum of same-sign
terms by 2 * 2^-9 = 3.9e-3; dS has both signs (each row's dS sums to zero), so the bound is
stated against the norm of the whole gradient: relative L2 <= 1e-2, and every element within
2e-2 of the largest reference magnitude.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import bf16_to_f64, to_torch_bf16

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2


@pytest.fixture(scope="module")
def hs2():
    import long_context_mqa_b200 as m
    assert torch.cuda.is_available()
    return m


def assert_grad_close(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    d = gpu - ref
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.abs(d).max() / max(np.abs(ref).max(), 1e-30))
    assert rel <= GRAD_REL_L2 and mx <= GRAD_MAX_REL, f"{what}: rel-L2 {rel:.3g} (<= {GRAD_REL_L2}), max/|ref|max {mx:.3g}"
    return rel, mx


def _forward(hs2, g):
    wl = g.wl
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    out, lse, idx = hs2.full_attn_select(q, k, v, scale=wl.scale, window=wl.window, topk=wl.topk)
    return q, k, v, out, lse, idx


@pytest.mark.parametrize("name,kw", [("prefill_32k", dict(Lq=300, Lk=300)), ("prefill_32k", dict(B=2, Lq=130, Lk=130)),
                                     ("prefill_32k", dict(Lq=200, Lk=700)), ("tiny_prefill", dict(Lq=1000, Lk=1000)),
                                     ("prefill_32k", dict(Lq=1, Lk=513))])
def test_full_backward_matches_oracle(hs2, name, kw):
    g = synth.SyntheticInputs(synth.small(name, **kw))
    wl = g.wl
    q, k, v, out, lse, _ = _forward(hs2, g)
    do_bits = g.grad_out(0)
    ws = torch.zeros(hs2.attn_bwd_workspace_bytes(wl.B, wl.Lq, wl.Lk, wl.H, wl.d), dtype=torch.uint8, device="cuda")
    dq, dk, dv = hs2.full_attn_bwd(q, k, v, out, lse, to_torch_bf16(do_bits), scale=wl.scale, workspace=ws)
    torch.cuda.synchronize()
    assert hs2.read_device_status(ws) == 0
    ref = oracle.attn_bwd(g.q, g.k, g.v, do_bits, wl.scale)
    assert_grad_close(bf16_to_f64(dq).reshape(ref["dq"].shape), ref["dq"], "dQ")
    assert_grad_close(dk.double().cpu().numpy(), ref["dk"], "dK")
    assert_grad_close(dv.double().cpu().numpy(), ref["dv"], "dV")


def test_full_backward_several_tiles(hs2):
    """1,536 queries x 64 heads: 12 key tiles, 768 row tiles, items split over key-tile chunks."""
    g = synth.SyntheticInputs(synth.small("prefill_32k", Lq=1536, Lk=1536))
    wl = g.wl
    q, k, v, out, lse, _ = _forward(hs2, g)
    do_bits = g.grad_out(0)
    dq, dk, dv = hs2.full_attn_bwd(q, k, v, out, lse, to_torch_bf16(do_bits), scale=wl.scale)
    torch.cuda.synchronize()
    ref = oracle.attn_bwd(g.q, g.k, g.v, do_bits, wl.scale)
    assert_grad_close(bf16_to_f64(dq).reshape(ref["dq"].shape), ref["dq"], "dQ")
    assert_grad_close(dk.double().cpu().numpy(), ref["dk"], "dK")
    assert_grad_close(dv.double().cpu().numpy(), ref["dv"], "dV")


def test_full_backward_training_shape_sampled(hs2):
    """The training shape (L = 32,768, 64 heads, d = 128): dQ on sampled rows against the oracle,
    and two identities that hold at any size: every row's dS sums to zero, so sum_j dK_j = 0;
    every row's p sums to one, so sum_j dV_j = sum of dO over rows and heads."""
    g = synth.SyntheticInputs(synth.WORKLOADS["prefill_32k"])
    wl = g.wl
    q, k, v, out, lse, _ = _forward(hs2, g)
    do_bits = g.grad_out(0)
    do = to_torch_bf16(do_bits)
    dq, dk, dv = hs2.full_attn_bwd(q, k, v, out, lse, do, scale=wl.scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.concatenate([[0, 1, 127, 128, 4095, wl.Lq - 1], rng.choice(wl.Lq, size=58, replace=False)])
    ref = oracle.attn_bwd(g.q, g.k, g.v, do_bits, wl.scale, rows=rows, want_kv=False)
    assert_grad_close(bf16_to_f64(dq).reshape(wl.Lq, wl.H, wl.d)[rows], ref["dq"], "dQ (sampled rows)")
    dk_sum = dk.double().sum(dim=1).cpu().numpy()
    assert np.abs(dk_sum).max() <= 1e-3 * float(dk.double().abs().sum(dim=1).max())
    dv_sum = dv.double().sum(dim=1).cpu().numpy()
    do_sum = do.double().sum(dim=(1, 2)).cpu().numpy()
    np.testing.assert_allclose(dv_sum, do_sum, rtol=0, atol=1e-2 * float(np.abs(do_sum).max()))


def _random_idx(rng, B, Lq, Lk, S):
    idx = np.full((B, Lq, S), -1, np.int32)
    for b in range(B):
        for i in range(Lq):
            n = int(rng.integers(1, min(S, Lk) + 1))
            idx[b, i, :n] = np.sort(rng.choice(Lk, size=n, replace=False))
    return idx


@pytest.mark.parametrize("name,B,Lq,Lk,S", [("prefill_32k", 2, 40, 3000, 1152), ("prefill_32k", 1, 7, 900, 300),
                                             ("tiny_prefill", 1, 50, 2000, 1152)])
def test_sparse_backward_random_indices(hs2, name, B, Lq, Lk, S):
    g = synth.SyntheticInputs(synth.small(name, B=B, Lq=Lq, Lk=Lk))
    wl = g.wl
    idx = _random_idx(np.random.default_rng(Lk + S), B, Lq, Lk, S)
    qs = g.q_sparse(0)
    q, k, v = to_torch_bf16(qs), to_torch_bf16(g.k), to_torch_bf16(g.v)
    idx_t = torch.from_numpy(idx).cuda()
    out, lse = hs2.sparse_attn(q, k, v, idx_t, scale=wl.scale, want_lse=True)
    do_bits = g.grad_out(1)
    ws = torch.zeros(hs2.attn_bwd_workspace_bytes(B, Lq, Lk, wl.H, wl.d), dtype=torch.uint8, device="cuda")
    dq, dk, dv = hs2.sparse_attn_bwd(q, k, v, idx_t, out, lse, to_torch_bf16(do_bits), scale=wl.scale, workspace=ws)
    torch.cuda.synchronize()
    assert hs2.read_device_status(ws) == 0
    ref = oracle.attn_bwd(qs, g.k, g.v, do_bits, wl.scale, idx=idx)
    assert_grad_close(bf16_to_f64(dq).reshape(ref["dq"].shape), ref["dq"], "sparse dQ")
    assert_grad_close(dk.double().cpu().numpy(), ref["dk"], "sparse dK")
    assert_grad_close(dv.double().cpu().numpy(), ref["dv"], "sparse dV")


def test_sparse_backward_unsorted_indices_with_repeats(hs2):
    """Index rows in no particular order, -1 slots anywhere and a key repeated within a row (each
    slot counts once, as in the forward): the paired kernel then concatenates the two rows' lists
    instead of merging them, and must still match the oracle."""
    rng = np.random.default_rng(77)
    B, Lq, Lk, S = 1, 9, 2000, 400
    g = synth.SyntheticInputs(synth.small("prefill_32k", B=B, Lq=Lq, Lk=Lk))
    wl = g.wl
    idx = np.full((B, Lq, S), -1, np.int32)
    for i in range(Lq):
        n = int(rng.integers(50, S))
        sel = rng.choice(Lk, size=n, replace=False).astype(np.int32)
        sel[: n // 10] = sel[n // 10: 2 * (n // 10)]  # repeats
        slots = rng.choice(S, size=n, replace=False)   # -1 slots scattered among the keys
        idx[0, i, slots] = sel
    qs = g.q_sparse(0)
    q, k, v = to_torch_bf16(qs), to_torch_bf16(g.k), to_torch_bf16(g.v)
    idx_t = torch.from_numpy(idx).cuda()
    out, lse = hs2.sparse_attn(q, k, v, idx_t, scale=wl.scale, want_lse=True)
    do_bits = g.grad_out(1)
    dq, dk, dv = hs2.sparse_attn_bwd(q, k, v, idx_t, out, lse, to_torch_bf16(do_bits), scale=wl.scale)
    torch.cuda.synchronize()
    ref = oracle.attn_bwd(qs, g.k, g.v, do_bits, wl.scale, idx=idx)
    assert_grad_close(bf16_to_f64(dq).reshape(ref["dq"].shape), ref["dq"], "sparse dQ (unsorted)")
    assert_grad_close(dk.double().cpu().numpy(), ref["dk"], "sparse dK (unsorted)")
    assert_grad_close(dv.double().cpu().numpy(), ref["dv"], "sparse dV (unsorted)")


def test_block_backward_accumulates_kv_gradients(hs2):
    """A hybrid block: the full layer's selection, then a sparse layer with its own Q over the same
    K, V and indices. The two backward calls add into one pair of dK, dV buffers (KV Reuse), which
    must equal the sum of the oracle's gradients of the two layers."""
    g = synth.SyntheticInputs(synth.small("prefill_32k", Lq=700, Lk=700))
    wl = g.wl
    q, k, v, out, lse, idx = _forward(hs2, g)
    qs_bits = g.q_sparse(0)
    qs = to_torch_bf16(qs_bits)
    out1, lse1 = hs2.sparse_attn(qs, k, v, idx, scale=wl.scale, want_lse=True)
    do0, do1 = g.grad_out(0), g.grad_out(1)
    dq0, dk, dv = hs2.full_attn_bwd(q, k, v, out, lse, to_torch_bf16(do0), scale=wl.scale)
    dq1, dk, dv = hs2.sparse_attn_bwd(qs, k, v, idx, out1, lse1, to_torch_bf16(do1), scale=wl.scale, dk=dk, dv=dv)
    torch.cuda.synchronize()
    idx_np = idx.cpu().numpy()
    r0 = oracle.attn_bwd(g.q, g.k, g.v, do0, wl.scale)
    r1 = oracle.attn_bwd(qs_bits, g.k, g.v, do1, wl.scale, idx=idx_np)
    assert_grad_close(bf16_to_f64(dq0).reshape(r0["dq"].shape), r0["dq"], "full dQ")
    assert_grad_close(bf16_to_f64(dq1).reshape(r1["dq"].shape), r1["dq"], "sparse dQ")
    assert_grad_close(dk.double().cpu().numpy(), r0["dk"] + r1["dk"], "block dK")
    assert_grad_close(dv.double().cpu().numpy(), r0["dv"] + r1["dv"], "block dV")


def test_backward_rejects_bad_arguments(hs2):
    g = synth.SyntheticInputs(synth.small("prefill_32k", Lq=64, Lk=64))
    q, k, v, out, lse, _ = _forward(hs2, g)
    do = to_torch_bf16(g.grad_out(0))
    with pytest.raises(hs2.HS2Error):
        hs2.full_attn_bwd(q, k, v, out, lse, do, scale=-1.0)
    bad_ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(hs2.HS2Error):
        hs2.full_attn_bwd(q, k, v, out, lse, do, workspace=bad_ws)
