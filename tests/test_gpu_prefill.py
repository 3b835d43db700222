"""GPU parity of the prefill path (Lq == Lk, and chunks Lq < Lk appended to a cache) and of the KV
Bridging GEMM against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_out_close, bf16_to_f64, check_selection, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import long_context_mqa_b200 as m
    assert torch.cuda.is_available()
    return m


def _prefill(hs2, g):
    wl = g.wl
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    out, lse, idx = hs2.full_attn_select(q, k, v, scale=wl.scale, window=wl.window, topk=wl.topk)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    return q, k, v, out, lse, idx


def _check(g, out, lse, idx, rows):
    wl = g.wl
    rows = np.asarray(rows, np.int64)
    ora = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, wl.window, wl.topk, rows=rows, want_score=True)
    gout = bf16_to_f64(out).reshape(wl.B * wl.Lq, wl.H, wl.d)[rows]
    assert_out_close(gout, ora["out"], "prefill attention output")
    glse = lse.double().cpu().numpy().reshape(wl.B * wl.Lq, wl.H)[rows]
    assert np.abs(glse - ora["lse"]).max() < 2e-3
    gidx = idx.cpu().numpy().reshape(wl.B * wl.Lq, -1)[rows]
    st = check_selection(gidx, ora["idx"], ora["score"], wl.Lk - wl.Lq + rows % wl.Lq, wl.window, wl.topk)
    assert st.ok(), st.failures
    return st


@pytest.mark.parametrize("B,L,W,K", [(1, 300, 128, 1024), (2, 1001, 128, 1024), (1, 1700, 128, 1024),
                                     (1, 3000, 128, 1024), (2, 2500, 64, 256), (1, 1234, 16, 40)])
def test_prefill_h64_all_rows(hs2, B, L, W, K):
    wl = synth.small("prefill_32k", B=B, Lq=L, Lk=L, window=W, topk=K)
    g = synth.SyntheticInputs(wl)
    _, _, _, out, lse, idx = _prefill(hs2, g)
    _check(g, out, lse, idx, np.arange(B * L))


def test_prefill_tiny_config_all_rows(hs2):
    """The tiny configuration: B1, L2048, 16 heads, head_dim 64, scale 1/8; every query row."""
    g = synth.SyntheticInputs(synth.WORKLOADS["tiny_prefill"])
    q, k, v, out, lse, idx = _prefill(hs2, g)
    _check(g, out, lse, idx, np.arange(2048))
    qs = g.q_sparse(0)
    o2 = hs2.sparse_attn(to_torch_bf16(qs), k, v, idx, scale=g.wl.scale)
    torch.cuda.synchronize()
    ref = oracle.sparse_attn(qs, g.k, g.v, idx.cpu().numpy(), g.wl.scale)
    assert_out_close(bf16_to_f64(o2).reshape(ref["out"].shape), ref["out"], "tiny sparse layer")


def test_prefill_tiny_ragged_h16(hs2):
    wl = synth.small("tiny_prefill", Lq=999, Lk=999)
    g = synth.SyntheticInputs(wl)
    _, _, _, out, lse, idx = _prefill(hs2, g)
    _check(g, out, lse, idx, np.arange(999))


def _stratified_rows(L, n, seed):
    rng = np.random.default_rng(seed)
    small = np.arange(0, min(L, 1152), 7)
    rest = rng.choice(np.arange(1152, L), size=max(0, n - len(small) - 1), replace=False) if L > 1152 else []
    return np.unique(np.concatenate([small, rest, [L - 1]]).astype(np.int64))


def test_prefill_full_size_sampled(hs2):
    """prefill_32k at full size (the launch the benchmark times), >= 512 stratified rows, plus its 4 sparse layers."""
    g = synth.SyntheticInputs(synth.WORKLOADS["prefill_32k"])
    wl = g.wl
    q, k, v, out, lse, idx = _prefill(hs2, g)
    rows = _stratified_rows(wl.Lq, 512, 1)
    st = _check(g, out, lse, idx, rows)
    print(f"prefill_32k: {len(rows)} rows, swaps {st.swaps} (max rel {st.max_swap_rel:.2e})")
    idx_np = idx.cpu().numpy()
    for layer in range(wl.n_sparse):
        qs = g.q_sparse(layer)
        o2 = hs2.sparse_attn(to_torch_bf16(qs), k, v, idx, scale=wl.scale)
        torch.cuda.synchronize()
        ref = oracle.sparse_attn(qs, g.k, g.v, idx_np, wl.scale, rows=rows)
        assert_out_close(bf16_to_f64(o2).reshape(wl.Lq, wl.H, wl.d)[rows], ref["out"], f"sparse layer {layer}")


def _bridge_check(gpu, ref):
    """bf16 output of an fp32-accumulated dot product: |err| <= 2^-8 |ref| + 1e-3."""
    gpu = np.asarray(gpu, np.float64)
    bound = np.abs(ref) * 2.0 ** -8 + 1e-3
    bad = np.abs(gpu - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements outside the bf16 rounding bound; max err {np.abs(gpu - ref).max():.3g}"


@pytest.mark.parametrize("T,hidden,n,d", [(300, 256, 2, 128), (1000, 2048, 4, 128), (129, 512, 4, 64)])
def test_bridge_small(hs2, T, hidden, n, d):
    rng = np.random.default_rng(T + hidden)
    h = synth.f32_to_bf16_bits(rng.standard_normal((T, hidden)).astype(np.float32))
    w = synth.f32_to_bf16_bits((rng.standard_normal((n, 2, hidden, d)) * 0.02).astype(np.float32))
    kv = hs2.bridge_kv_proj(to_torch_bf16(h), to_torch_bf16(w))
    torch.cuda.synchronize()
    _bridge_check(bf16_to_f64(kv), oracle.bridge_kv_proj(h, w))


def test_bridge_full_size_sampled(hs2):
    g = synth.SyntheticInputs(synth.WORKLOADS["prefill_32k"])
    wl = g.wl
    kv = hs2.bridge_kv_proj(to_torch_bf16(g.bridge_h), to_torch_bf16(g.bridge_w))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, 200), np.random.default_rng(3).choice(wl.bridge_T, 300, replace=False),
                                     [wl.bridge_T - 1]]))
    ref = oracle.bridge_kv_proj(g.bridge_h, g.bridge_w, rows=rows)
    _bridge_check(bf16_to_f64(kv)[:, :, rows], ref)


@pytest.mark.parametrize("B,Lq,Lk", [(1, 700, 3000), (2, 256, 1500), (1, 2, 5000), (1, 1299, 1300), (2, 129, 1152)])
def test_chunked_prefill_h64_all_rows(hs2, B, Lq, Lk):
    """A chunk of Lq queries appended to a cache of Lk - Lq tokens: query i at position Lk - Lq + i,
    every row against the oracle, and a sparse layer over the chunk's selection."""
    wl = synth.small("prefill_32k", B=B, Lq=Lq, Lk=Lk)
    g = synth.SyntheticInputs(wl)
    q, k, v, out, lse, idx = _prefill(hs2, g)
    _check(g, out, lse, idx, np.arange(B * Lq))
    qs = g.q_sparse(0)
    o2 = hs2.sparse_attn(to_torch_bf16(qs), k, v, idx, scale=wl.scale)
    torch.cuda.synchronize()
    ref = oracle.sparse_attn(qs, g.k, g.v, idx.cpu().numpy(), wl.scale)
    assert_out_close(bf16_to_f64(o2).reshape(ref["out"].shape), ref["out"], "sparse layer over a chunk")


@pytest.mark.parametrize("Lq", [300, 1])
def test_chunked_prefill_tiny_config(hs2, Lq):
    """16 heads, head_dim 64: a chunk (and a single query, which these shapes run on the prefill
    kernels) against a 2048-token cache."""
    wl = synth.small("tiny_prefill", Lq=Lq, Lk=2048)
    g = synth.SyntheticInputs(wl)
    _, _, _, out, lse, idx = _prefill(hs2, g)
    _check(g, out, lse, idx, np.arange(Lq))
