"""GPU parity of the sparse-attention layer (KV Reuse) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_out_close, bf16_to_f64, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import long_context_mqa_b200 as m
    assert torch.cuda.is_available()
    return m


def _random_idx(rng, B, Lq, Lk, S, fill_min=1):
    idx = np.full((B, Lq, S), -1, np.int32)
    for b in range(B):
        for i in range(Lq):
            n = int(rng.integers(fill_min, min(S, Lk) + 1))
            idx[b, i, :n] = np.sort(rng.choice(Lk, size=n, replace=False))
    return idx


@pytest.mark.parametrize("B,Lq,Lk,S", [(4, 1, 5000, 1152), (3, 1, 700, 1152), (2, 1, 3000, 200), (1, 5, 2000, 1152),
                                       (2, 3, 4000, 300)])
def test_sparse_random_indices_h64(hs2, B, Lq, Lk, S):
    rng = np.random.default_rng(B * 1000 + Lk + S)
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lq=Lq, Lk=Lk))
    idx = _random_idx(rng, B, Lq, Lk, S)
    qs = g.q_sparse(0)
    out, lse = hs2.sparse_attn(to_torch_bf16(qs), to_torch_bf16(g.k), to_torch_bf16(g.v),
                               torch.from_numpy(idx).cuda(), scale=g.wl.scale, want_lse=True)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("sparse")) == 0
    ref = oracle.sparse_attn(qs, g.k, g.v, idx, g.wl.scale)
    assert_out_close(bf16_to_f64(out).reshape(ref["out"].shape), ref["out"], "sparse out")
    assert np.abs(lse.double().cpu().numpy().reshape(ref["lse"].shape) - ref["lse"]).max() < 2e-3


def test_sparse_tiny_config_h16_d64(hs2):
    """The tiny prefill shape (16 heads, head_dim 64): oracle selection, every query row."""
    wl = synth.small("tiny_prefill", Lq=600, Lk=600)
    g = synth.SyntheticInputs(wl)
    full = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, 128, 1024)
    idx = full["idx"].reshape(1, wl.Lq, -1)
    qs = g.q_sparse(0)
    out = hs2.sparse_attn(to_torch_bf16(qs), to_torch_bf16(g.k), to_torch_bf16(g.v), torch.from_numpy(idx).cuda(),
                          scale=wl.scale)
    torch.cuda.synchronize()
    ref = oracle.sparse_attn(qs, g.k, g.v, idx, wl.scale)
    assert_out_close(bf16_to_f64(out).reshape(ref["out"].shape), ref["out"], "sparse out (16 heads, d=64)")


def test_sparse_bad_index_is_reported(hs2):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=1, Lk=500))
    idx = np.full((1, 1, 256), -1, np.int32)
    idx[0, 0, :10] = np.arange(10)
    idx[0, 0, 10] = 500  # == Lk: out of range
    ws = torch.zeros(hs2.sparse_attn_workspace_bytes(1, 1, 500, 64, 128, 256), dtype=torch.uint8, device="cuda")
    hs2.sparse_attn(to_torch_bf16(g.q_sparse(0)), to_torch_bf16(g.k), to_torch_bf16(g.v),
                    torch.from_numpy(idx).cuda(), workspace=ws)
    assert hs2.read_device_status(ws) == hs2.ERR_DEVICE_BOUNDS
    hs2.clear_device_status(ws)
    assert hs2.read_device_status(ws) == 0


def test_bounded_wait_reports_timeout(hs2):
    """A wait on a barrier nothing completes gives up, reports, and leaves the context usable."""
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    hs2.selftest_wait_timeout(ws, 20_000_000)
    assert hs2.read_device_status(ws) == hs2.ERR_DEVICE_TIMEOUT
    x = torch.ones(1000, device="cuda")
    assert float((x * 2).sum()) == 2000.0


@pytest.mark.parametrize("B,Lq,Lk,sorted_lists", [(1, 301, 3000, True), (1, 301, 3000, False), (2, 150, 2500, True)])
def test_sparse_many_rows(hs2, B, Lq, Lk, sorted_lists):
    """Many query rows (at least one per SM: one CTA per row, no split): ascending lists with -1
    tails (the full layer's output, whose all-invalid tiles are skipped) and unsorted lists with
    repeats and -1 slots anywhere, two sequences, a row that selected nothing (zeros), against the
    oracle."""
    rng = np.random.default_rng(31 + sorted_lists + B)
    S = 1152
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lq=Lq, Lk=Lk))
    if sorted_lists:
        idx = _random_idx(rng, B, Lq, Lk, S)
    else:
        idx = np.full((B, Lq, S), -1, np.int32)
        for b in range(B):
            for i in range(Lq):
                n = int(rng.integers(1, S))
                sel = rng.choice(Lk, size=n, replace=False).astype(np.int32)
                sel[: n // 8] = sel[n // 8: 2 * (n // 8)]
                idx[b, i, rng.choice(S, size=n, replace=False)] = sel
    idx[0, 7, :] = -1
    qs = g.q_sparse(0)
    ws = torch.zeros(hs2.sparse_attn_workspace_bytes(B, Lq, Lk, 64, 128, S), dtype=torch.uint8, device="cuda")
    out, lse = hs2.sparse_attn(to_torch_bf16(qs), to_torch_bf16(g.k), to_torch_bf16(g.v),
                               torch.from_numpy(idx).cuda(), scale=g.wl.scale, want_lse=True, workspace=ws)
    torch.cuda.synchronize()
    assert hs2.read_device_status(ws) == 0
    # the oracle defines no result for an empty selection; the kernel writes zeros there
    rows = np.array([r for r in range(B * Lq) if r != 7], dtype=np.int64)
    ref = oracle.sparse_attn(qs, g.k, g.v, idx, g.wl.scale, rows=rows)
    o = bf16_to_f64(out).reshape(B * Lq, 64, 128)
    assert np.all(o[7] == 0.0)
    assert_out_close(o[rows], ref["out"], "sparse out (paired rows)")
    assert np.abs(lse.double().cpu().numpy().reshape(B * Lq, 64)[rows] - ref["lse"]).max() < 2e-3
