"""GPU parity of the FP8 (e4m3) K/V cache path against the fp64 oracle.

The cache is the synthetic K and V rounded to e4m3 with one power-of-two scale per tensor
(``synth``); the oracle runs on its dequantised values (``oracle.e4m3_to_bf16``, the 8-bit
format decoded from its definition), which the kernels must reproduce to the usual bars: the
selection equal up to near-tie swaps, the outputs within max-abs 2e-2 and relative L2 5e-3.
"""
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


class Fp8Cache:
    """The e4m3 codes and scales of a workload's K/V, on the device, and their bf16 values."""

    def __init__(self, g):
        self.g, self.wl = g, g.wl
        (self.k8, self.ks), (self.v8, self.vs) = g.k8, g.v8
        self.k8_d = torch.from_numpy(self.k8).cuda()
        self.v8_d = torch.from_numpy(self.v8).cuda()
        self.k = oracle.e4m3_to_bf16(self.k8, self.ks)   # [B, Lk, d] bf16 bits, exact
        self.v = oracle.e4m3_to_bf16(self.v8, self.vs)


def _check_seq(c, b, n, out, lse, idx):
    """Sequence b (its first n tokens) against the oracle on that sequence alone."""
    wl, g = c.wl, c.g
    ora = oracle.full_attn_select(g.q[b:b + 1], c.k[b:b + 1, :n], c.v[b:b + 1, :n], wl.scale, wl.window, wl.topk,
                                  want_score=True)
    assert_out_close(bf16_to_f64(out[b:b + 1]).reshape(ora["out"].shape), ora["out"], f"sequence {b} (N={n})")
    assert np.abs(lse[b].double().cpu().numpy().reshape(ora["lse"].shape) - ora["lse"]).max() < 2e-3
    st = check_selection(idx[b].cpu().numpy().reshape(1, -1), ora["idx"], ora["score"], np.array([n - 1]),
                         wl.window, wl.topk)
    assert st.ok(), (b, n, st.failures)
    return st


def _check_all(c, out, lse, idx):
    wl, g = c.wl, c.g
    ora = oracle.full_attn_select(g.q, c.k, c.v, wl.scale, wl.window, wl.topk, want_score=True)
    assert_out_close(bf16_to_f64(out).reshape(ora["out"].shape), ora["out"], "full-attention output (FP8 cache)")
    assert np.abs(lse.double().cpu().numpy().reshape(ora["lse"].shape) - ora["lse"]).max() < 2e-3
    t_pos = np.full(wl.B, wl.Lk - 1)
    st = check_selection(idx.cpu().numpy().reshape(wl.B, -1), ora["idx"], ora["score"], t_pos, wl.window, wl.topk)
    assert st.ok(), st.failures
    return st


def _run(hs2, c, **kw):
    out, lse, idx = hs2.full_attn_select_fp8kv(to_torch_bf16(c.g.q), c.k8_d, c.v8_d, c.ks, c.vs, scale=c.wl.scale,
                                               window=c.wl.window, topk=c.wl.topk, **kw)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    return out, lse, idx


def test_e4m3_widening_matches_the_format(hs2):
    """The device conversions (to f16 and to bf16) of every non-NaN code against the oracle's
    decoding of the 8-bit format, bit for bit."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    yh, yb = hs2.selftest_e4m3(torch.from_numpy(codes).cuda())
    torch.cuda.synchronize()
    vals = oracle.e4m3_values()[codes]
    assert np.array_equal(yh.cpu().numpy().view(np.uint16), vals.astype(np.float16).view(np.uint16))
    assert np.array_equal(yb.cpu().numpy().view(np.uint16), oracle.e4m3_to_bf16(codes, 1.0))


@pytest.mark.parametrize("B,N", [(3, 100), (2, 1152), (1, 1153), (3, 3000), (2, 20000), (1, 40000)])
def test_fp8_decode_small(hs2, B, N):
    c = Fp8Cache(synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=N)))
    out, lse, idx = _run(hs2, c)
    _check_all(c, out, lse, idx)


def test_fp8_decode_repeatable(hs2):
    c = Fp8Cache(synth.SyntheticInputs(synth.small("decode_32k", B=2, Lk=9000)))
    r1 = [t.clone() for t in _run(hs2, c)]
    r2 = _run(hs2, c)
    assert all(torch.equal(a, b) for a, b in zip(r1, r2))


@pytest.mark.parametrize("name", ["decode_32k", "decode_256k", "decode_1m"])
def test_fp8_decode_full_size(hs2, name):
    """Full configuration sizes on the FP8 cache, the launch the benchmark's FP8 clause times,
    every sequence checked, then the four sparse layers over the same cache and the GPU indices."""
    c = Fp8Cache(synth.SyntheticInputs(synth.WORKLOADS[name]))
    out, lse, idx = _run(hs2, c)
    st = _check_all(c, out, lse, idx)
    print(f"{name} (e4m3 cache): swaps {st.swaps} (max rel {st.max_swap_rel:.2e})")
    for layer in range(c.wl.n_sparse):
        qs = c.g.q_sparse(layer)
        o2 = hs2.sparse_attn_fp8kv(to_torch_bf16(qs), c.k8_d, c.v8_d, c.ks, c.vs, idx, scale=c.wl.scale)
        torch.cuda.synchronize()
        assert hs2.read_device_status(hs2.cached_workspace("sparse")) == 0
        ref = oracle.sparse_attn(qs, c.k, c.v, idx.cpu().numpy(), c.wl.scale)
        assert_out_close(bf16_to_f64(o2).reshape(ref["out"].shape), ref["out"], f"sparse layer {layer} (FP8 cache)")


def test_fp8_decode_dominant_key_is_redone_exactly(hs2):
    """A key that head 0 prefers over every sampled key by far sits in a tile phase 1 does not
    sample: its p' passes the f16 range of P, the sequence is flagged, and the exact redo (every
    tile, p = 2^12 exp(s - lse)) must give the oracle's output, lse and selection."""
    B, N, j = 2, 40000, 200
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=N))
    c = Fp8Cache(g)
    q0 = bf16_to_f64(to_torch_bf16(g.q[1, 0, 0]))
    k_dom = 60.0 * q0 / np.linalg.norm(q0)
    kf = oracle.e4m3_values()[c.k8].astype(np.float32) * np.float32(c.ks)
    kf[1, j] = k_dom
    c.ks = synth.e4m3_scale(kf)
    c.k8 = synth.f32_to_e4m3(kf, c.ks)
    c.k8_d = torch.from_numpy(c.k8).cuda()
    c.k = oracle.e4m3_to_bf16(c.k8, c.ks)
    out, lse, idx = _run(hs2, c)
    _check_all(c, out, lse, idx)
    assert j in set(idx.cpu().numpy()[1, 0].tolist())


def _paged_fp8(c, lens, seed=7, spare=5):
    """The e4m3 cache of each sequence in randomly placed 128-token pages of shared pools;
    page tails and spare pages hold the NaN code 0x7F, unused table entries an id far outside
    the pool (neither may ever be read)."""
    rng = np.random.default_rng(seed)
    B, d = len(lens), c.wl.d
    tiles = [(n + 127) // 128 for n in lens]
    max_pages = max(tiles) + 2
    n_pages = sum(tiles) + spare
    perm = rng.permutation(n_pages)
    table = np.full((B, max_pages), 1 << 30, np.int32)
    kp = np.full((n_pages, 128, d), 0x7F, np.uint8)
    vp = np.full((n_pages, 128, d), 0x7F, np.uint8)
    nxt = 0
    for b, n in enumerate(lens):
        for i in range(tiles[b]):
            pg = int(perm[nxt]); nxt += 1
            table[b, i] = pg
            r = min(128, n - 128 * i)
            kp[pg, :r] = c.k8[b, 128 * i:128 * i + r]
            vp[pg, :r] = c.v8[b, 128 * i:128 * i + r]
    return (torch.from_numpy(kp).cuda(), torch.from_numpy(vp).cuda(), torch.from_numpy(table).cuda())


@pytest.mark.parametrize("lens", [[40000, 777, 129, 12345, 1, 128, 1153], [300, 70000]])
def test_fp8_decode_ragged_and_paged(hs2, lens):
    """Ragged lengths with NaN codes past each sequence (never read), each sequence against the
    oracle alone; the same tokens in a shuffled page pool give bit-identical results; a sparse
    layer over the selection, contiguous and paged, matches the oracle and itself."""
    B, Lk = len(lens), max(lens)
    c = Fp8Cache(synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk)))
    for b, n in enumerate(lens):
        c.k8_d[b, n:] = 0x7F
        c.v8_d[b, n:] = 0x7F
    ref = [t.clone() for t in _run(hs2, c, lens=lens)]
    for b, n in enumerate(lens):
        _check_seq(c, b, n, *ref)
    kp, vp, table = _paged_fp8(c, lens)
    q = to_torch_bf16(c.g.q)
    out, lse, idx = hs2.full_attn_select_fp8kv(q, kp, vp, c.ks, c.vs, lens=lens, page_table=table, scale=c.wl.scale)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(idx, ref[2])
    qs_bits = c.g.q_sparse(0)
    qs = to_torch_bf16(qs_bits)
    o_c = hs2.sparse_attn_fp8kv(qs, c.k8_d, c.v8_d, c.ks, c.vs, idx, scale=c.wl.scale).clone()
    o_p = hs2.sparse_attn_fp8kv(qs, kp, vp, c.ks, c.vs, idx, page_table=table, scale=c.wl.scale)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("sparse")) == 0
    assert torch.equal(o_c, o_p)
    ref_sp = oracle.sparse_attn(qs_bits, c.k, c.v, idx.cpu().numpy(), c.wl.scale)
    assert_out_close(bf16_to_f64(o_c).reshape(ref_sp["out"].shape), ref_sp["out"], "sparse layer (FP8, ragged)")


def test_fp8_sparse_prefill_rows(hs2):
    """Sparse attention of prefill rows (16 heads x 64, many query rows, the oracle's selection)
    over an FP8 cache, with lse."""
    wl = synth.small("tiny_prefill", Lq=1024, Lk=1024)
    g = synth.SyntheticInputs(wl)
    c = Fp8Cache(g)
    ora = oracle.full_attn_select(g.q, c.k, c.v, wl.scale, wl.window, wl.topk)
    idx = torch.from_numpy(ora["idx"].reshape(wl.B, wl.Lq, -1)).cuda()
    qs = g.q_sparse(0)
    out, lse = hs2.sparse_attn_fp8kv(to_torch_bf16(qs), c.k8_d, c.v8_d, c.ks, c.vs, idx, scale=wl.scale,
                                     want_lse=True)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("sparse")) == 0
    ref = oracle.sparse_attn(qs, c.k, c.v, ora["idx"].reshape(wl.B, wl.Lq, -1), wl.scale)
    assert_out_close(bf16_to_f64(out).reshape(ref["out"].shape), ref["out"], "sparse prefill rows (FP8 cache)")
    assert np.abs(lse.double().cpu().numpy().reshape(ref["lse"].shape) - ref["lse"]).max() < 2e-3


def test_fp8_rejects_bad_scales(hs2):
    c = Fp8Cache(synth.SyntheticInputs(synth.small("decode_32k", B=1, Lk=500)))
    q = to_torch_bf16(c.g.q)
    for ks in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(hs2.HS2Error):
            hs2.full_attn_select_fp8kv(q, c.k8_d, c.v8_d, ks, c.vs)


@pytest.mark.parametrize("name,kw", [("tiny_prefill", {"Lq": 1500, "Lk": 1500}),
                                     ("prefill_32k", {"B": 2, "Lq": 1100, "Lk": 1100}),
                                     ("prefill_32k", {"B": 1, "Lq": 700, "Lk": 2500}),
                                     ("prefill_32k", {"B": 2, "Lq": 1, "Lk": 3000})])
def test_fp8_prefill_and_chunks(hs2, name, kw):
    """Whole prompts, a chunk of 700 queries appended to a 1,800-token cache and a single query over
    an FP8 cache, every row against the oracle on the dequantised cache."""
    wl = synth.small(name, **kw)
    g = synth.SyntheticInputs(wl)
    c = Fp8Cache(g)
    out, lse, idx = hs2.full_attn_select_prefill_fp8kv(to_torch_bf16(g.q), c.k8_d, c.v8_d, c.ks, c.vs, scale=wl.scale,
                                                       window=wl.window, topk=wl.topk)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    rows = np.arange(wl.B * wl.Lq)
    ora = oracle.full_attn_select(g.q, c.k, c.v, wl.scale, wl.window, wl.topk, want_score=True)
    assert_out_close(bf16_to_f64(out).reshape(ora["out"].shape), ora["out"], f"{wl.name} output (FP8 cache)")
    assert np.abs(lse.double().cpu().numpy().reshape(ora["lse"].shape) - ora["lse"]).max() < 2e-3
    st = check_selection(idx.cpu().numpy().reshape(wl.B * wl.Lq, -1), ora["idx"], ora["score"],
                         wl.Lk - wl.Lq + rows % wl.Lq, wl.window, wl.topk)
    assert st.ok(), st.failures
