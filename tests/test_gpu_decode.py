"""GPU parity of the decode path (one query token per sequence) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_out_close, bf16_to_f64, check_selection, to_torch_bf16

pytestmark = pytest.mark.gpu

W, K = synth.WINDOW, synth.TOPK


@pytest.fixture(scope="module")
def hs2():
    import long_context_mqa_b200 as m
    assert torch.cuda.is_available()
    return m


def _run_full(hs2, g):
    wl = g.wl
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    out, lse, idx = hs2.full_attn_select(q, k, v, scale=wl.scale, window=wl.window, topk=wl.topk)
    torch.cuda.synchronize()
    ws = hs2.cached_workspace("full")
    assert hs2.read_device_status(ws) == 0
    return q, k, v, out, lse, idx


def _check_full(g, out, lse, idx, rows=None):
    wl = g.wl
    ora = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, wl.window, wl.topk, rows=rows, want_score=True)
    sel_rows = np.arange(wl.B * wl.Lq) if rows is None else np.asarray(rows)
    gout = bf16_to_f64(out).reshape(wl.B * wl.Lq, wl.H, wl.d)[sel_rows]
    assert_out_close(gout, ora["out"], "full-attention output")
    glse = lse.double().cpu().numpy().reshape(wl.B * wl.Lq, wl.H)[sel_rows]
    assert np.abs(glse - ora["lse"]).max() < 2e-3
    gidx = idx.cpu().numpy().reshape(wl.B * wl.Lq, -1)[sel_rows]
    t_pos = wl.Lk - wl.Lq + (sel_rows % wl.Lq)
    st = check_selection(gidx, ora["idx"], ora["score"], t_pos, wl.window, wl.topk)
    assert st.ok(), st.failures
    return ora, st


@pytest.mark.parametrize("B,N", [(3, 100), (2, 1000), (2, 1152), (1, 1153), (3, 3000), (2, 20000), (1, 40000)])
def test_decode_small(hs2, B, N):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=N))
    q, k, v, out, lse, idx = _run_full(hs2, g)
    _check_full(g, out, lse, idx)


def test_decode_all_ties_prefer_lower_index(hs2):
    """K == 0 makes every score equal: the older picks must be tokens 0..topk-1."""
    B, N = 2, 3000
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=N))
    q = to_torch_bf16(g.q)
    k = torch.zeros((B, N, 128), dtype=torch.bfloat16, device="cuda")
    v = to_torch_bf16(g.v)
    out, lse, idx = hs2.full_attn_select(q, k, v)
    torch.cuda.synchronize()
    expect = np.concatenate([np.arange(K), np.arange(N - W, N)])
    for b in range(B):
        np.testing.assert_array_equal(idx[b, 0].cpu().numpy(), expect)
    np.testing.assert_allclose(lse.cpu().numpy(), np.log(N), rtol=0, atol=1e-4)


def test_decode_repeatable(hs2):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=2, Lk=9000))
    _, _, _, out1, lse1, idx1 = _run_full(hs2, g)
    out1, lse1, idx1 = out1.clone(), lse1.clone(), idx1.clone()
    _, _, _, out2, lse2, idx2 = _run_full(hs2, g)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2) and torch.equal(idx1, idx2)


@pytest.mark.parametrize("name", ["decode_32k", "decode_256k", "decode_1m"])
def test_decode_full_size(hs2, name):
    """Full configuration sizes, the launch the benchmark times; every sequence checked."""
    g = synth.SyntheticInputs(synth.WORKLOADS[name])
    q, k, v, out, lse, idx = _run_full(hs2, g)
    ora, st = _check_full(g, out, lse, idx)
    print(f"{name}: swaps {st.swaps} (max rel {st.max_swap_rel:.2e})")
    # sparse layers of the same step reuse K, V and the GPU indices
    for layer in range(g.wl.n_sparse):
        qs = g.q_sparse(layer)
        o2 = hs2.sparse_attn(to_torch_bf16(qs), k, v, idx, scale=g.wl.scale)
        torch.cuda.synchronize()
        ref = oracle.sparse_attn(qs, g.k, g.v, idx.cpu().numpy(), g.wl.scale)
        assert_out_close(bf16_to_f64(o2).reshape(ref["out"].shape), ref["out"], f"sparse layer {layer}")


def test_decode_dominant_key_outside_the_phase1_sample_is_redone_exactly(hs2):
    """Phase 1 estimates each head's logsumexp from a sample of the tiles (every 4th tile here).
    A key that head 0 prefers over all sampled keys by about 2^74 sits in an unsampled tile: its
    unnormalised probability overflows the sampled reference, the sequence is flagged, and the
    exact redo (every tile) must give the oracle's output, lse and selection."""
    B, N, j = 2, 40000, 200  # 313 tiles per sequence: phase 1 takes tiles 0, 4, 8, ...; key 200 is in tile 1
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=N))
    q0 = bf16_to_f64(to_torch_bf16(g.q[1, 0, 0]))
    k_dom = 60.0 * q0 / np.linalg.norm(q0)
    g.k[1, j] = synth.f32_to_bf16_bits(k_dom.astype(np.float32))
    q, k, v, out, lse, idx = _run_full(hs2, g)
    ora, st = _check_full(g, out, lse, idx)
    assert j in set(idx.cpu().numpy()[1, 0].tolist())


def _check_seq(g, b, n, out, lse, idx):
    """Sequence b of a ragged batch against the oracle run on that sequence alone (n tokens)."""
    wl = g.wl
    ora = oracle.full_attn_select(g.q[b:b + 1], g.k[b:b + 1, :n], g.v[b:b + 1, :n], wl.scale, wl.window, wl.topk,
                                  want_score=True)
    assert_out_close(bf16_to_f64(out[b:b + 1]).reshape(ora["out"].shape), ora["out"], f"sequence {b} (N={n})")
    assert np.abs(lse[b].double().cpu().numpy().reshape(ora["lse"].shape) - ora["lse"]).max() < 2e-3
    st = check_selection(idx[b].cpu().numpy().reshape(1, -1), ora["idx"], ora["score"], np.array([n - 1]),
                         wl.window, wl.topk)
    assert st.ok(), (b, n, st.failures)


@pytest.mark.parametrize("lens", [[40000, 777, 129, 12345, 1, 128, 1153], [300, 70000], [5000, 5000, 5000]])
def test_decode_ragged_matches_each_sequence_alone(hs2, lens):
    """Sequences of different cache lengths in one call: each equals the oracle on that sequence
    alone; rows past a sequence's length are garbage the kernels must never read (NaN here)."""
    B, Lk = len(lens), max(lens)
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    for b, n in enumerate(lens):
        k[b, n:] = float("nan")
        v[b, n:] = float("nan")
    out, lse, idx = hs2.full_attn_select_ragged(q, k, v, lens, scale=g.wl.scale)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    for b, n in enumerate(lens):
        _check_seq(g, b, n, out, lse, idx)
    # a sparse layer over the ragged selection reuses K, V and the GPU indices
    qs = g.q_sparse(0)
    o2 = hs2.sparse_attn(to_torch_bf16(qs), k, v, idx, scale=g.wl.scale)
    torch.cuda.synchronize()
    ref = oracle.sparse_attn(qs, g.k, g.v, idx.cpu().numpy(), g.wl.scale)
    assert_out_close(bf16_to_f64(o2).reshape(ref["out"].shape), ref["out"], "sparse layer over ragged selection")


def test_decode_ragged_with_equal_lengths_is_the_batched_call(hs2):
    g = synth.SyntheticInputs(synth.small("decode_32k", B=3, Lk=20000))
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    out1, lse1, idx1 = [t.clone() for t in hs2.full_attn_select(q, k, v, scale=g.wl.scale)]
    out2, lse2, idx2 = hs2.full_attn_select_ragged(q, k, v, [20000] * 3, scale=g.wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2) and torch.equal(idx1, idx2)


def test_decode_ragged_long_and_short_at_full_scale(hs2):
    """One 262,144-token sequence next to short ones: the long sequence's work spreads over most
    SMs while the short ones finish in one tile or a few."""
    lens = [262144, 3000, 131072, 200]
    B, Lk = len(lens), max(lens)
    g = synth.SyntheticInputs(synth.small("decode_256k", B=B, Lk=Lk))
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    out, lse, idx = hs2.full_attn_select_ragged(q, k, v, lens, scale=g.wl.scale)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    for b, n in enumerate(lens):
        _check_seq(g, b, n, out, lse, idx)


def _paged_layout(g, lens, seed=7, spare=5):
    """The synthetic cache of each sequence copied into randomly placed 128-token pages of shared
    pools; page tails past a sequence and spare pages hold NaN, unused table entries an id far
    outside the pool (neither may ever be read)."""
    rng = np.random.default_rng(seed)
    B, d = len(lens), g.wl.d
    tiles = [(n + 127) // 128 for n in lens]
    max_pages = max(tiles) + 2
    n_pages = sum(tiles) + spare
    perm = rng.permutation(n_pages)
    table = np.full((B, max_pages), 1 << 30, np.int32)
    k = torch.full((n_pages, 128, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    v = torch.full((n_pages, 128, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    kc, vc = to_torch_bf16(g.k), to_torch_bf16(g.v)
    nxt = 0
    for b, n in enumerate(lens):
        for i in range(tiles[b]):
            pg = int(perm[nxt]); nxt += 1
            table[b, i] = pg
            r = min(128, n - 128 * i)
            k[pg, :r] = kc[b, 128 * i:128 * i + r]
            v[pg, :r] = vc[b, 128 * i:128 * i + r]
    return k, v, torch.from_numpy(table).cuda(), max_pages


@pytest.mark.parametrize("lens", [[40000, 777, 129, 12345, 1, 128], [262144, 3000]])
def test_decode_paged_equals_ragged_contiguous(hs2, lens):
    """A paged cache gives bit-for-bit the ragged call's results on the same tokens laid out
    contiguously (same tiles, same order, same arithmetic), and so does a sparse layer."""
    B, Lk = len(lens), max(lens)
    g = synth.SyntheticInputs(synth.small("decode_32k", B=B, Lk=Lk))
    q, k, v = to_torch_bf16(g.q), to_torch_bf16(g.k), to_torch_bf16(g.v)
    ref = [t.clone() for t in hs2.full_attn_select_ragged(q, k, v, lens, scale=g.wl.scale)]
    kp, vp, table, max_pages = _paged_layout(g, lens)
    out, lse, idx = hs2.full_attn_select_paged(q, kp, vp, table, lens, scale=g.wl.scale)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("full")) == 0
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(idx, ref[2])
    qs = to_torch_bf16(g.q_sparse(0))
    o_c = hs2.sparse_attn(qs, k, v, idx, scale=g.wl.scale).clone()
    o_p = hs2.sparse_attn_paged(qs, kp, vp, table, idx, scale=g.wl.scale)
    torch.cuda.synchronize()
    assert hs2.read_device_status(hs2.cached_workspace("sparse")) == 0
    assert torch.equal(o_c, o_p)
    if B <= 6:  # and against the oracle, per sequence
        for b, n in enumerate(lens):
            _check_seq(g, b, n, out, lse, idx)


def test_decode_paged_bad_page_id_is_reported(hs2):
    lens = [3000, 700]
    g = synth.SyntheticInputs(synth.small("decode_32k", B=2, Lk=3000))
    q = to_torch_bf16(g.q)
    kp, vp, table, _ = _paged_layout(g, lens)
    table[1, 2] = kp.shape[0] + 5   # a used entry outside the pool
    ws = torch.zeros(hs2.full_attn_select_paged_workspace_bytes(lens, table.shape[1], 64, 128), dtype=torch.uint8,
                     device="cuda")
    hs2.full_attn_select_paged(q, kp, vp, table, lens, scale=g.wl.scale, workspace=ws)
    assert hs2.read_device_status(ws) == hs2.ERR_DEVICE_BOUNDS
    hs2.clear_device_status(ws)
    assert hs2.read_device_status(ws) == 0
