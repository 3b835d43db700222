"""Pins of the fp64 oracle against things other than itself (CPU only).

Each check is chosen so that a plausible slip in the oracle (a wrong causal bound, a
dropped head, a window off by one, a reversed tie rule, a transposed weight, log2 instead
of ln) fails at least one of them:

* library routines in special cases: torch scaled_dot_product_attention (fp64, explicit
  mask), torch.softmax, numpy matmul;
* closed forms: all-zero keys, a two-key row, constant values;
* invariants the selection rule fixes: forced window, uniqueness, causality, the count
  min(t+1, window+topk), the probability mass sum_j score(t, j) = H;
* brute force: the chosen older tokens maximise the summed score over all subsets of the
  same size (tiny rows), with scores from an independent torch computation.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import f32_to_bf16_bits, bf16_bits_to_f32


def _rand_bf16(rng, shape, std=1.0):
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _t64(bits):
    return torch.from_numpy(bf16_bits_to_f32(bits).astype(np.float64))


def _causal_mask(Lq, Lk):
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    return j <= (Lk - Lq + i)


def _torch_dense(q, k, v, scale):
    """Reference by torch SDPA (fp64): q [B,Lq,H,d], k/v [B,Lk,d] -> out [B,Lq,H,d]."""
    Q = _t64(q).permute(0, 2, 1, 3)                       # B,H,Lq,d
    K = _t64(k)[:, None].expand(-1, q.shape[2], -1, -1)   # B,H,Lk,d
    V = _t64(v)[:, None].expand(-1, q.shape[2], -1, -1)
    m = _causal_mask(q.shape[1], k.shape[1])
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def _torch_probs(q, k, scale):
    """torch.softmax probabilities [B,H,Lq,Lk] with the causal mask (fp64)."""
    Q = _t64(q).permute(0, 2, 1, 3)
    K = _t64(k)[:, None]
    s = scale * (Q @ K.transpose(-1, -2))
    s = s.masked_fill(~_causal_mask(q.shape[1], k.shape[1]), float("-inf"))
    return torch.softmax(s, dim=-1).numpy()


@pytest.mark.parametrize("B,Lq,Lk,H,d", [(2, 37, 37, 3, 8), (1, 5, 41, 4, 16), (3, 1, 29, 2, 8)])
def test_attention_matches_torch_sdpa(B, Lq, Lk, H, d):
    rng = np.random.default_rng(1)
    q, k, v = _rand_bf16(rng, (B, Lq, H, d)), _rand_bf16(rng, (B, Lk, d)), _rand_bf16(rng, (B, Lk, d))
    scale = 1.0 / math.sqrt(d)
    r = oracle.full_attn_select(q, k, v, scale, 4, 6)
    ref = _torch_dense(q, k, v, scale).reshape(B * Lq, H, d)
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)


def test_closed_form_zero_keys():
    """K == 0: every logit is 0, so p = 1/(t+1), lse = ln(t+1), out = mean(v_0..v_t)."""
    rng = np.random.default_rng(2)
    B, L, H, d = 1, 20, 3, 8
    q = _rand_bf16(rng, (B, L, H, d))
    k = np.zeros((B, L, d), np.uint16)
    v = _rand_bf16(rng, (B, L, d))
    r = oracle.full_attn_select(q, k, v, 0.3, 4, 5, want_score=True)
    vf = bf16_bits_to_f32(v).astype(np.float64)[0]
    for t in range(L):
        np.testing.assert_allclose(r["lse"][t], math.log(t + 1), atol=1e-13)
        np.testing.assert_allclose(r["out"][t], np.broadcast_to(vf[: t + 1].mean(0), (H, d)), atol=1e-13)
        np.testing.assert_allclose(r["score"][t, : t + 1], H / (t + 1), atol=1e-13)
        # all scores tie -> lower indices win: the older picks are 0..min(k, n_old)-1
        n_old = max(0, t - 4 + 1)
        picks = sorted(set(r["idx"][t][r["idx"][t] >= 0]) - set(range(max(0, t - 3), t + 1)))
        assert picks == list(range(min(5, n_old)))


def test_closed_form_two_keys():
    """One head, q = e0, keys a*e0 and b*e0: lse = ln(exp(s a) + exp(s b)) at t = 1."""
    d = 8
    a, b, c = 1.5, -0.75, 2.0
    q = np.zeros((1, 2, 1, d), np.float32); q[0, :, 0, 0] = 1.0
    k = np.zeros((1, 2, d), np.float32); k[0, 0, 0] = a; k[0, 1, 0] = b
    v = np.zeros((1, 2, d), np.float32); v[0, 0, :] = 1.0; v[0, 1, :] = c
    s = 0.5
    r = oracle.full_attn_select(f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v), s, 1, 1)
    lse1 = math.log(math.exp(s * a) + math.exp(s * b))
    assert abs(r["lse"][1, 0] - lse1) < 1e-14
    assert abs(r["lse"][0, 0] - s * a) < 1e-15
    p0 = math.exp(s * a - lse1)
    np.testing.assert_allclose(r["out"][1, 0], p0 * 1.0 + (1 - p0) * c, atol=1e-14)


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(3)
    B, L, H, d = 2, 33, 4, 8
    q, k = _rand_bf16(rng, (B, L, H, d)), _rand_bf16(rng, (B, L, d))
    v = f32_to_bf16_bits(np.full((B, L, d), 0.625, np.float32))
    r = oracle.full_attn_select(q, k, v, 0.35, 4, 4)
    np.testing.assert_allclose(r["out"], 0.625, atol=1e-13)


def test_score_mass_and_softmax_probabilities():
    """score(t, j) equals torch's softmax summed over heads; its row mass is H."""
    rng = np.random.default_rng(4)
    B, L, H, d = 2, 24, 5, 16
    q, k, v = _rand_bf16(rng, (B, L, H, d)), _rand_bf16(rng, (B, L, d)), _rand_bf16(rng, (B, L, d))
    r = oracle.full_attn_select(q, k, v, 0.25, 4, 6, want_score=True)
    p = _torch_probs(q, k, 0.25)                  # B,H,L,L
    ref = p.sum(1).reshape(B * L, L)
    np.testing.assert_allclose(r["score"], ref, atol=1e-13)
    np.testing.assert_allclose(r["score"].sum(1), H, atol=1e-12)


def test_single_head_ranking_equals_logit_ranking():
    """H = 1: softmax is monotone, so the older picks are the top logits (numpy argsort)."""
    rng = np.random.default_rng(5)
    L, d, W, K = 60, 16, 8, 10
    q, k, v = _rand_bf16(rng, (1, L, 1, d)), _rand_bf16(rng, (1, L, d)), _rand_bf16(rng, (1, L, d))
    r = oracle.full_attn_select(q, k, v, 0.2, W, K)
    qf = bf16_bits_to_f32(q)[0, :, 0].astype(np.float64)
    kf = bf16_bits_to_f32(k)[0].astype(np.float64)
    for t in range(L):
        n_old = t - W + 1
        sel = set(r["idx"][t][r["idx"][t] >= 0].tolist())
        if n_old <= 0:
            assert sel == set(range(t + 1))
            continue
        logit = kf[:n_old] @ qf[t]
        order = np.lexsort((np.arange(n_old), -logit))[: min(K, n_old)]
        assert sel == set(order.tolist()) | set(range(t - W + 1, t + 1))


def test_planted_direction_ranking():
    """H = 1, q = u and k_j = alpha_j u: the picks are the tokens with the largest alpha."""
    d, L, W, K = 8, 30, 4, 5
    alpha = np.array([((j * 7) % 30) / 8.0 - 1.5 for j in range(L)], np.float32)  # distinct, bf16-exact
    u = np.zeros(d, np.float32); u[3] = 1.0
    q = np.broadcast_to(u, (1, L, 1, d)).copy()
    k = (alpha[:, None] * u[None, :])[None]
    v = np.zeros((1, L, d), np.float32)
    r = oracle.full_attn_select(f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v), 1.0, W, K)
    t = L - 1
    n_old = t - W + 1
    expect = set(np.argsort(-alpha[:n_old], kind="stable")[:K].tolist()) | set(range(t - W + 1, t + 1))
    assert set(r["idx"][t][r["idx"][t] >= 0].tolist()) == expect


@pytest.mark.parametrize("W,K", [(4, 1), (4, 3), (4, 8), (1, 2), (0, 3)])
def test_selection_brute_force_subsets(W, K):
    """Tiny rows: the older picks maximise the summed (torch) score over all same-size subsets."""
    rng = np.random.default_rng(10 + W * 10 + K)
    B, L, H, d = 1, 12, 3, 8
    q, k, v = _rand_bf16(rng, (B, L, H, d)), _rand_bf16(rng, (B, L, d)), _rand_bf16(rng, (B, L, d))
    r = oracle.full_attn_select(q, k, v, 0.4, W, K)
    sc = _torch_probs(q, k, 0.4).sum(1)[0]        # [L, L]
    for t in range(L):
        n_old = t - W + 1
        sel = set(r["idx"][t][r["idx"][t] >= 0].tolist())
        window = set(range(max(0, t - W + 1), t + 1))
        assert window <= sel
        older = sorted(sel - window)
        m = min(K, max(0, n_old))
        assert len(older) == m
        if m == 0:
            continue
        best = max(itertools.combinations(range(n_old), m), key=lambda s: sum(sc[t, j] for j in s))
        assert older == sorted(best)


def test_selection_invariants_on_planted_workload():
    wl = synth.small("tiny_prefill", Lq=300, Lk=300)
    g = synth.SyntheticInputs(wl)
    W, K = 32, 64
    r = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, W, K, want_score=True)
    S = W + K
    assert r["idx"].shape == (300, S)
    for t in range(300):
        row = r["idx"][t]
        valid = row[row >= 0]
        assert len(valid) == min(t + 1, S)
        assert (row[len(valid):] == -1).all()
        assert (np.diff(valid) > 0).all()                       # ascending, unique
        assert valid.max() <= t and valid.min() >= 0            # causal
        assert set(range(max(0, t - W + 1), t + 1)) <= set(valid.tolist())
        # every older pick scores at least as high as every older non-pick
        older = [j for j in valid if j <= t - W]
        rest = sorted(set(range(max(0, t - W + 1))) - set(older))
        if older and rest:
            assert r["score"][t, older].min() >= r["score"][t, rest].max()
    np.testing.assert_allclose(r["score"].sum(1), wl.H, atol=1e-11)


def test_sparse_equals_dense_when_everything_fits():
    """With window + topk >= t + 1 the selection is the whole causal row, so sparse == dense."""
    rng = np.random.default_rng(6)
    B, L, H, d = 2, 20, 3, 8
    q, k, v = _rand_bf16(rng, (B, L, H, d)), _rand_bf16(rng, (B, L, d)), _rand_bf16(rng, (B, L, d))
    q2 = _rand_bf16(rng, (B, L, H, d))
    full = oracle.full_attn_select(q, k, v, 0.3, 8, 12)
    idx = full["idx"].reshape(B, L, 20)
    sp = oracle.sparse_attn(q2, k, v, idx, 0.3)
    np.testing.assert_allclose(sp["out"], _torch_dense(q2, k, v, 0.3).reshape(B * L, H, d), atol=1e-12)


def test_sparse_matches_sdpa_with_index_mask():
    rng = np.random.default_rng(7)
    B, Lq, Lk, H, d, S = 2, 6, 50, 4, 16, 9
    q, k, v = _rand_bf16(rng, (B, Lq, H, d)), _rand_bf16(rng, (B, Lk, d)), _rand_bf16(rng, (B, Lk, d))
    idx = np.full((B, Lq, S), -1, np.int32)
    for b in range(B):
        for i in range(Lq):
            n = rng.integers(1, S + 1)
            idx[b, i, :n] = rng.choice(Lk, size=n, replace=False)
            rng.shuffle(idx[b, i])
    sp = oracle.sparse_attn(q, k, v, idx, 0.25)
    mask = torch.zeros(B, 1, Lq, Lk, dtype=torch.bool)
    for b in range(B):
        for i in range(Lq):
            for j in idx[b, i]:
                if j >= 0:
                    mask[b, 0, i, j] = True
    Q = _t64(q).permute(0, 2, 1, 3)
    K = _t64(k)[:, None].expand(-1, H, -1, -1)
    V = _t64(v)[:, None].expand(-1, H, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=0.25)
    np.testing.assert_allclose(sp["out"], ref.permute(0, 2, 1, 3).reshape(B * Lq, H, d).numpy(), atol=1e-12)


def test_sparse_rejects_bad_indices():
    rng = np.random.default_rng(8)
    q, k, v = _rand_bf16(rng, (1, 2, 2, 8)), _rand_bf16(rng, (1, 10, 8)), _rand_bf16(rng, (1, 10, 8))
    idx = np.full((1, 2, 4), -1, np.int32)
    idx[0, 0, 0] = 3
    with pytest.raises(RuntimeError):
        oracle.sparse_attn(q, k, v, idx, 0.3)          # row 1 has no valid index
    idx[0, 1, 0] = 10
    with pytest.raises(RuntimeError):
        oracle.sparse_attn(q, k, v, idx, 0.3)          # out of range


@pytest.mark.parametrize("T,hidden,n,d", [(7, 24, 2, 8), (33, 64, 4, 16), (5, 2048, 1, 128)])
def test_bridge_matches_numpy_matmul(T, hidden, n, d):
    rng = np.random.default_rng(9)
    h = _rand_bf16(rng, (T, hidden))
    w = _rand_bf16(rng, (n, 2, hidden, d), 0.02)
    kv = oracle.bridge_kv_proj(h, w)
    hf = bf16_bits_to_f32(h).astype(np.float64)
    wf = bf16_bits_to_f32(w).astype(np.float64)
    for layer in range(n):
        for kvi in range(2):
            np.testing.assert_allclose(kv[layer, kvi], hf @ wf[layer, kvi], rtol=1e-13, atol=1e-13)
    rows = [T - 1, 0]
    np.testing.assert_array_equal(oracle.bridge_kv_proj(h, w, rows=rows), kv[:, :, rows])


def test_row_sampling_matches_full_run():
    wl = synth.small("decode_32k", B=3, Lk=500, H=4, d=16)
    g = synth.SyntheticInputs(wl)
    full = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, 16, 32, want_score=True)
    part = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, 16, 32, rows=[2, 0], want_score=True)
    for key in ("out", "lse", "idx", "score"):
        np.testing.assert_array_equal(part[key], full[key][[2, 0]])


# ---------------------------------------------------------------------------------------------
# FP8 (e4m3) cache: the oracle's decoder and the input generator's encoder
# ---------------------------------------------------------------------------------------------
def test_e4m3_decoder_matches_torch_for_every_code():
    """The oracle's decoder of the 8-bit format against torch's float8_e4m3fn conversion."""
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    val = oracle.e4m3_values()
    assert np.array_equal(np.isnan(val), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(val[ok], ref[ok])


def test_e4m3_closed_forms():
    val = oracle.e4m3_values()
    assert val[0x38] == 1.0 and val[0xB8] == -1.0          # 0 0111 000: 2^(7-7)
    assert val[0x7E] == 448.0                              # largest finite: 2^8 * 1.75
    assert val[0x01] == 2.0 ** -9 and val[0x07] == 7 * 2.0 ** -9   # subnormals m/8 * 2^-6
    assert val[0x08] == 2.0 ** -6                          # smallest normal
    assert val[0x00] == 0.0 and val[0x80] == 0.0 and np.signbit(val[0x80])
    assert np.isnan(val[0x7F]) and np.isnan(val[0xFF])
    assert np.all(np.diff(val[:0x7F]) > 0)                 # codes 0..126 increase strictly


def test_e4m3_encoder_matches_torch():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(100000) * 40.0, rng.standard_normal(1000) * 0.01,
                        # ties between neighbouring codes go to the even code
                        [2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875, 448.0, -448.0, 0.0, 2.0 ** -6 * (1 - 1 / 16)]])
    x = x.astype(np.float32)
    for sc in (1.0, 2.0 ** -6):
        got = synth.f32_to_e4m3(x * np.float32(sc), sc)
        ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got, ref)
    with pytest.raises(ValueError):
        synth.f32_to_e4m3(np.array([449.0], np.float32), 1.0)


def test_e4m3_scale_and_dequantisation():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((3, 50, 8)) * 3).astype(np.float32)
    sc = synth.e4m3_scale(x)
    assert np.max(np.abs(x)) / sc <= 448.0 < 2 * np.max(np.abs(x)) / sc
    codes = synth.f32_to_e4m3(x, sc)
    deq = bf16_bits_to_f32(oracle.e4m3_to_bf16(codes, sc)).astype(np.float64)
    ref = torch.from_numpy(codes.reshape(-1)).view(torch.float8_e4m3fn).double().numpy().reshape(x.shape) * sc
    assert np.array_equal(deq, ref)
    # nearest code: the error is at most half a step (relative 2^-4 for normals, 2^-10 * sc below)
    err = np.abs(deq - x)
    assert np.all(err <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * sc) + 1e-12)
    with pytest.raises(ValueError):
        oracle.e4m3_to_bf16(codes, 0.3)


def test_attention_on_e4m3_cache_matches_torch_sdpa():
    """Attention over a dequantised e4m3 cache (through the bf16 view) against torch SDPA on
    torch's own decoding of the same codes."""
    rng = np.random.default_rng(13)
    B, Lq, Lk, H, d = 2, 1, 45, 4, 16
    q = _rand_bf16(rng, (B, Lq, H, d))
    kf = (rng.standard_normal((B, Lk, d)) * 2).astype(np.float32)
    vf = rng.standard_normal((B, Lk, d)).astype(np.float32)
    ks, vs = synth.e4m3_scale(kf), synth.e4m3_scale(vf)
    k8, v8 = synth.f32_to_e4m3(kf, ks), synth.f32_to_e4m3(vf, vs)
    kb, vb = oracle.e4m3_to_bf16(k8, ks), oracle.e4m3_to_bf16(v8, vs)
    r = oracle.full_attn_select(q, kb, vb, 0.25, 4, 8)
    dec = lambda c, s: torch.from_numpy(c.reshape(-1)).view(torch.float8_e4m3fn).double().reshape(c.shape) * s
    Q = _t64(q).permute(0, 2, 1, 3)
    K = dec(k8, ks)[:, None].expand(-1, H, -1, -1)
    V = dec(v8, vs)[:, None].expand(-1, H, -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=0.25).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(r["out"], o.reshape(B * Lq, H, d), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# HySparse (v1) block selection and gated window fusion
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("t,block,nb", [(40, 4, 3), (33, 5, 2), (23, 3, 4)])
def test_block_select_brute_force(t, block, nb):
    """The chosen blocks maximise the total score of their tokens at or before t over every set
    of the same size, and among equal totals the lexicographically lowest set wins."""
    rng = np.random.default_rng(t)
    # quantised scores so that equal block totals (ties) occur
    score = rng.integers(0, 4, size=t + 1).astype(np.float64)
    got = oracle.block_select(score, t, block=block, n_blocks=nb)
    blocks = range(t // block + 1)
    total = lambda S: sum(score[j * block:min((j + 1) * block, t + 1)].sum() for j in S)
    best = max(itertools.combinations(blocks, nb), key=lambda S: (total(S), [-j for j in S]))
    want = np.concatenate([np.arange(j * block, min((j + 1) * block, t + 1)) for j in sorted(best)])
    assert np.array_equal(got, want)


def test_block_select_closed_forms():
    # equal scores: the lowest blocks; at most n_blocks blocks: every token 0..t
    assert np.array_equal(oracle.block_select(np.ones(2000), 1999), np.arange(16 * 64))
    assert np.array_equal(oracle.block_select(np.ones(1000), 700), np.arange(701))
    # a block past t never competes; the partial block at t counts only its tokens <= t
    s = np.zeros(2000); s[1990:] = 100.0; s[0] = 1.0
    got = oracle.block_select(s, 1500, block=64, n_blocks=1)
    assert np.array_equal(got, np.arange(64))


def test_gated_window_fusion_reduces_to_its_branches():
    """gate 1: plain attention over the blocks' tokens; gate 0: the window branch, which for a
    query with fewer than `window` tokens before it is dense causal attention (torch SDPA)."""
    rng = np.random.default_rng(21)
    B, Lq, Lk, H, d = 1, 3, 90, 2, 8
    q, k, v = _rand_bf16(rng, (B, Lq, H, d)), _rand_bf16(rng, (B, Lk, d)), _rand_bf16(rng, (B, Lk, d))
    idx = np.full((B, Lq, 40), -1, np.int32)
    for i in range(Lq):
        sel = rng.choice(Lk - Lq + i + 1, size=40, replace=False)
        idx[0, i] = np.sort(sel)
    one = oracle.sparse_attn_v1(q, k, v, idx, np.ones((B, Lq, H)), 0.3, window=128)["out"]
    np.testing.assert_allclose(one, oracle.sparse_attn(q, k, v, idx, 0.3)["out"], rtol=0, atol=1e-13)
    zero = oracle.sparse_attn_v1(q, k, v, idx, np.zeros((B, Lq, H)), 0.3, window=128)["out"]
    np.testing.assert_allclose(zero, _torch_dense(q, k, v, 0.3).reshape(B * Lq, H, d), rtol=0, atol=1e-12)
    half = oracle.sparse_attn_v1(q, k, v, idx, np.full((B, Lq, H), 0.25), 0.3, window=128)["out"]
    np.testing.assert_allclose(half, 0.25 * one + 0.75 * zero, rtol=0, atol=1e-13)


def test_e4m3_cache_of_the_workload_is_the_bf16_cache_rounded():
    """The input generator's e4m3 cache decodes to within one e4m3 rounding of the same samples'
    bf16 cache (relative 2^-4 for normal values, half the subnormal step 2^-10 * scale below),
    and is deterministic."""
    g = synth.SyntheticInputs(synth.small("decode_32k", B=2, Lk=700))
    (k8, ks), (v8, vs) = g.k8, g.v8
    assert k8.dtype == np.uint8 and k8.shape == (2, 700, 128) and v8.shape == k8.shape
    for codes, sc, bf in ((k8, ks, g.k), (v8, vs, g.v)):
        deq = bf16_bits_to_f32(oracle.e4m3_to_bf16(codes, sc)).astype(np.float64)
        ref = bf16_bits_to_f32(bf).astype(np.float64)
        err = np.abs(deq - ref)
        # bf16 itself is within 2^-9 of the float32 sample; e4m3 within 2^-4 (or the subnormal step)
        assert np.all(err <= np.maximum(np.abs(ref) * (2.0 ** -4 + 2.0 ** -8), 2.0 ** -10 * sc + 1e-12))
        assert np.abs(deq).max() <= 448 * sc
    g2 = synth.SyntheticInputs(synth.small("decode_32k", B=2, Lk=700))
    assert np.array_equal(g2.k8[0], k8) and g2.k8[1] == ks


# ---------------------------------------------------------------------------------------------
# Attention backward (gradients of the full and sparse layers)
# ---------------------------------------------------------------------------------------------
def _torch_grads(q, k, v, do, scale, mask):
    """Gradients of torch SDPA (fp64) with K, V shared by every head (expanded, so autograd sums
    their gradients over the heads): q/do [B,Lq,H,d], k/v [B,Lk,d], mask [B or 1, Lq, Lk] bool."""
    Q = _t64(q).permute(0, 2, 1, 3).clone().requires_grad_(True)
    K = _t64(k).clone().requires_grad_(True)
    V = _t64(v).clone().requires_grad_(True)
    H = q.shape[2]
    o = torch.nn.functional.scaled_dot_product_attention(Q, K[:, None].expand(-1, H, -1, -1),
                                                         V[:, None].expand(-1, H, -1, -1),
                                                         attn_mask=mask[:, None], scale=scale)
    o.backward(_t64(do).permute(0, 2, 1, 3))
    return Q.grad.permute(0, 2, 1, 3).numpy(), K.grad.numpy(), V.grad.numpy()


@pytest.mark.parametrize("B,Lq,Lk,H,d", [(2, 13, 13, 3, 8), (1, 4, 19, 2, 16), (2, 1, 23, 4, 8)])
def test_attention_backward_matches_torch_autograd(B, Lq, Lk, H, d):
    rng = np.random.default_rng(40 + Lk)
    q, k, v, do = (_rand_bf16(rng, (B, Lq, H, d)), _rand_bf16(rng, (B, Lk, d)), _rand_bf16(rng, (B, Lk, d)),
                   _rand_bf16(rng, (B, Lq, H, d)))
    scale = 1.0 / math.sqrt(d)
    r = oracle.attn_bwd(q, k, v, do, scale)
    dq, dk, dv = _torch_grads(q, k, v, do, scale, _causal_mask(Lq, Lk)[None])
    np.testing.assert_allclose(r["dq"], dq.reshape(B * Lq, H, d), rtol=0, atol=1e-11)
    np.testing.assert_allclose(r["dk"], dk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(r["dv"], dv, rtol=0, atol=1e-11)
    # sampled rows give the same dQ rows
    rows = [0, B * Lq - 1]
    rs = oracle.attn_bwd(q, k, v, do, scale, rows=rows, want_kv=False)
    np.testing.assert_allclose(rs["dq"], r["dq"][rows], rtol=0, atol=0)


def test_sparse_attention_backward_matches_torch_autograd():
    """Sparse rows (random index sets, -1 padded) against autograd of SDPA with the same index
    mask; a repeated slot counts twice in the oracle, so the sets here are duplicate-free."""
    rng = np.random.default_rng(44)
    B, Lq, Lk, H, d, S = 2, 5, 30, 3, 8, 12
    q, k, v, do = (_rand_bf16(rng, (B, Lq, H, d)), _rand_bf16(rng, (B, Lk, d)), _rand_bf16(rng, (B, Lk, d)),
                   _rand_bf16(rng, (B, Lq, H, d)))
    idx = np.full((B, Lq, S), -1, np.int32)
    mask = torch.zeros((B, Lq, Lk), dtype=torch.bool)
    for b in range(B):
        for i in range(Lq):
            n = int(rng.integers(1, S + 1))
            sel = np.sort(rng.choice(Lk, size=n, replace=False))
            idx[b, i, :n] = sel
            mask[b, i, torch.from_numpy(sel.astype(np.int64))] = True
    r = oracle.attn_bwd(q, k, v, do, 0.4, idx=idx)
    dq, dk, dv = _torch_grads(q, k, v, do, 0.4, mask)
    np.testing.assert_allclose(r["dq"], dq.reshape(B * Lq, H, d), rtol=0, atol=1e-11)
    np.testing.assert_allclose(r["dk"], dk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(r["dv"], dv, rtol=0, atol=1e-11)


def test_attention_backward_is_the_derivative_of_the_forward():
    """Central differences of the oracle's own forward, loss = sum(dO * out), against the
    backward, for a few coordinates of Q, K and V (inputs perturbed in float64 through a
    value that bf16 represents exactly: the forward only reads bf16, so the step is 2^-4 of a
    coordinate that is a power of two)."""
    rng = np.random.default_rng(45)
    B, L, H, d = 1, 6, 2, 4
    q, k, v, do = (_rand_bf16(rng, (B, L, H, d)), _rand_bf16(rng, (B, L, d)), _rand_bf16(rng, (B, L, d)),
                   _rand_bf16(rng, (B, L, H, d)))
    scale = 0.5
    g = oracle.attn_bwd(q, k, v, do, scale)
    dof = bf16_bits_to_f32(do).astype(np.float64)

    def loss(qq, kk, vv):
        return float((oracle.full_attn_select(qq, kk, vv, scale, 1, 0)["out"] * dof.reshape(B * L, H, d)).sum())

    def setv(bits, pos, val):
        out = bits.copy()
        out[pos] = f32_to_bf16_bits(np.array([val], np.float32))[0]
        return out

    # the grid of exactly representable values around 1.0 with step 2^-7 is fine in bf16:
    # differences of +-2^-7 around a coordinate set to 1.0
    h = 2.0 ** -7
    for name, arr, pos, grad in (("q", q, (0, 3, 1, 2), g["dq"][3, 1, 2]), ("k", k, (0, 2, 1), g["dk"][0, 2, 1]),
                                 ("v", v, (0, 4, 3), g["dv"][0, 4, 3])):
        base = setv(arr, pos, 1.0)
        up, dn = setv(arr, pos, 1.0 + h), setv(arr, pos, 1.0 - h)
        args = {"q": q, "k": k, "v": v}
        args[name] = up
        lu = loss(args["q"], args["k"], args["v"])
        args[name] = dn
        ld = loss(args["q"], args["k"], args["v"])
        args[name] = base
        gb = oracle.attn_bwd(args["q"], args["k"], args["v"], do, scale)
        gval = {"q": gb["dq"][pos[1], pos[2], pos[3]] if name == "q" else None,
                "k": gb["dk"][pos] if name == "k" else None, "v": gb["dv"][pos] if name == "v" else None}[name]
        fd = (lu - ld) / (2 * h)
        assert abs(fd - gval) <= 1e-3 * max(1.0, abs(gval)), (name, fd, gval)


def test_attention_backward_identities():
    """Every row's dS sums to zero, so sum_j dK_j = 0; every row's p sums to one, so
    sum_j dV_j = sum of dO over rows and heads; K = 0 gives dQ = 0; the first row (one key)
    has dS = 0."""
    rng = np.random.default_rng(46)
    B, L, H, d = 2, 15, 3, 8
    q, k, v, do = (_rand_bf16(rng, (B, L, H, d)), _rand_bf16(rng, (B, L, d)), _rand_bf16(rng, (B, L, d)),
                   _rand_bf16(rng, (B, L, H, d)))
    r = oracle.attn_bwd(q, k, v, do, 0.35)
    np.testing.assert_allclose(r["dk"].sum(axis=1), 0.0, atol=1e-11)
    dof = bf16_bits_to_f32(do).astype(np.float64)
    np.testing.assert_allclose(r["dv"].sum(axis=1), dof.sum(axis=(1, 2)), atol=1e-11)
    np.testing.assert_allclose(r["dq"].reshape(B, L, H, d)[:, 0], 0.0, atol=1e-14)
    z = oracle.attn_bwd(q, np.zeros_like(k), v, do, 0.35)
    np.testing.assert_allclose(z["dq"], 0.0, atol=1e-14)
