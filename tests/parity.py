"""Host-side parity checks of CUDA results against the fp64 oracle.

Acceptance rules:
* selection: per query the GPU and oracle index sets must be equal except for swaps. The
  elements only one side picked are paired in oracle-score order; a pair (a, b) is accepted
  iff |score(a) - score(b)| <= 1e-5 * max(score(a), score(b)) with the oracle's fp64
  scores. The forced window must be present; indices must be unique, causal and exactly
  min(t+1, window+topk) of them, ascending, then -1 padding.
* outputs: max-abs error <= 2e-2 and relative L2 error <= 5e-3 against the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SWAP_REL_TOL = 1e-5
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3


def to_torch_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


@dataclass
class SelStats:
    rows: int = 0
    swaps: int = 0
    max_swap_rel: float = 0.0
    failures: list = field(default_factory=list)

    def ok(self) -> bool:
        return not self.failures


def check_selection(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_score: np.ndarray, t_pos: np.ndarray,
                    window: int, topk: int, rel_tol: float = SWAP_REL_TOL, max_report: int = 5) -> SelStats:
    """gpu_idx, ora_idx: [n, S]; ora_score: [n, Lk] fp64; t_pos: [n] query positions."""
    st = SelStats()
    S = window + topk
    for r in range(gpu_idx.shape[0]):
        st.rows += 1
        t = int(t_pos[r])
        g = gpu_idx[r]
        n_valid = min(t + 1, S)
        gv = g[:n_valid]
        problems = []
        if not (g[n_valid:] == -1).all():
            problems.append("padding is not -1")
        if (gv < 0).any() or (gv > t).any():
            problems.append("index out of causal range")
        if len(np.unique(gv)) != n_valid:
            problems.append("duplicate indices")
        if not (np.diff(gv) > 0).all():
            problems.append("not ascending")
        win = np.arange(max(0, t - window + 1), t + 1)
        if not np.isin(win, gv).all():
            problems.append("forced window missing")
        o = ora_idx[r][ora_idx[r] >= 0]
        a = np.setdiff1d(gv, o)   # picked only by the GPU
        b = np.setdiff1d(o, gv)   # picked only by the oracle
        if len(a) != len(b):
            problems.append(f"set sizes differ ({len(a)} vs {len(b)})")
        else:
            sc = ora_score[r]
            a = a[np.argsort(-sc[a], kind="stable")]
            b = b[np.argsort(-sc[b], kind="stable")]
            for x, y in zip(a, b):
                m = max(sc[x], sc[y])
                rel = abs(sc[x] - sc[y]) / m if m > 0 else 0.0
                st.max_swap_rel = max(st.max_swap_rel, rel)
                if rel > rel_tol:
                    problems.append(f"swap {x}<->{y} scores {sc[x]:.9g} vs {sc[y]:.9g} (rel {rel:.3g})")
                    break
                st.swaps += 1
        if problems and len(st.failures) < max_report:
            st.failures.append((r, t, problems))
    return st


def out_errors(gpu: np.ndarray, ref: np.ndarray) -> tuple[float, float]:
    gpu = np.asarray(gpu, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    diff = gpu - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30))
    return max_abs, rel_l2


def assert_out_close(gpu, ref, what: str, max_abs=OUT_MAX_ABS, rel_l2=OUT_REL_L2):
    ma, rl = out_errors(gpu, ref)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3g} (<= {max_abs}), rel-L2 {rl:.3g} (<= {rel_l2})"
    return ma, rl


def check_block_selection(gpu_row: np.ndarray, ora_tokens: np.ndarray, ora_bscore: np.ndarray, t: int,
                          block: int, n_blocks: int, window: int, rel_tol: float = SWAP_REL_TOL) -> SelStats:
    """One query's HySparse (v1) selection row: slots [0, n_blocks * block) must hold whole blocks'
    tokens <= t ascending then -1, the chosen blocks equal to the oracle's except swaps whose
    oracle block scores differ by <= rel_tol relative (paired in oracle-score order); slots
    [n_blocks * block, +window) must hold the window exactly."""
    st = SelStats(rows=1)
    nbs = n_blocks * block
    g = gpu_row[:nbs]
    n_valid = int((g >= 0).sum())
    gv = g[:n_valid]
    problems = []
    if not (g[n_valid:] == -1).all():
        problems.append("block slots: -1 padding not at the tail")
    if n_valid and ((gv > t).any() or not (np.diff(gv) > 0).all()):
        problems.append("block slots: not ascending / not causal")
    blocks = np.unique(gv // block)
    want_tok = np.concatenate([np.arange(j * block, min((j + 1) * block, t + 1)) for j in blocks]) if len(blocks) else gv
    if not np.array_equal(gv, want_tok):
        problems.append("block slots: not whole blocks")
    ob = np.unique(ora_tokens // block)
    a = np.setdiff1d(blocks, ob)
    b = np.setdiff1d(ob, blocks)
    if len(a) != len(b):
        problems.append(f"block set sizes differ ({len(blocks)} vs {len(ob)})")
    else:
        a = a[np.argsort(-ora_bscore[a], kind="stable")]
        b = b[np.argsort(-ora_bscore[b], kind="stable")]
        for x, y in zip(a, b):
            m = max(ora_bscore[x], ora_bscore[y])
            rel = abs(ora_bscore[x] - ora_bscore[y]) / m if m > 0 else 0.0
            st.max_swap_rel = max(st.max_swap_rel, rel)
            if rel > rel_tol:
                problems.append(f"block swap {x}<->{y} scores {ora_bscore[x]:.9g} vs {ora_bscore[y]:.9g}")
                break
            st.swaps += 1
    lo = max(0, t - window + 1)
    win = np.full(window, -1, np.int64)
    win[:t - lo + 1] = np.arange(lo, t + 1)
    if not np.array_equal(gpu_row[nbs:nbs + window], win):
        problems.append("window slots differ")
    if problems:
        st.failures.append((0, t, problems))
    return st
