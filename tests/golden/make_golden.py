"""Writes tests/golden/oracle_regression.json: oracle results on a small seeded workload.

Calls only the oracle (and the seeded input generator); nothing here comes from the CUDA
path. Re-run only when an oracle change is justified by a passage of the pages.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402

CASE = dict(base="tiny_prefill", Lq=160, Lk=160, window=16, topk=32, rows=[0, 15, 16, 47, 48, 100, 159])


def compute():
    wl = synth.small(CASE["base"], Lq=CASE["Lq"], Lk=CASE["Lk"])
    g = synth.SyntheticInputs(wl)
    r = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, CASE["window"], CASE["topk"], rows=CASE["rows"])
    idx_full = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, CASE["window"], CASE["topk"])["idx"]
    sp = oracle.sparse_attn(g.q_sparse(0), g.k, g.v, idx_full.reshape(1, wl.Lq, -1), wl.scale, rows=CASE["rows"])
    return {
        "case": CASE,
        "idx": r["idx"].tolist(),
        "lse": r["lse"].tolist(),
        "out_sum": r["out"].sum(axis=(1, 2)).tolist(),
        "sparse_out_sum": sp["out"].sum(axis=(1, 2)).tolist(),
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(compute(), f, indent=1)
