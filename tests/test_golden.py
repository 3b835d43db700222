"""Golden fixtures: the pages' constants, and a stored oracle regression case."""
import json
import os

import numpy as np

import synth

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_page_constants_are_the_defaults():
    c = json.load(open(os.path.join(HERE, "page_constants.json")))
    assert synth.WINDOW == c["window"]["value"]
    assert synth.TOPK == c["topk"]["value"]
    for name in ("decode_32k", "prefill_32k", "decode_256k", "decode_1m"):
        wl = synth.WORKLOADS[name]
        assert wl.H == c["q_heads"]["value"] and wl.window == 128 and wl.topk == 1024
    assert synth.WORKLOADS["prefill_32k"].bridge_hidden == c["hidden"]["value"]
    kv = c["kv_cache_gb_1m_fp8"]["value"]
    assert round(kv["Hybrid SWA"] / kv["HySparse2"], 1) == kv["ratio_vs_hybrid_swa"]


def test_oracle_regression_fixture():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    stored = json.load(open(os.path.join(HERE, "oracle_regression.json")))
    now = mg.compute()
    assert now["idx"] == stored["idx"]
    for key in ("lse", "out_sum", "sparse_out_sum"):
        np.testing.assert_allclose(np.array(now[key]), np.array(stored[key]), rtol=1e-12, atol=1e-12)
