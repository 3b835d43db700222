"""The C-ABI library loads and exports every symbol include/hs2.h declares (CPU only).

Only host-side paths are exercised here: version, status strings and argument validation
that rejects calls before anything touches a device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "hs2.h")).read()
    return re.findall(r"HS2_API\s+[\w\s\*]+?\b(hs2_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(_declared())
    for n in ("hs2_full_attn_select", "hs2_sparse_attn", "hs2_bridge_kv_proj", "hs2_full_attn_select_workspace_bytes",
              "hs2_sparse_attn_workspace_bytes", "hs2_bridge_kv_proj_workspace_bytes", "hs2_read_device_status",
              "hs2_status_string", "hs2_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import long_context_mqa_b200 as hs2
    lib = ctypes.CDLL(hs2.LIBRARY_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_status_strings():
    import long_context_mqa_b200 as hs2
    assert hs2.ABI_VERSION == 1
    for code, text in hs2.STATUS.items():
        assert hs2.lib.hs2_status_string(code).decode() == text


def test_null_arguments_are_rejected_before_any_launch():
    import long_context_mqa_b200 as hs2
    L = hs2.lib
    assert L.hs2_full_attn_select(None, None, None, 1, 1, 8, 64, 128, 0.1, 128, 1024, None, None, None, None, 0,
                                  None) == hs2.ERR_INVALID_ARG
    assert L.hs2_sparse_attn(None, None, None, None, 1, 1, 8, 64, 128, 8, 0.1, None, None, None, 0,
                             None) == hs2.ERR_INVALID_ARG
    assert L.hs2_bridge_kv_proj(None, 8, 64, None, 1, 128, None, None, 0, None) == hs2.ERR_INVALID_ARG
    assert L.hs2_read_device_status(None, None) == hs2.ERR_WORKSPACE


@pytest.mark.parametrize("B,Lk", [(8, 262144), (2, 1048576), (32, 32768), (1, 100)])
def test_workspace_queries_are_sane(B, Lk):
    import long_context_mqa_b200 as hs2
    n = hs2.full_attn_select_workspace_bytes(B, 1, Lk, 64, 128)
    assert n >= 256
    # scores (4 B) + boundary keys (8 B) per older token dominate
    assert n >= B * max(Lk - 128, 0) * 12
    assert hs2.full_attn_select_workspace_bytes(0, 1, Lk, 64, 128) == 0
    assert hs2.sparse_attn_workspace_bytes(B, 1, Lk, 64, 128, 1152) >= 256


def test_ragged_workspace_query_and_argument_checks():
    import long_context_mqa_b200 as hs2
    lens = [262144, 3000, 1, 128, 129]
    n = hs2.full_attn_select_ragged_workspace_bytes(lens, 262144, 64, 128)
    # room for the longest sequence's older tokens in every row, at least
    assert n >= len(lens) * (262144 - 128) * 12
    # equal lengths: the batched call's workspace
    assert hs2.full_attn_select_ragged_workspace_bytes([5000] * 3, 5000, 64, 128) == \
        hs2.full_attn_select_workspace_bytes(3, 1, 5000, 64, 128)
    L = hs2.lib
    bad = (ctypes.c_int32 * 2)(10, 0)      # a length of 0
    assert L.hs2_full_attn_select_ragged_workspace_bytes(2, bad, 100, 64, 128, 128, 1024) == 0
    over = (ctypes.c_int32 * 2)(10, 101)   # longer than Lk
    assert L.hs2_full_attn_select_ragged_workspace_bytes(2, over, 100, 64, 128, 128, 1024) == 0
    many = (ctypes.c_int32 * 257)(*([10] * 257))  # more sequences than the schedule's tables hold
    assert L.hs2_full_attn_select_ragged_workspace_bytes(257, many, 100, 64, 128, 128, 1024) == 0
    assert L.hs2_full_attn_select_ragged(None, None, None, 2, bad, 100, 64, 128, 0.1, 128, 1024, None, None, None,
                                         None, 0, None) == hs2.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        hs2.full_attn_select_ragged_workspace_bytes([10, 0], 100, 64, 128)


def test_fp8_workspace_queries_and_argument_checks():
    import long_context_mqa_b200 as hs2
    L = hs2.lib
    # decode over an e4m3 cache: the ragged call's workspace (lens NULL: every sequence full)
    assert hs2.full_attn_select_fp8kv_workspace_bytes(8, None, 262144, 64, 128) == \
        hs2.full_attn_select_ragged_workspace_bytes([262144] * 8, 262144, 64, 128)
    lens = [40000, 3000, 1]
    assert hs2.full_attn_select_fp8kv_workspace_bytes(3, lens, 40000, 64, 128) == \
        hs2.full_attn_select_ragged_workspace_bytes(lens, 40000, 64, 128)
    # prompts and chunks: room for the widened bf16 K and V; one query: the decode workspace
    ws = L.hs2_full_attn_select_prefill_fp8kv_workspace_bytes(2, 1000, 3000, 64, 128, 128, 1024)
    assert ws >= 2 * 2 * 3000 * 128 * 2
    assert L.hs2_full_attn_select_prefill_fp8kv_workspace_bytes(2, 1, 3000, 64, 128, 128, 1024) == \
        hs2.full_attn_select_fp8kv_workspace_bytes(2, None, 3000, 64, 128)
    assert L.hs2_full_attn_select_prefill_fp8kv_workspace_bytes(2, 3001, 3000, 64, 128, 128, 1024) == 0
    # rejected before any device work: null pointers, then (with aligned stand-in addresses that
    # are never dereferenced) scales that are not positive and finite, and a page table whose
    # width does not match Lk
    assert L.hs2_full_attn_select_fp8kv(None, None, None, 1.0, 1.0, 1, None, 100, None, 0, 0, 64, 128, 0.1, 128, 1024,
                                        None, None, None, None, 0, None) == hs2.ERR_INVALID_ARG
    a = 1 << 20
    for ks in (0.0, -2.0, float("inf"), float("nan")):
        assert L.hs2_full_attn_select_fp8kv(a, a, a, ks, 1.0, 1, None, 100, None, 0, 0, 64, 128, 0.1, 128, 1024,
                                            a, a, a, a, 1 << 20, None) == hs2.ERR_INVALID_ARG
        assert L.hs2_sparse_attn_fp8kv(a, a, a, 1.0, ks, a, 1, 1, 100, None, 0, 0, 64, 128, 1152, 0.1, a, None, a,
                                       1 << 20, None) == hs2.ERR_INVALID_ARG
        assert L.hs2_full_attn_select_prefill_fp8kv(a, a, a, ks, 1.0, 1, 50, 100, 64, 128, 0.1, 128, 1024, a, a, a, a,
                                                    1 << 20, None) == hs2.ERR_INVALID_ARG
    assert L.hs2_full_attn_select_fp8kv(a, a, a, 1.0, 1.0, 1, None, 1000, a, 4, 10, 64, 128, 0.1, 128, 1024,
                                        a, a, a, a, 1 << 20, None) == hs2.ERR_INVALID_ARG  # 4 pages != 1000 rows
    assert L.hs2_sparse_attn_fp8kv(a, a, a, 1.0, 1.0, a, 1, 1, 1000, a, 4, 10, 64, 128, 1152, 0.1, a, None, a,
                                   1 << 20, None) == hs2.ERR_INVALID_ARG
    assert L.hs2_selftest_e4m3(a, a, a, 3, None) == hs2.ERR_INVALID_ARG  # odd count


def test_marshalling_module_checks_arguments_before_any_call():
    """The C++ marshalling module of the binding (its fast path, taken when every buffer is given)
    loads, and rejects host tensors, wrong dtypes and shapes with ValueError without calling the
    library."""
    import torch
    import long_context_mqa_b200 as hs2
    assert hs2._fast is not None, "the marshalling module was not built"
    q = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    kv = torch.zeros(1, 10, 128, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 64)
    idx = torch.zeros(1, 1, 1152, dtype=torch.int32)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError):
        hs2.full_attn_select(q, kv, kv, out=q, lse=lse, idx=idx, workspace=ws)
    with pytest.raises(ValueError):
        hs2.sparse_attn(q, kv, kv, idx, out=q, workspace=ws)
    with pytest.raises(ValueError):  # a wrong dtype is reported the same way by the C++ checks
        hs2._fast.full_attn_select(q.float(), kv, kv, 0.1, 128, 1024, q, lse, idx, ws, 0)
