"""The software 2^x of the score pass (csrc/tc.cuh, exp2_fma2).

CPU: the kernel header holds exactly the coefficients fit_exp2.py fits, and that polynomial with
the range reduction stays within 3e-7 relative error of 2^x (float64 reference) over the inputs the
score pass feeds it. GPU: the device function itself, against float64 2^x and against the MUFU
approximation it is mixed with.
"""
import os
import re
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "long_context_mqa_b200"))
import fit_exp2  # noqa: E402


def _header_coefficients():
    src = open(os.path.join(ROOT, "long_context_mqa_b200", "csrc", "tc.cuh")).read()
    body = src[src.index("void exp2_fma2("):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"__uint_as_float\((0x[0-9a-f]+)u\)", body)
    # c5 once, then c4..c0 each twice (one per lane of the pair)
    order = [hexes[0]] + hexes[1::2]
    return np.array([int(h, 16) for h in order], dtype=np.uint32).view(np.float32)[::-1]  # c0..c5


def _soft_exp2_f32(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The device algorithm step by step in float32 (round to nearest after every operation)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = fit_exp2.horner_f32(c, f)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_header_holds_the_fitted_coefficients():
    np.testing.assert_array_equal(_header_coefficients(), fit_exp2.fit())


def test_polynomial_error_bound_over_the_score_range():
    c = _header_coefficients()
    x = np.concatenate([np.linspace(-126.0, 0.0, 400001), np.linspace(-1.0, 1.0, 100001)]).astype(np.float32)
    y = _soft_exp2_f32(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 3e-7
    # far below the clamp the result is 2^-126, a zero next to any sum of probabilities
    assert _soft_exp2_f32(np.array([-300.0, -1e30], np.float32), c).max() <= 2.0 ** -126 * (1 + 1e-6)


@pytest.mark.gpu
def test_device_exp2_matches_float64_and_mufu():
    import torch
    import long_context_mqa_b200 as hs2
    x = torch.cat([torch.linspace(-126.0, 0.0, 1 << 20), torch.linspace(-1.0, 1.0, 1 << 16),
                   torch.tensor([-300.0, -1e30])]).float().cuda()
    ys, ym = hs2.selftest_exp2(x)
    torch.cuda.synchronize()
    xs = x.double().cpu().numpy()
    ref = np.exp2(xs)
    soft = ys.double().cpu().numpy()
    mufu = ym.double().cpu().numpy()
    big = xs > -126.0
    assert np.max(np.abs(soft[big] / ref[big] - 1.0)) < 3e-7
    assert np.max(np.abs(mufu[big] / ref[big] - 1.0)) < 3e-7
    assert np.all(soft[~big] <= 2.0 ** -126 * (1 + 1e-6))
    # the host model of the device algorithm agrees to within one unit in the last place (the
    # device fuses each multiply-add; the host model rounds the product and the sum separately)
    host = _soft_exp2_f32(x.cpu().numpy(), _header_coefficients()).view(np.int32).astype(np.int64)
    dev = ys.cpu().numpy().view(np.int32).astype(np.int64)
    assert np.max(np.abs(host - dev)) <= 2
