"""Fits the polynomial of the software exp2 used by the score pass (csrc/tc.cuh: exp2_fma2).

2^x is split as 2^j * 2^f with j = round(x) and f in [-1/2, 1/2] (Cody and Waite's range
reduction); 2^f is a degree-5 polynomial whose coefficients minimise the maximum relative error
on [-1/2, 1/2], found here by iteratively reweighted least squares (Lawson's algorithm: the
weights grow where the error is largest until the error equioscillates). Run it to print the
coefficients as float32 and the resulting error bounds; tests/test_exp2_poly.py checks that the
kernel header holds these values.
"""
import numpy as np

DEGREE = 5


def fit(degree: int = DEGREE, iters: int = 60):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    w = np.ones_like(f)
    V = np.vander(f, degree + 1, increasing=True)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq((V / y[:, None]) * w[:, None], w, rcond=None)
        err = (V @ c) / y - 1.0
        w = w * (1.0 + 50.0 * np.abs(err) / np.abs(err).max())
        w /= w.mean()
    return c.astype(np.float32)


def horner_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    f32 = f.astype(np.float32)
    p = np.full_like(f32, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f32 + c32[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001)
    exact = np.abs((np.vander(f, DEGREE + 1, increasing=True) @ c.astype(np.float64)) / np.exp2(f) - 1).max()
    f32 = np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f) - 1).max()
    print("coefficients c0..c5 (float32):")
    for i, x in enumerate(c):
        print(f"  c{i} = {float(x):.9e}f  ({np.float32(x).view(np.uint32):#010x})")
    print(f"max relative error: {exact:.3e} (exact arithmetic), {f32:.3e} (float32 Horner)")
