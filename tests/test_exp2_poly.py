"""Error bound of the FMA-pipe 2^x used for a share of the 8-bit attention's
exponentials (exp2_poly in the kernels' PTX helper header): Cody-Waite range reduction
to f in [-0.5, 0.5] and a degree-3 polynomial. The coefficients are read from the source,
and the same float32 steps are replayed here over a dense grid."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "video_diffusion_transformer_wan_b200", "csrc", "ptx.cuh")


def _coefficients():
    text = open(SRC).read()
    body = re.search(r"float exp2_poly\(float x\) \{(.*?)\n\}", text, re.S).group(1)
    assert "fmaxf(x, -125.0f)" in body and "12582912.0f" in body        # clamp, 1.5 * 2^23 rounding
    fmas = re.findall(r"fmaf\(([^;]*)\);", body)
    c3, c2 = (float(v.strip().rstrip("f")) for v in fmas[0].split(",")[0:3:2])
    c1 = float(fmas[1].split(",")[2].strip().rstrip("f"))
    c0 = float(fmas[2].split(",")[2].strip().rstrip("f"))
    return c3, c2, c1, c0


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_poly_replay(x):
    c3, c2, c1, c0 = (np.float32(v) for v in _coefficients())
    x = np.maximum(np.float32(x), np.float32(-125.0))
    t = np.float32(x + np.float32(12582912.0))
    n = np.round(np.float64(t) - 12582912.0)                  # the integer in t's low mantissa bits
    f = np.float32(x - np.float32(t - np.float32(12582912.0)))
    p = _fma32(c3, f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    return np.float64(p) * np.exp2(n)


def test_range_reduction_and_polynomial_error_bound():
    x = np.concatenate([np.linspace(-40.0, 8.0, 400001), np.linspace(-125.0, -40.0, 20001)]).astype(np.float32)
    got = np.array([exp2_poly_replay(v) for v in x[::7]])
    ref = np.exp2(np.float64(x[::7]))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 8e-5                                   # stated: 7.5e-5 (13.7 bits)
    assert rel.max() < 2.0 ** -9                               # far inside the E4M3 (and bf16) spacing of P


def test_exact_at_integers_and_clamped_below():
    for k in range(-20, 9):
        assert abs(exp2_poly_replay(float(k)) / 2.0 ** k - 1) <= 8e-5
    assert exp2_poly_replay(-1000.0) < 1e-37                  # clamped to 2^-125: a zero weight
