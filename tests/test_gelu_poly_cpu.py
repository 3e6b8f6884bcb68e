"""The device GELU's polynomial (aut_ptx.cuh, gelu_fast), evaluated here in
fp32 as the kernels do, against the exact erf GELU x * Phi(x): within 5e-7
plus the fp32 rounding of the result everywhere, including the clamped tails
and x = 0."""
import os
import re

import numpy as np
from scipy.special import ndtr

HDR = os.path.join(os.path.dirname(__file__), "..", "audio_encoder_aut_b200", "csrc", "aut_ptx.cuh")


def _coefficients():
    src = open(HDR).read()
    body = src[src.index("AUT_DEV float gelu_fast(float x)"):]
    body = body[:body.index("}")]
    first = re.search(r"float s = ([-+0-9.e]+)f;", body).group(1)
    rest = re.findall(r"s = fmaf\(s, a, ([-+0-9.e]+)f\);", body)
    return [np.float32(first)] + [np.float32(c) for c in rest]  # highest degree first


def _gelu_fp32(x):
    x = x.astype(np.float32)
    a = np.minimum(np.abs(x), np.float32(6.0))
    cs = _coefficients()
    s = np.full_like(a, cs[0])
    for c in cs[1:]:
        s = (s * a + c).astype(np.float32)
    t = (np.float32(-0.72134752044448170) * a * a + s).astype(np.float32)
    h = np.exp2(t.astype(np.float64)).astype(np.float32)
    return np.where(x >= 0, x * (np.float32(1) - h), x * h).astype(np.float64)


def test_device_gelu_polynomial_matches_exact_gelu():
    assert len(_coefficients()) == 8
    x = np.concatenate([np.linspace(-12, 12, 400001), [0.0, -6.0, 6.0, -1e-30, 1e-30]])
    ref = x * ndtr(x)
    err = np.abs(_gelu_fp32(x) - ref)
    # fit error (<= 4.8e-7) plus the fp32 rounding of the final product and of 1 - h
    bound = 5e-7 + 2.0 ** -22 * np.abs(ref)
    assert (err <= bound).all(), (err - bound).max()
    assert _gelu_fp32(np.array([0.0]))[0] == 0.0
