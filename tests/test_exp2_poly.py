"""The forward kernel's FMA-pipe exponential (csrc/fwd2.cu, exp2_fma): its
cubic's coefficients are the ones the Remez exchange in
split_kv_block_b200/exp2_poly.py computes, and the kernel's arithmetic,
emulated step by step in float32 (Cody-Waite split by the 1.5 * 2^23 rounding
constant, Horner, exponent-bit add), stays within the stated relative error of
2^x over the range the softmax uses."""
import os
import re

import numpy as np

from split_kv_block_b200.exp2_poly import remez_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _kernel_coefficients():
    src = open(os.path.join(ROOT, "split_kv_block_b200", "csrc", "fwd2.cu")).read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("}")]
    nums = [float(v) for v in re.findall(r"([0-9]+\.[0-9]+)f", body)]
    return nums


def test_coefficients_match_the_remez_fit():
    coef, err = remez_exp2()
    assert err < 8e-5
    nums = _kernel_coefficients()
    # c3, c2 in the first fmaf, then c1, then c0 (after the clamp -126 and the 1.5 * 2^23 constant)
    k3, k2, k1, k0 = nums[-4:]
    for got, want in zip((k0, k1, k2, k3), coef):
        assert abs(got - float(np.float32(want))) <= 1e-8 * max(1.0, abs(want))


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _exp2_fma(x):
    """The kernel's steps, one float32 rounding per instruction."""
    x = np.maximum(np.float32(x), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = np.float32(x + magic)
    f = np.float32(x - np.float32(t - magic))
    nums = [np.float32(v) for v in _kernel_coefficients()[-4:]]
    c3, c2, c1, c0 = nums
    q = _fma32(c3, f, c2)
    q = _fma32(q, f, c1)
    q = _fma32(q, f, c0)
    bits = q.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 9.0, 400001), np.arange(-125, 10, dtype=np.float64) + 0.5,
                        np.arange(-125, 10, dtype=np.float64)]).astype(np.float32)
    got = _exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 8e-5 + 2e-7
    # the sign is never touched, and below the clamp the value is about 2^-125 (negligible beside 1)
    assert np.all(got > 0)
    assert 0 < _exp2_fma(np.float32(-1e4)) < 3e-38
