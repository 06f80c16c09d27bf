"""Error bound of the FMA-pipe 2^x used by the backward softmax (Cody-Waite
range reduction + fitted degree-3 polynomial, see sm100.cuh): the same fp32
evaluation in numpy against exact 2^x, over the softmax range x <= 0."""
import numpy as np

C = np.array([0.9999280572, 0.6932609677, 0.2426111400, 0.0551716685], dtype=np.float32)


def exp2_poly(x):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(C[3]) * f + C[2]
    p = (p.astype(np.float32) * f + C[1]).astype(np.float32)
    p = (p * f + C[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001), -np.random.default_rng(0).random(100000) * 20])
    y = exp2_poly(x.astype(np.float32)).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4          # far below bf16 rounding (2^-9 = 2.0e-3)


def test_deep_underflow_is_negligible():
    y = exp2_poly(np.array([-126.0, -200.0, -np.inf], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(y) < 2.0 ** -120)
