"""CPU checks of numerical helpers used inside the kernels.

exp2_poly_f2 (csrc/flux_device.cuh) evaluates 2^x on the FMA pipe: round-to-nearest
argument reduction with the 1.5 * 2^23 constant, a cubic for 2^f on [-1/2, 1/2], and
an integer add into the exponent field.  Its steps are emulated here in float32 and
compared with numpy's exp2 in float64."""

import numpy as np

C = [np.float32(0.9999280572), np.float32(0.6932609677), np.float32(0.2426111400),
     np.float32(0.0551716685)]


def exp2_poly(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t + np.float32(-12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (C[3] * f + C[2]).astype(np.float32)
    p = (p * f + C[1]).astype(np.float32)
    p = (p * f + C[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_poly_exp2_relative_error():
    x = np.linspace(-125.0, 8.0, 400_001).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_poly_exp2_masked_inputs_are_negligible():
    got = exp2_poly(np.array([-np.inf, -1e30, -300.0, -126.0], dtype=np.float32))
    assert np.allclose(got, 2.0 ** -125, rtol=1e-4)
