"""The polynomial 2^x used by the attention kernel to relieve the MUFU pipe (no GPU).

The coefficients are read from the kernel header and the same float32 steps (round-to-nearest
range reduction through 1.5*2^23, Horner evaluation, integer add into the exponent field) are
replayed in numpy; the result must be within 1e-4 relative of 2^x, far inside bf16's 2^-9.
"""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "block_sparse_attention_gather_b200", "csrc",
                   "spark_ptx.cuh")


def _coeffs():
    src = open(HDR).read()
    val = {n: np.float32(float(v)) for n, v in
           re.findall(r"constexpr float (kExp2C[0-3]) = ([0-9.]+)f;", src)}
    return val["kExp2C0"], val["kExp2C1"], val["kExp2C2"], val["kExp2C3"]


def exp2_poly_np(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_poly_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64)
    got = exp2_poly_np(x.astype(np.float32)).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4


def test_poly_handles_masked_columns():
    got = exp2_poly_np(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(got <= np.float32(2.0 ** -125)) and np.all(got >= 0)
