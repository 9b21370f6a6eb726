"""Error bound of the FMA-pipe exponential used by the kernels (host check).

The kernels evaluate 2^x for a quarter of the probabilities with a degree-3
polynomial instead of the MUFU unit (``exp2_fma2`` in csrc/fa_ptx.cuh).  This
test reads the coefficients from that header, repeats the kernel's float32
arithmetic step by step (shifter rounding, exact reduction, Horner with fused
multiply-adds, exponent-field addition) and checks the relative error bound
stated in the header against float64 ``exp2``, plus exactness at integers.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "exact_attention_112_b200", "csrc", "fa_ptx.cuh")


def _coeffs():
    src = open(HDR).read()
    body = src[src.index("float2 exp2_fma2(float2 x)"):]
    m = re.search(r"c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f", body)
    assert m, "coefficients not found in exp2_fma2"
    return [np.float32(float(v)) for v in m.groups()]


def _fma(a, b, c):
    # one rounding, as the hardware fused multiply-add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma(x):
    c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    j = (x + np.float32(12582912.0)).astype(np.float32)
    n = (j + np.float32(-12582912.0)).astype(np.float32)
    f = _fma(n, np.float32(-1.0), x)
    q = _fma(np.full_like(f, c3), f, np.full_like(f, c2))
    q = _fma(q, f, np.full_like(f, c1))
    q = _fma(q, f, np.full_like(f, 1.0))
    bits = q.view(np.int32) + (j.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-120.0, 8.0, 1_000_001).astype(np.float32)
    rel = np.abs(exp2_fma(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.1e-4, rel.max()


def test_exact_at_integers():
    n = np.arange(-120, 9).astype(np.float32)
    np.testing.assert_array_equal(exp2_fma(n), np.exp2(n.astype(np.float64)).astype(np.float32))


def test_reduction_is_round_to_nearest():
    # f = x - rint(x) stays within [-1/2, 1/2], so the polynomial is only
    # evaluated where it was fitted
    x = np.linspace(-50.0, 8.0, 100_001).astype(np.float32)
    j = (x + np.float32(12582912.0)).astype(np.float32)
    n = (j + np.float32(-12582912.0)).astype(np.float32)
    assert np.all(np.abs(x - n) <= 0.5)
