"""The soft-cap's polynomial tanh (forward kernel, attn_fwd.cu).

Where every |s / cap| of a warp's rows in a tile is at most kTanhPolyBound, part of the pairs
take cap * tanh(a) from the odd Taylor series through a^7 with the cap folded into the
coefficients, evaluated by Horner's rule in a^2 with one rounding per fused multiply-add.  A
float32 model of those steps is checked against cap * tanh(a) in float64 over the whole bound.
The bound and the coefficient expressions are read from the CUDA source so the test follows
them.  CPU only.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "block_sparse_masked_x128_b200", "csrc", "attn_fwd.cu")


def _source():
    return open(SRC).read()


def _bound():
    return float(re.search(r"kTanhPolyBound\s*=\s*([0-9.eE+-]+)f", _source()).group(1))


def _coeffs(cap):
    # k1 = cap, k3 = cap * (-1/3), k5 = cap * (2/15), k7 = cap * (-17/315), as the kernel forms them.
    text = _source()
    fracs = []
    for name in ("k3", "k5", "k7"):
        m = re.search(rf"const float2 {name} = make_float2\(cap \* \(([-0-9.]+)f / ([0-9.]+)f\)", text)
        fracs.append(np.float32(np.float32(m.group(1)) / np.float32(m.group(2))))
    cap = np.float32(cap)
    return cap, (cap * fracs[0]).astype(np.float32), (cap * fracs[1]).astype(np.float32), \
        (cap * fracs[2]).astype(np.float32)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def capped_model(a, cap):
    k1, k3, k5, k7 = _coeffs(cap)
    a = a.astype(np.float32)
    a2 = (a * a).astype(np.float32)
    t = _fma32(np.full_like(a, k7), a2, np.full_like(a, k5))
    t = _fma32(t, a2, np.full_like(a, k3))
    t = _fma32(t, a2, np.full_like(a, k1))
    return (a * t).astype(np.float32)


def test_coefficients_are_the_taylor_series_of_tanh():
    k1, k3, k5, k7 = (float(c) for c in _coeffs(1.0))
    assert k1 == 1.0
    assert abs(k3 + 1 / 3) < 1e-7 and abs(k5 - 2 / 15) < 1e-7 and abs(k7 + 17 / 315) < 1e-7


def test_relative_error_over_the_bound():
    bound = _bound()
    assert 0 < bound <= 0.25
    cap = 30.0 * np.log2(np.e)   # the soft-cap in log2 units, as the kernel holds it
    a = np.linspace(-bound, bound, 2_000_001).astype(np.float32)
    a = a[a != 0]
    got = capped_model(a, cap).astype(np.float64)
    want = np.float64(np.float32(cap)) * np.tanh(a.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    # Truncation (first omitted term 62/2835 a^9) is below 6e-8 of tanh at the bound; the rest
    # is float32 rounding of a few operations.
    assert rel.max() < 3e-7
    trunc = 62 / 2835 * bound ** 9 / np.tanh(bound)
    assert trunc < 6e-8


def test_odd_and_exact_at_zero():
    cap = 30.0 * np.log2(np.e)
    a = np.array([0.0, 1e-30, 0.05, 0.2], dtype=np.float32)
    got = capped_model(a, cap)
    assert got[0] == 0.0
    assert np.array_equal(capped_model(-a, cap), -got)
