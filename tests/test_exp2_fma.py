"""The FMA-pipe 2^x used for part of each softmax row (exp2_fma2 in sm100_ptx.cuh).

A float32 model of the same steps -- round-to-nearest via 1.5 * 2^23, exact reduction
f = a - n, degree-3 polynomial in f with one rounding per fused multiply-add, and n added to
the exponent bits -- is checked against 2^x in float64.  The coefficients are read from the
CUDA source so the test follows them.  CPU only.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "block_sparse_masked_x128_b200", "csrc", "sm100_ptx.cuh")


def _coeffs():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"kExp2C{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)))
            for i in range(4)]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_model(a):
    c0, c1, c2, c3 = _coeffs()
    a = np.maximum(a.astype(np.float32), np.float32(-126.0))
    rnd = np.float32(12582912.0)
    t = (a + rnd).astype(np.float32)
    neg_n = _fma32(t, np.float32(-1.0), rnd)
    f = (a + neg_n).astype(np.float32)
    q = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    # After the lazy rescale, exponents lie in (-inf, 8]; results below 2^-125 are negligible
    # next to a row sum >= 1.
    a = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    got = exp2_fma_model(a).astype(np.float64)
    rel = np.abs(got / np.exp2(a.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4


def test_integers_are_close_to_powers_of_two():
    n = np.arange(-120, 9).astype(np.float32)
    got = exp2_fma_model(n).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(n.astype(np.float64)) - 1) < 1e-4)


def test_tiny_and_masked_inputs_stay_tiny_and_non_negative():
    a = np.array([-126.0, -127.0, -1000.0, -np.inf], dtype=np.float32)
    got = exp2_fma_model(a)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -125)


def test_coefficients_are_the_lawson_minimax_fit():
    # The constants in the CUDA source are (to float32 precision of the fit) the minimax
    # relative-error cubic that fit_exp2.py computes.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_fit_exp2", os.path.join(ROOT, "block_sparse_masked_x128_b200", "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coeffs, rel = mod.fit()
    src = np.array([float(c) for c in _coeffs()])
    assert np.abs(src - coeffs).max() < 2e-6
    assert rel < 7.6e-5
