"""The float64 causal-masked softmax oracle against what the page and the mathematics fix
("Fuse the causal mask into the SDPA fallback softmax", MLX pull request 3919: the chain
greater_equal -> where(finfo.min) -> softmax, masked entries exactly zero)."""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import workloads as wl


def _scores(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).float().numpy()


def test_select_values_are_the_dtype_minimum():
    assert oracle.BF16_MIN == float(torch.finfo(torch.bfloat16).min)
    assert oracle.FP16_MIN == float(torch.finfo(torch.float16).min)
    assert oracle.finfo_min("bf16") == oracle.BF16_MIN


@pytest.mark.parametrize("m", [-1e30, -60.0, 0.0, 7.5, 1e30])
def test_exp_of_min_minus_max_underflows_to_exact_zero(m):
    # The page's bit-identity argument: exp(finfo.min - max) is exactly 0, in float32 too.
    assert math.exp(oracle.BF16_MIN - m) == 0.0
    assert np.exp(np.float32(oracle.BF16_MIN) - np.float32(m)) == np.float32(0.0)


def test_one_live_key_gives_one_and_zeros():
    s = _scores((1, 1, 4, 16), 1)
    p = oracle.masked_softmax(s, offset=0)
    assert p[0, 0, 0, 0] == 1.0 and np.all(p[0, 0, 0, 1:] == 0.0)


def test_masked_entries_are_zero_and_live_ones_a_library_softmax():
    s = _scores((2, 3, 40, 64), 2)
    offset = 24
    p = oracle.masked_softmax(s, offset)
    keep = oracle.causal_keep(40, 64, offset)
    assert np.all(p[..., ~keep] == 0.0)
    for q in (0, 7, 39):
        n = q + offset + 1
        ref = scipy.special.softmax(s[..., q, :n].astype(np.float64), axis=-1)
        assert np.abs(p[..., q, :n] - ref).max() < 1e-15
    assert np.abs(p.sum(-1) - 1.0).max() < 1e-13


def test_fully_masked_rows_are_uniform_like_the_chain():
    # offset -5: rows 0..4 see no key; every entry is finfo.min, so the chain gives 1/K.
    s = _scores((1, 1, 8, 32), 3)
    p = oracle.masked_softmax(s, offset=-5)
    assert np.all(p[0, 0, :5] == 1.0 / 32)
    assert p[0, 0, 5, 0] == 1.0 and np.all(p[0, 0, 5, 1:] == 0.0)


def test_without_the_mask_it_is_the_plain_softmax():
    s = _scores((1, 2, 5, 33), 4)
    p = oracle.masked_softmax(s, offset=0, causal=False)
    assert np.abs(p - scipy.special.softmax(s.astype(np.float64), axis=-1)).max() < 1e-15


def test_brute_force_loops_on_a_tiny_case():
    s = _scores((1, 1, 4, 6), 5)[0, 0]
    offset = 2
    p = oracle.masked_softmax(s[None, None], offset)[0, 0]
    for q in range(4):
        vals = [s[q, kv] if q + offset >= kv else oracle.BF16_MIN for kv in range(6)]
        m = max(vals)
        e = [math.exp(x - m) for x in vals]
        tot = sum(e)
        for kv in range(6):
            assert abs(p[q, kv] - e[kv] / tot) < 1e-15


def test_rows_subset_equals_full():
    s = _scores((1, 2, 30, 48), 6)
    full = oracle.masked_softmax(s, 18)
    sub = oracle.masked_softmax(s, 18, rows=[0, 5, 29])
    assert np.array_equal(sub, full[..., [0, 5, 29], :])


def test_pin_catches_minus_infinity_as_the_select_value():
    s = _scores((1, 1, 8, 32), 3)
    keep = oracle.causal_keep(8, 32, -5)
    x = np.where(keep, s[0, 0].astype(np.float64), -np.inf)
    with np.errstate(invalid="ignore"):
        wrong = np.exp(x - x.max(-1, keepdims=True))
        wrong = wrong / wrong.sum(-1, keepdims=True)
    assert np.isnan(wrong[:5]).all()          # the uniform-row pin above fails on this


def test_pin_catches_an_off_by_one_offset():
    s = _scores((1, 1, 4, 16), 1)
    wrong = oracle.masked_softmax(s, offset=-1)     # q + offset > kv, one key short
    assert wrong[0, 0, 0, 0] != 1.0


def test_softmax_workload_recipe():
    w = wl.SOFTMAX_WORKLOADS[0]
    assert (w.B, w.H, w.Q, w.K, w.offset) == (1, 8, 1024, 32768, 31744)
    small = w.scaled(Q=64, K=512)
    assert small.offset == 448
    a, b = wl.make_scores(small), wl.make_scores(small)
    assert torch.equal(a, b) and a.dtype == torch.bfloat16 and a.shape == (1, 8, 64, 512)
