"""Pins of the float64 backward oracle (oracle/backward.py) against things it does not
compute itself: central finite differences of the forward oracle on tiny inputs, closed
forms (a window of one gives dV = dO and zero dQ, dK), and rows without live keys.  Planted
mistakes in its inputs (a wrong score_mod derivative, swapped K and V, a wrong scale) are
each caught.  CPU only."""
import numpy as np
import pytest

import oracle

C, SW, DOC = oracle.MASK_CAUSAL, oracle.MASK_SLIDING_WINDOW, oracle.MASK_DOCUMENT


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _loss(q, k, v, dout, mm, sm, scale):
    O, _ = oracle.attention(q, k, v, mm, sm, scale=scale)
    return float((O * dout).sum())


def _numeric_grads(q, k, v, dout, mm, sm, scale, eps=1e-6):
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(g.shape):
            x = args[which][idx]
            args[which][idx] = x + eps
            lp = _loss(*args, dout, mm, sm, scale)
            args[which][idx] = x - eps
            lm = _loss(*args, dout, mm, sm, scale)
            args[which][idx] = x
            g[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


CASES = [(C, 0, None, 0), (C | SW, 3, None, oracle.SCORE_SOFTCAP), (DOC, 0, [0, 0, 1, 1, 1, 2], 0),
         (C | DOC, 0, [0, 0, 0, 1, 1, 1], oracle.SCORE_ALIBI),
         (C, 0, None, oracle.SCORE_SOFTCAP | oracle.SCORE_ALIBI), (0, 0, None, oracle.SCORE_SOFTCAP)]


@pytest.mark.parametrize("kind,window,doc,score", CASES)
def test_gradients_equal_finite_differences(kind, window, doc, score):
    q, k, v, dout = (_rand((1, 2, 6, 3), s) * 1.5 for s in (11, 12, 13, 14))
    mm = oracle.make_mask_mod(kind, window=window or None, document_id=doc)
    sm = oracle.make_score_mod(score, H=2, softcap=2.0)          # a small cap bends the scores
    smg = oracle.make_score_mod_grad(score, softcap=2.0)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, mm, sm, smg, scale=0.7, chunk=4)
    nq, nk, nv = _numeric_grads(q, k, v, dout, mm, sm, 0.7)
    for a, n in ((dq, nq), (dk, nk), (dv, nv)):
        assert np.abs(a - n).max() < 1e-6 * max(1.0, np.abs(n).max())


def test_query_and_key_lengths_may_differ():
    q, dout = _rand((1, 1, 5, 4), 21), _rand((1, 1, 5, 4), 22)
    k, v = _rand((1, 1, 7, 4), 23), _rand((1, 1, 7, 4), 24)
    mm = oracle.sliding_window(3)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, mm)
    nq, nk, nv = _numeric_grads(q, k, v, dout, mm, None, None)
    for a, n in ((dq, nq), (dk, nk), (dv, nv)):
        assert np.abs(a - n).max() < 1e-6


def test_window_of_one_passes_gradients_straight_to_v():
    # Each row attends only to itself: O = V, so dV = dO and the scores get no gradient.
    q, k, v, dout = (_rand((2, 3, 9, 5), s) for s in (31, 32, 33, 34))
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, oracle.sliding_window(1))
    assert np.array_equal(dv, dout)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12


def test_rows_without_live_keys_get_zero_gradient():
    # Query rows 4.. see no key of a 4-long key sequence under this window.
    q, dout = _rand((1, 1, 8, 4), 41), _rand((1, 1, 8, 4), 42)
    k, v = _rand((1, 1, 4, 4), 43), _rand((1, 1, 4, 4), 44)
    mm = oracle.sliding_window(2)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, mm)
    assert np.all(np.isfinite(dq)) and np.all(dq[:, :, 5:] == 0)
    nq, nk, nv = _numeric_grads(q, k, v, dout, mm, None, None)
    assert np.abs(dk - nk).max() < 1e-6 and np.abs(dv - nv).max() < 1e-6


def test_score_mod_and_its_derivative_go_together():
    q = _rand((1, 1, 4, 2), 1)
    with pytest.raises(ValueError):
        oracle.attention_backward(q, q, q, q, oracle.causal, oracle.make_score_mod(1, H=1))


# ---------------------------------------------------------------- planted mistakes

def _fd_mismatch(dq, dk, dv, q, k, v, dout, mm, sm, scale):
    nq, nk, nv = _numeric_grads(q, k, v, dout, mm, sm, scale)
    return max(np.abs(dq - nq).max(), np.abs(dk - nk).max(), np.abs(dv - nv).max())


def test_pin_catches_a_wrong_score_mod_derivative():
    q, k, v, dout = (_rand((1, 1, 6, 3), s) * 2.0 for s in (51, 52, 53, 54))
    sm = oracle.make_score_mod(oracle.SCORE_SOFTCAP, H=1, softcap=1.5)
    identity = lambda s, b, h, qi, ki: np.ones_like(s)             # the soft-cap ignored
    grads = oracle.attention_backward(q, k, v, dout, oracle.causal, sm, identity, scale=1.0)
    assert _fd_mismatch(*grads, q, k, v, dout, oracle.causal, sm, 1.0) > 1e-3


def test_pin_catches_swapped_k_and_v():
    q, k, v, dout = (_rand((1, 1, 6, 3), s) for s in (61, 62, 63, 64))
    dq, dk, dv = oracle.attention_backward(q, v, k, dout, oracle.causal)
    assert _fd_mismatch(dq, dv, dk, q, k, v, dout, oracle.causal, None, None) > 1e-3


def test_pin_catches_a_wrong_scale():
    q, k, v, dout = (_rand((1, 1, 6, 3), s) for s in (71, 72, 73, 74))
    grads = oracle.attention_backward(q, k, v, dout, oracle.causal, scale=1.0)
    assert _fd_mismatch(*grads, q, k, v, dout, oracle.causal, None, None) > 1e-3


def test_row_subsets_split_the_gradient():
    # Restricting to query rows R gives exact dQ on R and R's share of dK, dV: two disjoint
    # subsets add up to the whole, and a key only the last rows see gets its whole gradient
    # from those rows.
    g = np.random.default_rng(41)
    q, k, v, do = (g.standard_normal((1, 2, 40, 8)) for _ in range(4))
    mm = oracle.causal
    full = oracle.attention_backward(q, k, v, do, mm)
    a = oracle.attention_backward(q, k, v, do, mm, rows=np.arange(0, 17))
    b = oracle.attention_backward(q, k, v, do, mm, rows=np.arange(17, 40))
    for t in range(3):
        assert np.abs(a[t] + b[t] - full[t]).max() < 1e-12
    assert np.array_equal(a[0][:, :, 17:], np.zeros_like(a[0][:, :, 17:]))
    assert np.abs(b[1][:, :, 17:] - full[1][:, :, 17:]).max() < 1e-12
    assert np.abs(b[2][:, :, 17:] - full[2][:, :, 17:]).max() < 1e-12
