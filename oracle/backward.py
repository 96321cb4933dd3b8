"""Float64 reference gradients of the attention forward (test infrastructure; see the
package doc).

The pages name a deterministic FlexAttention backward ("PyTorch 2.13 brings custom AI
attention to Mac", section "What Else Shipped in PyTorch 2.13?") and the dQ write-order
parameters of [CBM] create_block_mask (``compute_dq_write_order``, ``dq_kv_order``), but give
no formula: the gradient is the derivative of the forward definition in ``attention.py``,
written out here step by step with the scores materialised in row chunks.  For one (b, h):

  s   = scale * q k^T               s' = score_mod(s),  -inf where mask_mod is false
  P   = softmax(s') by rows         O  = P v
  dV  = P^T dO                      dP = dO v^T
  Di  = sum_d dO[i, d] * O[i, d]    dS' = P * (dP - Di)      (softmax backward)
  dS  = dS' * score_mod'(s)         dQ = scale * dS k,  dK = scale * dS^T q

A row with no live key has P = 0 and contributes nothing.  score_mod' is the derivative of
the score_mod with respect to its score argument (``make_score_mod_grad``).
"""
from __future__ import annotations

import math
from typing import Callable, Optional

import numpy as np

from .attention import SCORE_ALIBI, SCORE_SOFTCAP


def soft_cap_grad(cap: float):
    """d/ds of cap * tanh(s / cap) = 1 - tanh(s / cap)^2."""
    def grad(score, b, h, q_idx, kv_idx):
        t = np.tanh(score / cap)
        return 1.0 - t * t
    return grad


def make_score_mod_grad(kind: int, softcap: float = 30.0):
    """Derivative functor matching ``make_score_mod(kind, ...)``; None when kind is 0.

    The ALiBi bias does not depend on the score (derivative 1); with both mods the soft-cap
    comes first, so the chain rule leaves the soft-cap's derivative.
    """
    if kind & ~(SCORE_SOFTCAP | SCORE_ALIBI):
        raise ValueError("unknown score kind bits")
    if kind & SCORE_SOFTCAP:
        return soft_cap_grad(float(softcap))
    if kind & SCORE_ALIBI:
        return lambda score, b, h, q_idx, kv_idx: np.ones_like(score)
    return None


def attention_backward(q, k, v, dout, mask_mod: Callable, score_mod: Optional[Callable] = None,
                       score_mod_grad: Optional[Callable] = None, scale: Optional[float] = None,
                       chunk: int = 512, rows=None):
    """(dQ, dK, dV) of sum(dout * O) for O = attention(q, k, v, mask_mod, score_mod, scale).

    q: (B, H, Sq, D); k, v: (B, H, Skv, D); dout: (B, H, Sq, D); all upcast to float64.
    score_mod_grad must be given whenever score_mod is.  ``rows`` restricts the sum to the
    given query rows: dQ is then exact on those rows (zero elsewhere) and dK, dV hold those
    rows' contributions only, which are the whole gradient for any key that no other query
    row sees (for sampled checks at full size).
    """
    if (score_mod is None) != (score_mod_grad is None):
        raise ValueError("score_mod and score_mod_grad go together")
    q, k, v, dout = (np.asarray(t, dtype=np.float64) for t in (q, k, v, dout))
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    kv_idx = np.arange(Skv)[None, :]
    row_list = np.arange(Sq) if rows is None else np.asarray(rows)
    for b in range(B):
        for h in range(H):
            for c0 in range(0, len(row_list), chunk):
                r = row_list[c0:c0 + chunk]
                q_idx = r[:, None]
                s = scale * (q[b, h, r, :] @ k[b, h].T)
                s_mod = score_mod(s, b, h, q_idx, kv_idx) if score_mod is not None else s
                live = np.broadcast_to(mask_mod(b, h, q_idx, kv_idx), s.shape)
                s_mod = np.where(live, s_mod, -np.inf)
                m = s_mod.max(axis=1)
                has = np.isfinite(m)
                p = np.exp(s_mod - np.where(has, m, 0.0)[:, None])
                p = p / np.where(has, p.sum(axis=1), 1.0)[:, None]      # rows without keys: 0
                o = p @ v[b, h]
                do = dout[b, h, r, :]
                dv[b, h] += p.T @ do
                dp = do @ v[b, h].T
                di = (do * o).sum(axis=1)
                ds = p * (dp - di[:, None])
                if score_mod_grad is not None:
                    ds = ds * np.where(live, score_mod_grad(s, b, h, q_idx, kv_idx), 0.0)
                dq[b, h, r, :] = scale * (ds @ k[b, h])
                dk[b, h] += scale * (ds.T @ q[b, h, r, :])
    return dq, dk, dv
