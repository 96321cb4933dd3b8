"""Float64 reference of the causal-masked softmax over materialised scores (test
infrastructure; see the package doc).

[MLX-3919] "Fuse the causal mask into the SDPA fallback softmax" (ml-explore/mlx pull
request 3919, Summary and Description): when attention falls back to separate ops, a causal
mask is applied as the chain

    keep   = q_idx + offset >= kv_idx                   (greater_equal)
    masked = where(keep, scores, finfo(dtype).min)      (where, the dtype's lowest finite)
    probs  = softmax(masked) along the key axis         (precise: computed in float32)

and the fused kernel applies the same select where it loads the scores, so its result is the
chain's, element for element.  Masked entries come out exactly zero: exp(finfo.min - max)
underflows to 0.  A row whose keys are all masked holds finfo.min everywhere, so its max is
finfo.min and the chain gives the uniform 1/K (not NaN, as a -inf mask would).

Here the chain is written out in float64 on the already-rounded scores; the select value is
finfo(dtype).min of the scores' 16-bit type, exactly as the page states.  ``offset`` is the
position of query row 0 among the keys (the page's "mask offsets"; kv_len - q_len when a
chunk of queries closes a longer context).
"""
from __future__ import annotations

import numpy as np

# finfo(bfloat16).min and finfo(float16).min as exact binary values.
BF16_MIN = -(2.0 - 2.0 ** -7) * 2.0 ** 127      # -3.3895313892515355e38
FP16_MIN = -65504.0


def finfo_min(dtype: str) -> float:
    """The select value of the chain: the dtype's lowest finite number."""
    return {"bf16": BF16_MIN, "fp16": FP16_MIN}[dtype]


def causal_keep(Q: int, K: int, offset: int) -> np.ndarray:
    """greater_equal step of the chain: keep[q, kv] = q + offset >= kv, shape (Q, K)."""
    q_idx = np.arange(Q)[:, None]
    kv_idx = np.arange(K)[None, :]
    return (q_idx + offset) >= kv_idx


def masked_softmax(scores, offset: int, dtype: str = "bf16", causal: bool = True,
                   rows=None) -> np.ndarray:
    """probs = softmax(where(q + offset >= kv, scores, finfo.min)) over the last axis.

    scores: (..., Q, K) holding the rounded 16-bit values (any float type; upcast to
    float64).  causal=False is the plain softmax (the chain's last step alone).  ``rows``
    restricts the result to the given query rows (for sampled checks at full size).
    """
    s = np.asarray(scores, dtype=np.float64)
    Q, K = s.shape[-2], s.shape[-1]
    row_idx = np.arange(Q) if rows is None else np.asarray(rows)
    s = s[..., row_idx, :]
    if causal:
        keep = causal_keep(Q, K, offset)[row_idx]
        s = np.where(keep, s, finfo_min(dtype))
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)
