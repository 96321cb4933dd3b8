"""Float64 CPU oracle for block-sparse masked attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs (the
``cpu_baseline`` sample and the ``--impl reference`` arm) may use it.  It shares
no code with the CUDA library.

It is the plain definition of what the method computes, written out with
materialised scores and an explicit dense mask, in the order and notation of
the pages (see each function's docstring for the passage it follows):

  mask_mod(b, h, q_idx, kv_idx) -> bool        allowed (query, key) pairs
  score_mod(score, b, h, q_idx, kv_idx) -> f   value change on live scores
  create_block_mask(...)                        per-tile partial / full lists
  attention(q, k, v, mask_mod, score_mod)       softmax(score_mod(scale*QK^T)
                                                masked) @ V, and logsumexp
  attention_backward(q, k, v, dO, ...)          dQ, dK, dV of that definition
  masked_softmax(scores, offset)                causal select + softmax over
                                                materialised scores (the unfused chain)

Every function is pinned by a "not gpu" test against facts the pages or the
mathematics fix; where a function follows a reading of the pages (the composition
order of soft-cap and ALiBi, for one), the pin checks that reading.
"""
from .backward import attention_backward, make_score_mod_grad, soft_cap_grad  # noqa: F401
from .masked_softmax import masked_softmax, causal_keep, finfo_min, BF16_MIN, FP16_MIN  # noqa: F401
from .attention import (  # noqa: F401
    causal, sliding_window, document, sequence_lengths, conjunction, all_true, make_mask_mod,
    dense_mask, soft_cap, alibi, alibi_slopes, compose_score_mods,
    make_score_mod, create_block_mask, attention, live_positions,
    MASK_CAUSAL, MASK_SLIDING_WINDOW, MASK_DOCUMENT, SCORE_SOFTCAP, SCORE_ALIBI,
)
