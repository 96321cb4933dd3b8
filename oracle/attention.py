"""Float64 reference definitions (test infrastructure; see the package doc).

Citations name the page and its section:
  [FA-Mac]  "How to Use FlexAttention on Apple Silicon: Sliding-Window and
            Document Masks with block_mask" (dreaming.press)
  [SWA]     "Sliding-Window Self-Attention" (crackedaicode Flax exercise)
  [CBM]     "tensorplay.nn.attention.create_block_mask" (API reference page)
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence

import numpy as np

MASK_CAUSAL = 1
MASK_SLIDING_WINDOW = 2
MASK_DOCUMENT = 4
SCORE_SOFTCAP = 1
SCORE_ALIBI = 2


# --------------------------------------------------------------------------
# mask_mod functors: mask_mod(b, h, q_idx, kv_idx) -> bool
# [FA-Mac] "The two hooks": a mask_mod says whether a query/key pair may attend.
# Arguments broadcast like numpy index grids.
# --------------------------------------------------------------------------

def causal(b, h, q_idx, kv_idx):
    """[FA-Mac] "Mask 1: causal": a query sees keys at or before its position."""
    return q_idx >= kv_idx


def sliding_window(W: int):
    """[SWA] "State the boundary precisely": query i may read key j iff 0 <= i - j < W.

    W counts the current position, so W - 1 earlier keys are visible.  The
    same band is [FA-Mac] "Mask 2": causal_mask & (q_idx - kv_idx < W).
    """
    if W <= 0:
        raise ValueError("window must be positive")

    def mask_mod(b, h, q_idx, kv_idx):
        d = q_idx - kv_idx
        return (d >= 0) & (d < W)
    return mask_mod


def document(document_id):
    """[FA-Mac] "Mask 3: document-packed": document_id[q_idx] == document_id[kv_idx]."""
    doc = np.asarray(document_id)

    def mask_mod(b, h, q_idx, kv_idx):
        return doc[q_idx] == doc[kv_idx]
    return mask_mod


def sequence_lengths(kv_lens):
    """Per-batch context length: key kv_idx of batch b exists iff kv_idx < kv_lens[b].

    A batch of sequences of different lengths shares one KV_LEN-long layout (padded, or paged
    as PagedAttention through block indices, "PyTorch 2.13 brings custom AI attention to
    Mac", "What Attention Patterns Does FlexAttention Support?"); the padding is masked.
    """
    lens = np.asarray(kv_lens)

    def mask_mod(b, h, q_idx, kv_idx):
        return kv_idx < lens[b]
    return mask_mod


def all_true(b, h, q_idx, kv_idx):
    """No mask: every pair is allowed."""
    return np.ones(np.broadcast(q_idx, kv_idx).shape, dtype=bool)


def conjunction(*mods):
    """[FA-Mac] Masks 2 and 3 AND predicates together (causal_mask & window_mask)."""
    def mask_mod(b, h, q_idx, kv_idx):
        out = all_true(b, h, q_idx, kv_idx)
        for m in mods:
            out = out & m(b, h, q_idx, kv_idx)
        return out
    return mask_mod


def make_mask_mod(kind: int, window: Optional[int] = None, document_id=None, kv_lens=None):
    """The mask_mod for a bit set of kinds (causal 1, sliding window 2, document 4), AND the
    per-batch sequence lengths when kv_lens is given."""
    mods = []
    if kv_lens is not None:
        mods.append(sequence_lengths(kv_lens))
    if kind & MASK_CAUSAL:
        mods.append(causal)
    if kind & MASK_SLIDING_WINDOW:
        mods.append(sliding_window(int(window)))
    if kind & MASK_DOCUMENT:
        if document_id is None:
            raise ValueError("document mask needs document_id")
        mods.append(document(document_id))
    if kind & ~(MASK_CAUSAL | MASK_SLIDING_WINDOW | MASK_DOCUMENT):
        raise ValueError("unknown mask kind bits")
    return conjunction(*mods) if mods else all_true


def dense_mask(mask_mod, Q_LEN: int, KV_LEN: int, b: int = 0, h: int = 0,
               rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """The explicit (Q_LEN, KV_LEN) boolean mask, or only the given query rows.

    [SWA] "Build and apply the mask": i = arange(T)[:, None], j = arange(T)[None, :].
    """
    q_idx = (np.arange(Q_LEN) if rows is None else np.asarray(rows))[:, None]
    kv_idx = np.arange(KV_LEN)[None, :]
    m = mask_mod(b, h, q_idx, kv_idx)
    return np.broadcast_to(m, (q_idx.shape[0], KV_LEN)).astype(bool)


# --------------------------------------------------------------------------
# score_mod functors: score_mod(score, b, h, q_idx, kv_idx) -> score
# [FA-Mac] "The two hooks": a score_mod returns a modified attention score and
# runs on every live position; it never changes which positions are live.
# --------------------------------------------------------------------------

def soft_cap(cap: float):
    """[FA-Mac] "Bonus: a score_mod for soft-capping": cap * tanh(score / cap)."""
    def score_mod(score, b, h, q_idx, kv_idx):
        return cap * np.tanh(score / cap)
    return score_mod


def alibi_slopes(H: int) -> np.ndarray:
    """Per-head ALiBi slopes 2^(-8(h+1)/H), h = 0..H-1 (the workload's stated form)."""
    return np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=np.float64)


def alibi(slopes):
    """ALiBi additive bias slope_h * (kv_idx - q_idx).

    [FA-Mac] "The two hooks" and the FlexAttention news article describe ALiBi only as an
    additive bias that penalises attention to distant tokens.  Reading: the bias is
    slope_h * (kv_idx - q_idx), which is <= 0 wherever a causal mask lets a key through.
    """
    sl = np.asarray(slopes, dtype=np.float64)

    def score_mod(score, b, h, q_idx, kv_idx):
        return score + sl[h] * (kv_idx - q_idx).astype(np.float64)
    return score_mod


def compose_score_mods(*mods):
    """Apply score_mods left to right.

    With both soft-cap and ALiBi the pages fix no order.  Reading: soft-cap first, then
    the bias (30*tanh(s/30) + bias), so the distance penalty is not squashed into
    [-30, 30].  The composition is pinned to that reading by closed forms: scores
    s = cap*ln(a), whose capped value is the rational cap*(a^2-1)/(a^2+1), plus the
    exact bias -2^-(h+1)*(q_idx - kv_idx).
    """
    def score_mod(score, b, h, q_idx, kv_idx):
        for m in mods:
            score = m(score, b, h, q_idx, kv_idx)
        return score
    return score_mod


def make_score_mod(kind: int, H: int, softcap: float = 30.0, slopes=None):
    mods = []
    if kind & SCORE_SOFTCAP:
        mods.append(soft_cap(float(softcap)))
    if kind & SCORE_ALIBI:
        mods.append(alibi(alibi_slopes(H) if slopes is None else slopes))
    if kind & ~(SCORE_SOFTCAP | SCORE_ALIBI):
        raise ValueError("unknown score kind bits")
    return compose_score_mods(*mods) if mods else None


# --------------------------------------------------------------------------
# Block mask: [CBM] create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN, BLOCK_SIZE=128,
# separate_full_blocks=True); [FA-Mac] "Mask 1": B=None, H=None broadcast.
# --------------------------------------------------------------------------

def create_block_mask(mask_mod, B: Optional[int], H: Optional[int], Q_LEN: int,
                      KV_LEN: int, BLOCK_SIZE=128,
                      separate_full_blocks: bool = True) -> dict:
    """Brute-force block metadata from the dense mask.

    BLOCK_SIZE is an int or a (q, kv) pair ([CBM] Parameters, BLOCK_SIZE: a single int is used
    for both query and key/value).  The dense mask is reshaped to (QB, BQ, KVB, BKV) tiles; a
    tile with no true entry is
    dead (skipped, [FA-Mac] "The two hooks"), a tile whose entries are all true is full,
    and any other live tile is partial.  With separate_full_blocks the full tiles go to
    their own lists so mask_mod can be skipped there; without it every live tile is
    listed as partial ([CBM] Parameters, separate_full_blocks).

    Readings where the pages are silent: positions past Q_LEN / KV_LEN count as
    masked, so a ragged edge tile is never full; each list holds ascending kv-block
    indices and is padded with 0 after its count; B or H of None/0 is stored as one
    broadcast entry.
    """
    if isinstance(BLOCK_SIZE, (tuple, list)):
        BQ, BKV = (int(x) for x in BLOCK_SIZE)
    else:
        BQ = BKV = int(BLOCK_SIZE)
    QB = -(-Q_LEN // BQ)
    KVB = -(-KV_LEN // BKV)
    Bp = 1 if not B else int(B)
    Hp = 1 if not H else int(H)
    kv_num = np.zeros((Bp, Hp, QB), dtype=np.int32)
    kv_idx = np.zeros((Bp, Hp, QB, KVB), dtype=np.int32)
    full_num = np.zeros((Bp, Hp, QB), dtype=np.int32)
    full_idx = np.zeros((Bp, Hp, QB, KVB), dtype=np.int32)
    for b in range(Bp):
        for h in range(Hp):
            for i in range(QB):
                rows = np.arange(i * BQ, min((i + 1) * BQ, Q_LEN))
                m = np.zeros((BQ, KVB * BKV), dtype=bool)
                m[: len(rows), :KV_LEN] = dense_mask(mask_mod, Q_LEN, KV_LEN, b, h, rows)
                tiles = m.reshape(BQ, KVB, BKV)
                any_t = tiles.any(axis=(0, 2))
                all_t = tiles.all(axis=(0, 2))
                full = all_t if separate_full_blocks else np.zeros_like(all_t)
                partial = any_t & ~full
                p = np.nonzero(partial)[0]
                f = np.nonzero(full)[0]
                kv_num[b, h, i] = len(p)
                kv_idx[b, h, i, : len(p)] = p
                full_num[b, h, i] = len(f)
                full_idx[b, h, i, : len(f)] = f
    return {"kv_num_blocks": kv_num, "kv_indices": kv_idx,
            "full_kv_num_blocks": full_num, "full_kv_indices": full_idx,
            "BLOCK_SIZE": (BQ, BKV), "Q_LEN": Q_LEN, "KV_LEN": KV_LEN}


def live_positions(mask_mod, Q_LEN: int, KV_LEN: int, b: int = 0, h: int = 0,
                   chunk: int = 1024) -> int:
    """Number of true entries of the dense mask (counted in row chunks)."""
    total = 0
    for r0 in range(0, Q_LEN, chunk):
        rows = np.arange(r0, min(r0 + chunk, Q_LEN))
        total += int(dense_mask(mask_mod, Q_LEN, KV_LEN, b, h, rows).sum())
    return total


# --------------------------------------------------------------------------
# Attention: the plain definition with materialised scores.
# --------------------------------------------------------------------------

def attention(q, k, v, mask_mod: Callable, score_mod: Optional[Callable] = None,
              scale: Optional[float] = None, rows: Optional[Sequence[int]] = None,
              chunk: int = 512):
    """O = softmax(masked score_mod(scale * q k^T)) v and lse = log sum exp per row.

    q, k, v: arrays (B, H, S, D) holding the already-rounded inputs; computed in float64.
    [FA-Mac] "The two hooks": mask_mod decides which pairs are live and score_mod changes
    live scores only; the news article and [SWA] "A dense mask does not make the
    calculation sparse" describe the (H, T, T) score tensor this function builds in row
    chunks.  Readings: score_mod sees the score after scaling (scale defaults to
    1/sqrt(D), the SDPA default); lse is the natural log over live positions after
    score_mod; a row with no live key gives O = 0 and lse = -inf.
    ``rows`` restricts the computation to the given query indices (for sampled checks at
    full size); O then has shape (B, H, len(rows), D).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    row_list = np.arange(Sq) if rows is None else np.asarray(rows)
    O = np.zeros((B, H, len(row_list), v.shape[3]), dtype=np.float64)
    lse = np.full((B, H, len(row_list)), -np.inf, dtype=np.float64)
    kv_idx = np.arange(Skv)[None, :]
    for b in range(B):
        for h in range(H):
            for c0 in range(0, len(row_list), chunk):
                r = row_list[c0:c0 + chunk]
                q_idx = r[:, None]
                s = scale * (q[b, h, r, :] @ k[b, h].T)
                if score_mod is not None:
                    s = score_mod(s, b, h, q_idx, kv_idx)
                live = np.broadcast_to(mask_mod(b, h, q_idx, kv_idx), s.shape)
                s = np.where(live, s, -np.inf)
                m = s.max(axis=1)
                has = np.isfinite(m)
                m_safe = np.where(has, m, 0.0)
                p = np.exp(s - m_safe[:, None])
                l_sum = p.sum(axis=1)
                o = p @ v[b, h]
                O[b, h, c0:c0 + len(r)] = np.where(has[:, None], o / np.where(has, l_sum, 1.0)[:, None], 0.0)
                lse[b, h, c0:c0 + len(r)] = np.where(has, m_safe + np.log(np.where(has, l_sum, 1.0)), -np.inf)
    return O, lse
