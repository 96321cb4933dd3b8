"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something other than itself: a matrix the pages
print, a fact they state, a closed form, a library routine in a special case, or a
pure-Python brute force on tiny inputs.  The last group plants plausible mistakes in
the oracle's inputs or functors and checks that a pin catches each one.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as wl


def _load_golden(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    return np.array(rows, dtype=bool)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- masks

def test_sliding_window_T6_W3_is_the_printed_matrix(golden_dir):
    want = _load_golden(golden_dir, "sliding_window_T6_W3.txt")
    got = oracle.dense_mask(oracle.sliding_window(3), 6, 6)
    assert np.array_equal(got, want)


def test_sliding_window_last_row_reads_keys_three_to_five():
    # "Query five can read keys three, four and five."
    got = oracle.dense_mask(oracle.sliding_window(3), 6, 6)
    assert np.array_equal(got[-1], np.array([0, 0, 0, 1, 1, 1], dtype=bool))


def test_wrong_boundaries_are_rejected_by_the_printed_matrix(golden_dir):
    # The page names two wrong predicates; the fixture must tell each apart.
    want = _load_golden(golden_dir, "sliding_window_T6_W3.txt")
    i = np.arange(6)[:, None]
    j = np.arange(6)[None, :]
    one_extra_key = (i >= j) & (i - j <= 3)
    future_keys = (i - j < 3)
    assert not np.array_equal(one_extra_key, want)
    assert not np.array_equal(future_keys, want)


def test_window_one_is_self_only_and_window_ge_T_is_causal_triangle():
    T = 9
    assert np.array_equal(oracle.dense_mask(oracle.sliding_window(1), T, T), np.eye(T, dtype=bool))
    tri = np.tril(np.ones((T, T), dtype=bool))
    for W in (T, T + 1, 5 * T):
        assert np.array_equal(oracle.dense_mask(oracle.sliding_window(W), T, T), tri)
    assert np.array_equal(oracle.dense_mask(oracle.causal, T, T), tri)


@pytest.mark.parametrize("W", [1, 2, 5, 36, 37, 50])
def test_sliding_window_allowed_range_brute_force(W):
    # "allowed key indices run from max(0, i - W + 1) through i, inclusive"
    T = 37
    m = oracle.dense_mask(oracle.sliding_window(W), T, T)
    for i in range(T):
        for j in range(T):
            assert m[i, j] == (max(0, i - W + 1) <= j <= i)


def test_document_mask_brute_force():
    doc = np.array([0, 0, 0, 1, 1, 2, 2, 2, 2], dtype=np.int32)
    mm = oracle.make_mask_mod(oracle.MASK_CAUSAL | oracle.MASK_DOCUMENT, document_id=doc)
    m = oracle.dense_mask(mm, 9, 9)
    for i in range(9):
        for j in range(9):
            assert m[i, j] == (j <= i and doc[i] == doc[j])


def test_mask_kinds_combine_as_conjunction():
    T = 40
    doc = wl.doc_ids_from_lengths([7, 20, 13])
    c = oracle.dense_mask(oracle.causal, T, T)
    s = oracle.dense_mask(oracle.sliding_window(6), T, T)
    d = oracle.dense_mask(oracle.document(doc), T, T)
    got = oracle.dense_mask(oracle.make_mask_mod(7, window=6, document_id=doc), T, T)
    assert np.array_equal(got, c & s & d)
    assert oracle.dense_mask(oracle.make_mask_mod(0), 5, 7).all()


# ---------------------------------------------------------------- block metadata

def _block_mask_python_loops(pred, Q, KV, BS, separate_full):
    """Independent brute force: plain loops over tiles and elements (BS an int or a pair)."""
    BQ, BKV = BS if isinstance(BS, tuple) else (BS, BS)
    QB, KVB = -(-Q // BQ), -(-KV // BKV)
    kvn, kvi, fn, fi = [], [], [], []
    for i in range(QB):
        part, full = [], []
        for j in range(KVB):
            n_true, n_all = 0, 0
            for a in range(BQ):
                for c in range(BKV):
                    qq, kk = i * BQ + a, j * BKV + c
                    n_all += 1
                    if qq < Q and kk < KV and pred(qq, kk):
                        n_true += 1
            if n_true == 0:
                continue
            if n_true == n_all and separate_full:
                full.append(j)
            else:
                part.append(j)
        kvn.append(len(part)); fn.append(len(full))
        kvi.append(part + [0] * (KVB - len(part)))
        fi.append(full + [0] * (KVB - len(full)))
    return np.array(kvn), np.array(kvi), np.array(fn), np.array(fi)


@pytest.mark.parametrize("BS", [4, (4, 3), (2, 5)])
@pytest.mark.parametrize("separate_full", [True, False])
@pytest.mark.parametrize("case", ["causal", "swa5", "swa9", "doc", "doc_swa", "none"])
def test_block_metadata_matches_python_brute_force(case, separate_full, BS):
    Q = KV = 22           # ragged: not a multiple of the block sizes
    doc = wl.doc_ids_from_lengths([5, 3, 9, 5])
    preds = {
        "causal": (oracle.MASK_CAUSAL, None, lambda q, k: q >= k),
        "swa5": (oracle.MASK_SLIDING_WINDOW, 5, lambda q, k: 0 <= q - k < 5),
        "swa9": (oracle.MASK_CAUSAL | oracle.MASK_SLIDING_WINDOW, 9, lambda q, k: 0 <= q - k < 9),
        "doc": (oracle.MASK_DOCUMENT, None, lambda q, k: doc[q] == doc[k]),
        "doc_swa": (oracle.MASK_DOCUMENT | oracle.MASK_SLIDING_WINDOW, 3,
                    lambda q, k: doc[q] == doc[k] and 0 <= q - k < 3),
        "none": (0, None, lambda q, k: True),
    }
    kind, W, pred = preds[case]
    mm = oracle.make_mask_mod(kind, window=W, document_id=doc)
    bm = oracle.create_block_mask(mm, None, None, Q, KV, BS, separate_full)
    kvn, kvi, fn, fi = _block_mask_python_loops(pred, Q, KV, BS, separate_full)
    assert np.array_equal(bm["kv_num_blocks"][0, 0], kvn)
    assert np.array_equal(bm["kv_indices"][0, 0], kvi)
    assert np.array_equal(bm["full_kv_num_blocks"][0, 0], fn)
    assert np.array_equal(bm["full_kv_indices"][0, 0], fi)


def _counts(bm):
    p = int(bm["kv_num_blocks"].sum())
    f = int(bm["full_kv_num_blocks"].sum())
    QB = bm["kv_num_blocks"].shape[-1]
    KVB = bm["kv_indices"].shape[-1]
    return p, f, QB * KVB - p - f


def test_block_counts_causal_8k_closed_form():
    # Causal over QB blocks: QB diagonal tiles partial, QB(QB-1)/2 full, the rest dead.
    bm = oracle.create_block_mask(oracle.causal, None, None, 8192, 8192)
    assert _counts(bm) == (64, 2016, 2016)


def test_block_counts_causal_32k_closed_form():
    bm = oracle.create_block_mask(oracle.causal, None, None, 32768, 32768)
    assert _counts(bm) == (256, 32640, 32640)


def test_block_counts_sliding_window_1024_over_8k():
    # Per query block i: distance d = i - j; d = 0 and d = 8 partial, d = 1..7 full.
    mm = oracle.make_mask_mod(oracle.MASK_CAUSAL | oracle.MASK_SLIDING_WINDOW, window=1024)
    bm = oracle.create_block_mask(mm, None, None, 8192, 8192)
    p, f, d = _counts(bm)
    assert (p, f, d) == (120, 420, 3556)
    # "A 1k-token window over an 8k context leaves roughly seven-eighths of the blocks
    # fully masked" ([FA-Mac] Mask 2).
    assert abs(d / 4096 - 7 / 8) < 0.01


def test_document_packing_costs_about_a_quarter():
    # [FA-Mac] Mask 3: four packed documents cost close to a quarter of one long sequence.
    S = 8192
    doc = wl.doc_ids_from_lengths([2048] * 4)
    mm = oracle.make_mask_mod(oracle.MASK_CAUSAL | oracle.MASK_DOCUMENT, document_id=doc)
    live_doc = oracle.live_positions(mm, S, S)
    live_causal = oracle.live_positions(oracle.causal, S, S)
    assert live_causal == S * (S + 1) // 2
    assert live_doc == 4 * 2048 * 2049 // 2
    assert abs(live_doc / live_causal - 0.25) < 0.001
    bm = oracle.create_block_mask(mm, None, None, S, S)
    assert _counts(bm) == (64, 480, 3552)


def test_block_mask_broadcast_and_per_head_shapes():
    bm0 = oracle.create_block_mask(oracle.causal, None, None, 256, 256)
    bm1 = oracle.create_block_mask(oracle.causal, 2, 3, 256, 256)
    assert bm0["kv_indices"].shape == (1, 1, 2, 2)
    assert bm1["kv_indices"].shape == (2, 3, 2, 2)
    for b in range(2):
        for h in range(3):
            assert np.array_equal(bm1["kv_indices"][b, h], bm0["kv_indices"][0, 0])


# ---------------------------------------------------------------- attention

def _sdpa_f64(q, k, v, is_causal):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=is_causal).numpy()


@pytest.mark.parametrize("is_causal", [True, False])
def test_attention_matches_torch_sdpa_in_its_special_cases(is_causal):
    q, k, v = (_rand((2, 3, 70, 16), s) for s in (1, 2, 3))
    mm = oracle.causal if is_causal else oracle.all_true
    O, lse = oracle.attention(q, k, v, mm)
    assert np.abs(O - _sdpa_f64(q, k, v, is_causal)).max() < 1e-12


def test_window_one_gives_v_and_lse_the_diagonal_score():
    # [SWA]: W = 1 permits only self-attention; softmax over one entry is exactly 1.
    q, k, v = (_rand((1, 2, 33, 8), s) for s in (4, 5, 6))
    O, lse = oracle.attention(q, k, v, oracle.sliding_window(1), scale=0.3)
    assert np.array_equal(O, v)
    s_ii = 0.3 * np.einsum("bhsd,bhsd->bhs", q, k)
    assert np.abs(lse - s_ii).max() < 1e-12


def test_document_packed_equals_each_document_alone():
    # [FA-Mac] Mask 3: no cross-contamination between packed documents.
    lengths = [13, 30, 21]
    doc = wl.doc_ids_from_lengths(lengths)
    S = sum(lengths)
    q, k, v = (_rand((1, 2, S, 8), s) for s in (7, 8, 9))
    mm = oracle.make_mask_mod(oracle.MASK_CAUSAL | oracle.MASK_DOCUMENT, document_id=doc)
    O, lse = oracle.attention(q, k, v, mm)
    start = 0
    for L in lengths:
        sl = slice(start, start + L)
        Od, lsed = oracle.attention(q[:, :, sl], k[:, :, sl], v[:, :, sl], oracle.causal)
        assert np.abs(O[:, :, sl] - Od).max() < 1e-12
        assert np.abs(lse[:, :, sl] - lsed).max() < 1e-12
        start += L


def test_masked_positions_do_not_change_the_output():
    # [SWA] "Build and apply the mask": the last query cannot read row zero.
    T, W = 24, 5
    q, k, v = (_rand((1, 1, T, 8), s) for s in (10, 11, 12))
    O, _ = oracle.attention(q, k, v, oracle.sliding_window(W))
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, :T - W] += 3.0
    v2[0, 0, :T - W] -= 5.0
    O2, _ = oracle.attention(q, k2, v2, oracle.sliding_window(W))
    assert np.array_equal(O[0, 0, -1], O2[0, 0, -1])


def test_lse_normalises_the_live_probabilities():
    q, k, v = (_rand((1, 2, 50, 8), s) for s in (13, 14, 15))
    doc = wl.doc_ids_from_lengths([20, 30])
    mm = oracle.make_mask_mod(7, window=9, document_id=doc)
    sm = oracle.make_score_mod(oracle.SCORE_SOFTCAP | oracle.SCORE_ALIBI, H=2, softcap=5.0)
    O, lse = oracle.attention(q, k, v, mm, sm, scale=0.7)
    qi, ki = np.arange(50)[:, None], np.arange(50)[None, :]
    for h in range(2):
        s = sm(0.7 * q[0, h] @ k[0, h].T, 0, h, qi, ki)
        s = np.where(oracle.dense_mask(mm, 50, 50), s, -np.inf)
        assert np.abs(np.exp(s - lse[0, h][:, None]).sum(axis=1) - 1.0).max() < 1e-12


def test_rows_subset_equals_full_computation():
    q, k, v = (_rand((1, 2, 40, 8), s) for s in (16, 17, 18))
    mm = oracle.sliding_window(7)
    O, lse = oracle.attention(q, k, v, mm)
    rows = [0, 5, 39, 17]
    Or, lser = oracle.attention(q, k, v, mm, rows=rows)
    assert np.array_equal(Or, O[:, :, rows])
    assert np.array_equal(lser, lse[:, :, rows])


def test_row_with_no_live_key_gives_zero_and_minus_inf():
    q, k, v = (_rand((1, 1, 6, 4), s) for s in (19, 20, 21))

    def none_for_row_two(b, h, qi, ki):
        return np.broadcast_to(qi != 2, np.broadcast(qi, ki).shape) & (qi >= ki)
    O, lse = oracle.attention(q, k, v, none_for_row_two)
    assert np.all(O[0, 0, 2] == 0) and lse[0, 0, 2] == -np.inf
    assert np.isfinite(lse[0, 0, [0, 1, 3, 4, 5]]).all()


# ---------------------------------------------------------------- score mods

def test_soft_cap_with_huge_cap_is_no_score_mod():
    q, k, v = (_rand((1, 2, 30, 8), s) for s in (22, 23, 24))
    O0, l0 = oracle.attention(q, k, v, oracle.causal)
    O1, l1 = oracle.attention(q, k, v, oracle.causal, oracle.soft_cap(1e6))
    assert np.abs(O0 - O1).max() < 1e-9 and np.abs(l0 - l1).max() < 1e-9


def test_soft_cap_bounds_scores_and_keeps_the_live_set():
    sm = oracle.soft_cap(30.0)
    s = np.array([-1e4, -31.0, -1.0, 0.0, 1e-3, 2.0, 29.0, 1e5])
    out = sm(s, 0, 0, 0, 0)
    assert np.all(np.abs(out) <= 30.0) and np.all(np.diff(out) > 0)
    assert out[3] == 0.0 and abs(out[4] - 1e-3) < 1e-9


def test_alibi_slopes_for_eight_heads_are_powers_of_two():
    assert np.array_equal(oracle.alibi_slopes(8), 2.0 ** -np.arange(1, 9))


def test_alibi_matches_a_hand_written_bias_matrix():
    # T = 4, H = 2, slopes 1/2 and 1/16: bias[h, i, j] = slope_h * (j - i), written out by
    # hand; below the diagonal (the keys a causal mask keeps) every entry is <= 0.
    bias = {
        0: [[0, .5, 1, 1.5], [-.5, 0, .5, 1], [-1, -.5, 0, .5], [-1.5, -1, -.5, 0]],
        1: [[0, 1 / 16, 2 / 16, 3 / 16], [-1 / 16, 0, 1 / 16, 2 / 16],
            [-2 / 16, -1 / 16, 0, 1 / 16], [-3 / 16, -2 / 16, -1 / 16, 0]],
    }
    sm = oracle.alibi([0.5, 1 / 16])
    qi, ki = np.arange(4)[:, None], np.arange(4)[None, :]
    for h in (0, 1):
        assert np.array_equal(sm(np.zeros((4, 4)), 0, h, qi, ki), np.array(bias[h]))


# Soft-cap then ALiBi ("Bonus: a score_mod for soft-capping" for the cap; the bias is the
# additive distance penalty of "The two hooks"; the order is the stated reading: cap first,
# then add slope_h * (kv_idx - q_idx)).  Scores are chosen as s = cap * ln(a), where
# tanh(ln a) = (a^2 - 1) / (a^2 + 1) exactly, so every expected value is a rational closed
# form computed here without a tanh; the H = 8 slopes are 2^-(h+1).
_COMPOSE_A = [Fraction(1), Fraction(2), Fraction(3), Fraction(1, 3), Fraction(1, 10), Fraction(1000)]
_COMPOSE_H = [0, 3, 7]
_COMPOSE_DIST = [0, 1, 37, 16383]          # q_idx - kv_idx >= 0: keys a causal mask keeps


def _compose_table(cap=30):
    rows = []
    for a in _COMPOSE_A:
        capped = Fraction(cap) * (a * a - 1) / (a * a + 1)
        for h in _COMPOSE_H:
            for d in _COMPOSE_DIST:
                rows.append((cap * math.log(float(a)), h, d,
                             float(capped - Fraction(d, 2 ** (h + 1)))))
    return rows


def _apply(sm, s, h, d):
    q_idx = np.array([[d + 5]])
    kv_idx = np.array([[5]])
    return float(sm(np.array([[s]]), 0, h, q_idx, kv_idx)[0, 0])


def test_soft_cap_then_alibi_matches_closed_forms():
    sm = oracle.make_score_mod(oracle.SCORE_SOFTCAP | oracle.SCORE_ALIBI, H=8, softcap=30.0)
    for s, h, d, want in _compose_table():
        got = _apply(sm, s, h, d)
        assert abs(got - want) <= 1e-12 * max(1.0, abs(want)), (s, h, d, got, want)


def test_composition_pin_catches_the_bias_inside_the_tanh():
    slopes = oracle.alibi_slopes(8)
    wrong = lambda s, b, h, qi, ki: 30.0 * np.tanh((s + slopes[h] * (ki - qi)) / 30.0)
    bad = [abs(_apply(wrong, s, h, d) - want) > 1e-6 for s, h, d, want in _compose_table()]
    assert any(bad) and sum(bad) >= len(bad) // 2


def test_composition_pin_catches_the_cap_applied_after_the_bias():
    wrong = oracle.compose_score_mods(oracle.alibi(oracle.alibi_slopes(8)), oracle.soft_cap(30.0))
    bad = [abs(_apply(wrong, s, h, d) - want) > 1e-6 for s, h, d, want in _compose_table()]
    assert any(bad) and sum(bad) >= len(bad) // 2


def test_composition_pin_catches_a_slope_of_the_wrong_head():
    shifted = np.concatenate([[1.0], oracle.alibi_slopes(8)[:-1]])    # 2^-h instead of 2^-(h+1)
    wrong = oracle.compose_score_mods(oracle.soft_cap(30.0), oracle.alibi(shifted))
    assert any(abs(_apply(wrong, s, h, d) - want) > 1e-6 for s, h, d, want in _compose_table())


def test_score_mod_only_changes_live_values():
    # [FA-Mac] "The two hooks": the score_mod changes values, never sparsity.
    q, k, v = (_rand((1, 2, 40, 8), s) for s in (25, 26, 27))
    mm = oracle.sliding_window(6)
    sm = oracle.make_score_mod(3, H=2, softcap=4.0)
    O, lse = oracle.attention(q, k, v, mm, sm)
    k2 = k.copy()
    k2[0, :, :10] += 7.0
    O2, _ = oracle.attention(q, k2, v, mm, sm)
    assert np.array_equal(O[:, :, 16:], O2[:, :, 16:])


# ---------------------------------------------------------------- workload generators

def test_document_lengths_of_the_packed_workload():
    w = wl.WORKLOADS[3]
    lens = wl.doc_lengths(w.S, w.n_docs, 512, w.seed)
    assert len(lens) == 4 and sum(lens) == 8192 and min(lens) >= 512
    ids = wl.make_doc_ids(w)
    assert ids.shape == (8192,) and ids.dtype == np.int32
    assert np.array_equal(np.unique(ids), np.arange(4))
    assert np.all(np.diff(ids) >= 0)
    # The stated recipe: three sorted cuts from default_rng(4).integers(0, 6145, 3), the gaps
    # of [0, cuts, 6144], each plus 512.
    cuts = np.sort(np.random.default_rng(4).integers(0, 6145, 3))
    edges = np.concatenate([[0], cuts, [6144]])
    assert list(lens) == [int(g) + 512 for g in np.diff(edges)] == [4975, 1465, 891, 861]


def test_three_document_example_of_the_page():
    d = wl.three_doc_ids_from_page()
    assert d[2047] == 0 and d[2048] == 1 and d[4999] == 1 and d[5000] == 2


def test_qkv_generation_is_seeded():
    w = wl.WORKLOADS[0]
    a = wl.make_qkv(w)
    b = wl.make_qkv(w)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert a[0].dtype == torch.float16 and a[0].shape == (1, 2, 512, 64)
    assert not torch.equal(a[0], a[1])


# ---------------------------------------------------------------- planted mistakes

def test_pin_catches_a_dropped_scale():
    q, k, v = (_rand((1, 2, 30, 16), s) for s in (1, 2, 3))
    O, _ = oracle.attention(q, k, v, oracle.causal, scale=1.0)
    assert np.abs(O - _sdpa_f64(q, k, v, True)).max() > 1e-3


def test_pin_catches_swapped_k_and_v():
    q, k, v = (_rand((1, 2, 30, 16), s) for s in (1, 2, 3))
    O, _ = oracle.attention(q, v, k, oracle.causal)
    assert np.abs(O - _sdpa_f64(q, k, v, True)).max() > 1e-3


def test_pin_catches_a_flipped_alibi_sign():
    sm = oracle.alibi([-0.5, -1 / 16])
    qi, ki = np.arange(4)[:, None], np.arange(4)[None, :]
    assert sm(np.zeros((4, 4)), 0, 0, qi, ki)[1, 0] != -0.5


def test_pin_catches_an_off_by_one_window():
    # A window that also lets key i - W through breaks the brute-force range check.
    T, W = 12, 4
    wrong = oracle.dense_mask(oracle.sliding_window(W + 1), T, T)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    assert not np.array_equal(wrong, (j >= np.maximum(0, i - W + 1)) & (j <= i))


def test_pin_catches_a_mask_applied_before_the_soft_cap():
    # Masking with -inf and then soft-capping turns dead keys into -cap, which leaks weight:
    # the lse identity over live entries then fails.
    q, k, v = (_rand((1, 1, 20, 8), s) for s in (31, 32, 33))
    cap = 2.0
    s = 0.5 * q[0, 0] @ k[0, 0].T
    live = oracle.dense_mask(oracle.causal, 20, 20)
    wrong = cap * np.tanh(np.where(live, s, -np.inf) / cap)
    p = np.exp(wrong - wrong.max(axis=1, keepdims=True))
    leaked = p[~live].sum()
    assert leaked > 1e-3
    _, lse = oracle.attention(q, k, v, oracle.causal, oracle.soft_cap(cap), scale=0.5)
    right = np.where(live, cap * np.tanh(s / cap), -np.inf)
    assert np.abs(np.exp(right - lse[0, 0][:, None]).sum(axis=1) - 1).max() < 1e-12
    assert math.isfinite(float(lse[0, 0, 0]))


# ---------------------------------------------------------------- per-batch sequence lengths

def test_sequence_lengths_brute_force():
    mm = oracle.sequence_lengths([3, 7])
    for b, L in ((0, 3), (1, 7)):
        m = oracle.dense_mask(mm, 5, 9, b=b)
        assert np.array_equal(m, np.array([[kv < L for kv in range(9)] for _ in range(5)]))


def test_sequence_lengths_equal_truncated_keys():
    # A batch element with length L attends exactly as if its K, V had L rows.
    q, k, v = (_rand((2, 2, 12, 8), s) for s in (61, 62, 63))
    lens = [5, 12]
    mm = oracle.make_mask_mod(oracle.MASK_CAUSAL | oracle.MASK_SLIDING_WINDOW, window=4, kv_lens=lens)
    O, L = oracle.attention(q, k, v, mm)
    for b, n in enumerate(lens):
        base = oracle.make_mask_mod(oracle.MASK_CAUSAL | oracle.MASK_SLIDING_WINDOW, window=4)
        Ob, Lb = oracle.attention(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], base)
        assert np.abs(O[b:b + 1] - Ob).max() < 1e-12
        fin = np.isfinite(Lb)
        assert np.array_equal(np.isfinite(L[b:b + 1]), fin) and np.abs(L[b:b + 1][fin] - Lb[fin]).max() < 1e-12


def test_block_metadata_with_sequence_lengths_is_per_batch():
    lens = [300, 1000, 129]
    mm = oracle.make_mask_mod(oracle.MASK_CAUSAL, kv_lens=lens)
    bm = oracle.create_block_mask(mm, 3, None, 1000, 1000)
    for b, n in enumerate(lens):
        one = oracle.create_block_mask(oracle.causal, None, None, 1000, n)
        kvb = one["kv_indices"].shape[-1]
        for key in ("kv_num_blocks", "full_kv_num_blocks"):
            assert np.array_equal(bm[key][b, 0], one[key][0, 0])
        for key in ("kv_indices", "full_kv_indices"):
            assert np.array_equal(bm[key][b, 0, :, :kvb], one[key][0, 0])
            assert np.all(bm[key][b, 0, :, kvb:] == 0)
