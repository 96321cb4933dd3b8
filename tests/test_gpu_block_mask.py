"""Block-mask builder on the GPU against the oracle's brute force: bit-exact, whole tensors."""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_common import assert_block_mask_equal, gpu_block_mask, oracle_mask_mod

pytestmark = pytest.mark.gpu

C, SW, DOC = wl.MASK_CAUSAL, wl.MASK_SLIDING_WINDOW, wl.MASK_DOCUMENT


@pytest.mark.parametrize("w", wl.WORKLOADS, ids=[w.name for w in wl.WORKLOADS])
def test_block_mask_of_each_workload(w):
    doc = wl.make_doc_ids(w)
    bm = gpu_block_mask(w.mask_kind, None, None, w.S, w.S, w.window, doc)
    ref = oracle.create_block_mask(oracle_mask_mod(w.mask_kind, w.window or None, doc), None, None,
                                   w.S, w.S)
    assert_block_mask_equal(bm, ref)


def test_block_mask_three_documents_of_the_page():
    doc = wl.three_doc_ids_from_page(8192)
    bm = gpu_block_mask(C | DOC, None, None, 8192, 8192, 0, doc)
    ref = oracle.create_block_mask(oracle_mask_mod(C | DOC, None, doc), None, None, 8192, 8192)
    assert_block_mask_equal(bm, ref)


@pytest.mark.parametrize("kind,window,Q,KV", [
    (C, 0, 1000, 1000),            # ragged edge tiles are never full
    (C, 0, 300, 700),
    (SW, 1, 512, 512),             # window one: diagonal tiles only
    (SW, 130, 640, 640),
    (C | SW, 129, 1025, 1025),
    (SW, 5000, 1024, 1024),        # window wider than the sequence: causal
    (0, 0, 384, 256),              # no mask: everything full
    (SW, 128, 512, 128),           # query rows past KV_LEN + W - 1 have no live key
])
def test_block_mask_odd_shapes(kind, window, Q, KV):
    bm = gpu_block_mask(kind, None, None, Q, KV, window)
    ref = oracle.create_block_mask(oracle_mask_mod(kind, window or None), None, None, Q, KV)
    assert_block_mask_equal(bm, ref)


@pytest.mark.parametrize("lengths", [[100, 1, 900, 23], [128, 256, 640], [1000], [7] * 50 + [650]])
@pytest.mark.parametrize("kind", [DOC, C | DOC, SW | DOC])
def test_block_mask_documents(lengths, kind):
    doc = wl.doc_ids_from_lengths(lengths)
    S = len(doc)
    bm = gpu_block_mask(kind, None, None, S, S, 200 if kind & SW else 0, doc)
    ref = oracle.create_block_mask(oracle_mask_mod(kind, 200 if kind & SW else None, doc), None, None, S, S)
    assert_block_mask_equal(bm, ref)


def test_block_mask_interleaved_document_ids():
    # Ids need not form contiguous runs: every tile then needs the element-wise path.
    rng = np.random.default_rng(7)
    doc = rng.integers(0, 3, 768).astype(np.int32)
    bm = gpu_block_mask(C | DOC, None, None, 768, 768, 0, doc)
    ref = oracle.create_block_mask(oracle_mask_mod(C | DOC, None, doc), None, None, 768, 768)
    assert_block_mask_equal(bm, ref)


@pytest.mark.parametrize("kind,window", [(C, 0), (C | SW, 300)])
def test_block_mask_without_separate_full_blocks(kind, window):
    bm = gpu_block_mask(kind, None, None, 2048, 2048, window, None, separate_full=False)
    ref = oracle.create_block_mask(oracle_mask_mod(kind, window or None), None, None, 2048, 2048,
                                   separate_full_blocks=False)
    assert_block_mask_equal(bm, ref)
    assert int(bm.full_kv_num_blocks.sum()) == 0


def test_block_mask_per_batch_and_head():
    bm = gpu_block_mask(C | SW, 2, 3, 1024, 1024, 256)
    ref = oracle.create_block_mask(oracle_mask_mod(C | SW, 256), 2, 3, 1024, 1024)
    assert_block_mask_equal(bm, ref)
