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


def _oracle_transposed(ref):
    """Per kv block, the query blocks whose tile is partial / full, from the oracle's lists."""
    QB, KVB = ref["kv_indices"].shape[2], ref["kv_indices"].shape[3]
    out = {}
    for which, num, idx in (("q", "kv_num_blocks", "kv_indices"), ("full_q", "full_kv_num_blocks", "full_kv_indices")):
        m = np.zeros((QB, KVB), bool)
        for i in range(QB):
            m[i, ref[idx][0, 0, i, :ref[num][0, 0, i]]] = True
        n = m.sum(axis=0).astype(np.int32)
        lists = np.zeros((KVB, QB), np.int32)
        for j in range(KVB):
            r = np.nonzero(m[:, j])[0]
            lists[j, :len(r)] = r
        out[f"{which}_num_blocks"], out[f"{which}_indices"] = n, lists
    return out


BLOCK_PAIRS = [
    (C, 0, 1000, 1000, (256, 128)),
    (C | SW, 300, 1536, 1536, (64, 192)),
    (C | DOC, 0, 2048, 2048, (128, 256)),
    (C, 0, 700, 1100, (100, 50)),
    (SW, 129, 1025, 1025, (512, 512)),
]


@pytest.mark.parametrize("kind,window,Q,KV,bs", BLOCK_PAIRS)
def test_block_size_pairs_match_the_oracle(kind, window, Q, KV, bs):
    # "create_block_mask", Parameters: BLOCK_SIZE is an int or a (q, kv) tuple.  The lists read
    # back are at that size; the forward walks its own 128 x 128 tiles, so its result is the
    # same bit for bit as with the default block size.
    import torch
    fa = __import__("block_sparse_masked_x128_b200")
    doc = wl.doc_ids_from_lengths([700, 1, 900, 447]) if kind & DOC else None
    doc_t = torch.from_numpy(doc).cuda() if doc is not None else None
    bm = fa.create_block_mask(kind, None, None, Q, KV, window=window, doc_id=doc_t, BLOCK_SIZE=bs)
    assert (bm.info.BLOCK_SIZE, bm.info.KV_BLOCK_SIZE) == bs
    ref = oracle.create_block_mask(oracle_mask_mod(kind, window or None, doc), None, None, Q, KV, bs)
    assert_block_mask_equal(bm, ref)
    tr = _oracle_transposed(ref)
    for name, want in tr.items():
        assert np.array_equal(getattr(bm, name).cpu().numpy()[0, 0], want), name
    g = torch.Generator().manual_seed(51)
    q = torch.randn(1, 2, Q, 64, generator=g).to(torch.bfloat16).cuda()
    k, v = (torch.randn(1, 2, KV, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(2))
    base = gpu_block_mask(kind, None, None, Q, KV, window, doc)
    a = fa.flex_attention(q, k, v, bm)
    b = fa.flex_attention(q, k, v, base)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def _upload(ref):
    import torch
    return [torch.from_numpy(np.ascontiguousarray(ref[n])).cuda()
            for n in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")]


@pytest.mark.parametrize("bs,with_full", [((128, 128), True), ((256, 256), True), ((256, 128), False),
                                          ((128, 384), True)])
def test_from_kv_blocks_runs_the_same_attention(bs, with_full):
    # BlockMask.from_kv_blocks: caller lists at a block size that is a multiple of 128 become the
    # kernels' tiles; the mask_mod is applied on partial tiles, so the attention is the mask's.
    import torch
    from gpu_common import compare, run_oracle
    fa = __import__("block_sparse_masked_x128_b200")
    Q = KV = 1536
    kind, window = C | SW, 700
    ref = oracle.create_block_mask(oracle_mask_mod(kind, window), None, None, Q, KV, bs)
    kvn, kvi, fn, fi = _upload(ref)
    if with_full:
        bm = fa.block_mask_from_kv_blocks(kvn, kvi, fn, fi, Q_LEN=Q, KV_LEN=KV, BLOCK_SIZE=bs,
                                          mask_kind=kind, window=window)
    else:   # every live block listed as partial
        ref_all = oracle.create_block_mask(oracle_mask_mod(kind, window), None, None, Q, KV, bs,
                                           separate_full_blocks=False)
        kvn, kvi = _upload(ref_all)[:2]
        bm = fa.block_mask_from_kv_blocks(kvn, kvi, Q_LEN=Q, KV_LEN=KV, BLOCK_SIZE=bs,
                                          mask_kind=kind, window=window)
    torch.cuda.synchronize()
    assert torch.equal(bm.kv_indices, kvi) and torch.equal(bm.kv_num_blocks, kvn)
    w = wl.Workload("from_kv_blocks", B=1, H=2, S=Q, D=128, dtype="bf16", mask_kind=kind,
                    window=window, seed=52)
    q, k, v = wl.make_qkv(w)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)
    if with_full and bs == (128, 128):
        b2 = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), gpu_block_mask(kind, None, None, Q, KV, window))
        assert torch.equal(out, b2[0]) and torch.equal(lse, b2[1])


def test_from_kv_blocks_reports_lists_out_of_range():
    import torch
    fa = __import__("block_sparse_masked_x128_b200")
    ref = oracle.create_block_mask(oracle.causal, None, None, 512, 512, 128)
    kvn, kvi, fn, fi = _upload(ref)
    kvi[0, 0, 3, 0] = 9            # kv block 9 of 4
    bm = fa.block_mask_from_kv_blocks(kvn, kvi, fn, fi, Q_LEN=512, KV_LEN=512, mask_kind=C)
    assert bm.device_status() == fa.FA_ERR_INVALID_ARG
    assert bm.device_status() == fa.FA_OK      # read and cleared
