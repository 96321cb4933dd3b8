"""The backward (fa_backward: dQ, dK, dV over the block mask) on the GPU against the float64
oracle's derivative of the forward definition, on the same seeded inputs.

Tolerance, derived from the arithmetic: the kernels round P and dS once each to the 16-bit
input type (relative 2^-9 for bf16) before the tensor-core sums, accumulate in fp32, and
round the gradient once more to the input type; a gradient element therefore carries an
error of a few 2^-9 of the size of the terms it sums.  The tests bound the largest error by
2e-2 of the largest reference element and the mean error by 1e-2 of the mean reference
magnitude.  Oracle-sized cases compare every element; full-size workloads compare a whole
(b, h) slice (8k) or the rows the oracle computes from a subset of query rows (32k).
Determinism: the kernels sum in a fixed order, so repeated calls are bitwise identical.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_common import fa_module, gpu_block_mask

pytestmark = pytest.mark.gpu

C, SW, DOC = wl.MASK_CAUSAL, wl.MASK_SLIDING_WINDOW, wl.MASK_DOCUMENT
MAX_REL = 2e-2
MEAN_REL = 1e-2


def _run_gpu(w, q, k, v, do, doc=None, dq_kv_order=True, Q=None, KV=None, score=None):
    fa = fa_module()
    Q = q.shape[2] if Q is None else Q
    KV = k.shape[2] if KV is None else KV
    sk = w.score_kind if score is None else score
    doc_t = torch.from_numpy(doc).cuda() if doc is not None else None
    bm = fa.create_block_mask(w.mask_kind, None, None, Q, KV, window=w.window, doc_id=doc_t,
                              dq_kv_order=dq_kv_order)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = fa.flex_attention(qd, kd, vd, bm, score_mod=sk, softcap=w.softcap or 30.0,
                                 scale=w.scale)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, lse, dod, bm, score_mod=sk,
                                            softcap=w.softcap or 30.0, scale=w.scale)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    return dq, dk, dv, (qd, kd, vd, dod, out, lse, bm, sk)


def _oracle(w, q, k, v, do, doc=None, rows=None, score=None, b=None, h=None):
    sk = w.score_kind if score is None else score
    mm = oracle.make_mask_mod(w.mask_kind, window=w.window or None, document_id=doc)
    sm = oracle.make_score_mod(sk, H=q.shape[1], softcap=w.softcap or 30.0)
    sg = oracle.make_score_mod_grad(sk, w.softcap or 30.0)
    sl = (slice(None) if b is None else slice(b, b + 1), slice(None) if h is None else slice(h, h + 1))
    args = [t[sl].float().numpy() for t in (q, k, v, do)]
    if h is not None and sm is not None:
        # score_mods see the head index: evaluate them at head h on the one-head slice
        sm0, sg0 = sm, sg
        sm = lambda s, bb, hh, qi, ki: sm0(s, bb, h, qi, ki)
        sg = lambda s, bb, hh, qi, ki: sg0(s, bb, h, qi, ki)
    return oracle.attention_backward(*args, mm, sm, sg, scale=w.scale, rows=rows)


def _compare(got, want, what, rows_sel=None):
    g = got.float().cpu().numpy().astype(np.float64)
    if rows_sel is not None:
        g = g[rows_sel]
        want = want[rows_sel]
    err = np.abs(g - want)
    scale_max = np.abs(want).max()
    scale_mean = np.abs(want).mean()
    stats = {"what": what, "err_max": float(err.max()), "ref_max": float(scale_max),
             "err_mean": float(err.mean()), "ref_mean": float(scale_mean)}
    assert err.max() <= MAX_REL * scale_max + 1e-6, stats
    assert err.mean() <= MEAN_REL * scale_mean + 1e-7, stats
    return stats


SMALL = [
    wl.WORKLOADS[0],
    wl.WORKLOADS[1].scaled(S=1024),
    wl.WORKLOADS[2].scaled(S=1024, H=2),
    wl.WORKLOADS[3].scaled(S=1024, H=2),
    wl.WORKLOADS[4].scaled(S=1024, H=2),
    wl.Workload("nomask_d128_fp16", B=1, H=2, S=640, D=128, dtype="fp16", mask_kind=0, seed=41),
    wl.Workload("window_d64_bf16", B=2, H=1, S=768, D=64, dtype="bf16", mask_kind=C | SW,
                window=200, score_kind=wl.SCORE_ALIBI, seed=42),
    wl.Workload("softcap_d64_fp16", B=1, H=2, S=512, D=64, dtype="fp16", mask_kind=C,
                score_kind=wl.SCORE_SOFTCAP, softcap=5.0, seed=43),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name + f"_S{w.S}" for w in SMALL])
def test_backward_matches_oracle_everywhere(w):
    q, k, v = wl.make_qkv(w)
    do = wl.make_dout(w)
    doc = wl.make_doc_ids(w)
    dq, dk, dv, _ = _run_gpu(w, q, k, v, do, doc)
    rdq, rdk, rdv = _oracle(w, q, k, v, do, doc)
    _compare(dq, rdq, "dq")
    _compare(dk, rdk, "dk")
    _compare(dv, rdv, "dv")


RAGGED = [(1000, 1000, C, 0, 64, "bf16"), (300, 700, C, 0, 128, "bf16"), (700, 300, 0, 0, 64, "fp16"),
          (1000, 1000, C | DOC, 0, 128, "bf16"), (555, 555, C | SW, 100, 128, "fp16")]


@pytest.mark.parametrize("Q,KV,kind,window,D,dtype", RAGGED)
def test_backward_ragged_lengths(Q, KV, kind, window, D, dtype):
    w = wl.Workload("ragged_bwd", B=1, H=2, S=Q, D=D, dtype=dtype, mask_kind=kind, window=window, seed=44)
    g = torch.Generator().manual_seed(44 + Q + KV)
    td = wl.torch_dtype(dtype)
    q = torch.randn(1, 2, Q, D, generator=g).to(td)
    k = torch.randn(1, 2, KV, D, generator=g).to(td)
    v = torch.randn(1, 2, KV, D, generator=g).to(td)
    do = torch.randn(1, 2, Q, D, generator=g).to(td)
    doc = wl.doc_ids_from_lengths([300, 1, 450, 249]) if kind & DOC else None
    dq, dk, dv, _ = _run_gpu(w, q, k, v, do, doc)
    rdq, rdk, rdv = _oracle(w, q, k, v, do, doc)
    _compare(dq, rdq, "dq")
    _compare(dk, rdk, "dk")
    _compare(dv, rdv, "dv")


def test_backward_is_bitwise_repeatable_in_either_dq_order():
    fa = fa_module()
    w = wl.WORKLOADS[3].scaled(S=2048, H=4)
    q, k, v = wl.make_qkv(w)
    do = wl.make_dout(w)
    doc = wl.make_doc_ids(w)
    grads = {}
    for order in (True, False):
        dq, dk, dv, st = _run_gpu(w, q, k, v, do, doc, dq_kv_order=order)
        qd, kd, vd, dod, out, lse, bm, sk = st
        assert bm.info.dq_kv_order == (1 if order else 0)
        for _ in range(2):
            again = fa.flex_attention_backward(qd, kd, vd, out, lse, dod, bm, scale=w.scale)
            torch.cuda.synchronize()
            assert all(torch.equal(a, b) for a, b in zip(again, (dq, dk, dv)))
        grads[order] = (dq, dk, dv)
    # The two dQ write orders sum the same terms in another order: equal up to rounding, and
    # dK, dV (whose order does not change) bitwise.
    assert torch.equal(grads[True][1], grads[False][1]) and torch.equal(grads[True][2], grads[False][2])
    rdq = _oracle(w, q, k, v, do, doc)[0]
    for order in (True, False):
        _compare(grads[order][0], rdq, f"dq order {order}")


def test_transposed_lists_match_the_oracle():
    w = wl.WORKLOADS[3].scaled(S=2048)
    doc = wl.make_doc_ids(w)
    bm = gpu_block_mask(w.mask_kind, None, None, w.S, w.S, 0, doc)
    ref = oracle.create_block_mask(oracle.make_mask_mod(w.mask_kind, document_id=doc), None, None, w.S, w.S)
    # Column j of the tile grid: the query blocks whose tile is partial / full.
    QB = w.S // 128
    part = np.zeros((QB, QB), bool)
    full = np.zeros((QB, QB), bool)
    for i in range(QB):
        part[i, ref["kv_indices"][0, 0, i, :ref["kv_num_blocks"][0, 0, i]]] = True
        full[i, ref["full_kv_indices"][0, 0, i, :ref["full_kv_num_blocks"][0, 0, i]]] = True
    for name, m in (("q", part), ("full_q", full)):
        num = getattr(bm, f"{name}_num_blocks").cpu().numpy()[0, 0]
        idx = getattr(bm, f"{name}_indices").cpu().numpy()[0, 0]
        for j in range(QB):
            want = np.nonzero(m[:, j])[0]
            assert num[j] == len(want)
            assert np.array_equal(idx[j, :len(want)], want) and np.all(idx[j, len(want):] == 0)


def test_backward_workspace_and_argument_checks():
    fa = fa_module()
    w = wl.WORKLOADS[1].scaled(S=512, H=2)
    q, k, v = (t.cuda() for t in wl.make_qkv(w))
    bm = gpu_block_mask(C, None, None, 512, 512)
    out, lse = fa.flex_attention(q, k, v, bm)
    do = torch.randn_like(q)
    assert fa.fa_backward_workspace_bytes(1, 2, 500) == 2 * 2 * 512 * 4
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        fa.flex_attention_backward(q, k, v, out, lse, do, bm, workspace=small)
    with pytest.raises(fa.FaError) as e:
        fa.fa_backward(fa.fa_tensor(q), fa.fa_tensor(k), fa.fa_tensor(v), fa.fa_tensor(out),
                       fa.fa_tensor(do), lse.data_ptr(), bm.handle, 0, None, -1.0, fa.fa_tensor(q.clone()),
                       fa.fa_tensor(k.clone()), fa.fa_tensor(v.clone()), small.data_ptr(), 16)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    dq, dk, dv = fa.flex_attention_backward(q, k, v, out, lse, do, bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK


def test_full_size_8k_causal_one_slice():
    # The 8k causal workload in the launch configuration the bench times, one (b, h) slice
    # compared element by element.
    w = wl.WORKLOADS[1]
    q, k, v = wl.make_qkv(w)
    do = wl.make_dout(w)
    dq, dk, dv, _ = _run_gpu(w, q, k, v, do)
    h = 5
    rdq, rdk, rdv = _oracle(w, q, k, v, do, b=0, h=h)
    _compare(dq[:, h:h + 1], rdq, "dq")
    _compare(dk[:, h:h + 1], rdk, "dk")
    _compare(dv[:, h:h + 1], rdv, "dv")


@pytest.mark.parametrize("w", [wl.WORKLOADS[2], wl.WORKLOADS[3], wl.WORKLOADS[4]],
                         ids=[w.name for w in wl.WORKLOADS[2:5]])
def test_full_size_sampled_rows(w):
    q, k, v = wl.make_qkv(w)
    do = wl.make_dout(w)
    doc = wl.make_doc_ids(w)
    dq, dk, dv, _ = _run_gpu(w, q, k, v, do, doc)
    S = w.S
    b, h = w.B - 1, w.H - 1
    # dQ on sampled query rows (each needs only its own row).
    qrows = sorted({0, 1, 127, 128, S // 2, S - 129, S - 1} |
                   set(np.random.default_rng(w.seed).integers(0, S, 5).tolist()))
    rdq = _oracle(w, q, k, v, do, doc, rows=qrows, b=b, h=h)[0]
    _compare(dq[b:b + 1, h:h + 1], rdq, "dq rows", rows_sel=(0, 0, qrows))
    # dK, dV on the last 256 keys: under a causal mask only the last 256 queries see them.
    keys = np.arange(S - 256, S)
    _, rdk, rdv = _oracle(w, q, k, v, do, doc, rows=keys, b=b, h=h)
    _compare(dk[b:b + 1, h:h + 1], rdk, "dk rows", rows_sel=(0, 0, keys))
    _compare(dv[b:b + 1, h:h + 1], rdv, "dv rows", rows_sel=(0, 0, keys))


def test_backward_with_per_batch_sequence_lengths():
    # kv_lens masks keys past each batch element's own length (the mask's kv_lens); the
    # backward reads the same lengths on its partial tiles.
    fa = fa_module()
    B, H, S, D = 2, 2, 700, 64
    lens = np.array([700, 433], dtype=np.int32)
    g = torch.Generator().manual_seed(61)
    q, k, v, do = (torch.randn(B, H, S, D, generator=g).to(torch.bfloat16) for _ in range(4))
    bm = fa.create_block_mask(C, B, None, S, S, kv_lens=torch.from_numpy(lens).cuda())
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = fa.flex_attention(qd, kd, vd, bm)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, lse, dod, bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    mm = oracle.make_mask_mod(C, kv_lens=lens)
    rdq, rdk, rdv = oracle.attention_backward(*(t.float().numpy() for t in (q, k, v, do)), mm)
    _compare(dq, rdq, "dq")
    _compare(dk, rdk, "dk")
    _compare(dv, rdv, "dv")
    # Keys past a batch element's length get no gradient at all.
    assert not torch.any(dk[1, :, lens[1]:]) and not torch.any(dv[1, :, lens[1]:])


@pytest.mark.parametrize("bs", [(256, 256), (128, 384)])
def test_backward_from_kv_blocks_and_other_block_sizes(bs):
    # The kernels work on 128-wide tiles whatever BLOCK_SIZE the lists are read back at, and a
    # mask built from caller lists (BlockMask.from_kv_blocks) holds the same tiles: the
    # gradients are bitwise those of the 128 x 128 mask.
    fa = fa_module()
    Q = KV = 1536
    kind, window = C | SW, 700
    w = wl.Workload("bwd_lists", B=1, H=2, S=Q, D=64, dtype="bf16", mask_kind=kind, window=window, seed=62)
    q, k, v = (t.cuda() for t in wl.make_qkv(w))
    do = wl.make_dout(w).cuda()
    grads = []
    ref = oracle.create_block_mask(oracle.make_mask_mod(kind, window=window), None, None, Q, KV, bs)
    lists = [torch.from_numpy(np.ascontiguousarray(ref[n])).cuda()
             for n in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")]
    masks = [fa.create_block_mask(kind, None, None, Q, KV, window=window),
             fa.create_block_mask(kind, None, None, Q, KV, window=window, BLOCK_SIZE=bs),
             fa.block_mask_from_kv_blocks(*lists, Q_LEN=Q, KV_LEN=KV, BLOCK_SIZE=bs, mask_kind=kind,
                                          window=window)]
    for bm in masks:
        out, lse = fa.flex_attention(q, k, v, bm)
        grads.append(fa.flex_attention_backward(q, k, v, out, lse, do, bm))
        torch.cuda.synchronize()
        assert bm.device_status() == fa.FA_OK
    for g in grads[1:]:
        assert all(torch.equal(a, b) for a, b in zip(g, grads[0]))
    rdq, rdk, rdv = _oracle(w, *(t.cpu() for t in (q, k, v, do)))
    _compare(grads[0][0], rdq, "dq")
    _compare(grads[0][1], rdk, "dk")
    _compare(grads[0][2], rdv, "dv")
