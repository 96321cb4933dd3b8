"""Fused forward on the GPU against the float64 oracle on the same seeded inputs.

Oracle-sized cases compare every output element; full-size workloads (in the launch
configuration the benchmark times) compare sampled query rows the oracle computes one by
one.  Bit-exact checks cover what the method fixes exactly: a window of one returns V, keys
outside a row's mask cannot change it, packed documents equal separate runs, and the
separate_full_blocks setting does not change the arithmetic.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_common import compare, fa_module, gpu_block_mask, run_gpu, run_oracle, workload_inputs

pytestmark = pytest.mark.gpu

C, SW, DOC = wl.MASK_CAUSAL, wl.MASK_SLIDING_WINDOW, wl.MASK_DOCUMENT

# Oracle-sized versions of the five workloads (several tiles and pairs, ragged doc edges).
SMALL = [
    wl.WORKLOADS[0],
    wl.WORKLOADS[1].scaled(S=1024),
    wl.WORKLOADS[2].scaled(S=2048, H=4),
    wl.WORKLOADS[3].scaled(S=2048, H=4),
    wl.WORKLOADS[4].scaled(S=2048),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name + f"_S{w.S}" for w in SMALL])
def test_forward_matches_oracle_everywhere(w):
    q, k, v = wl.make_qkv(w)
    doc = wl.make_doc_ids(w)
    out, lse, _ = run_gpu(w, q, k, v, doc)
    O, L = run_oracle(w, q, k, v, doc)
    compare(out, lse, O, L)


def _sample_rows(S, seed, n_random=8):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, 255, 256, S // 2 - 1, S // 2, S - 129, S - 128, S - 2, S - 1]
    return sorted(set(fixed) | set(rng.integers(0, S, n_random).tolist()))


@pytest.mark.parametrize("w", wl.WORKLOADS, ids=[w.name for w in wl.WORKLOADS])
def test_forward_full_size_sampled_rows(w):
    q, k, v, doc = workload_inputs(w)
    out, lse, _ = run_gpu(w, q, k, v, doc)
    rows = _sample_rows(w.S, w.seed)
    if doc is not None:   # rows around every document boundary
        starts = np.flatnonzero(np.diff(doc)) + 1
        rows = sorted(set(rows) | {int(s) + d for s in starts for d in (-1, 0, 1)})
    O, L = run_oracle(w, q, k, v, doc, rows=rows)
    compare(out, lse, O, L, rows=rows)


@pytest.mark.parametrize("w", wl.WORKLOADS, ids=[w.name for w in wl.WORKLOADS])
def test_forward_full_size_one_whole_slice(w):
    # Every row of one (b, h) slice at the workload's full size, in the launch configuration
    # the benchmark times (all heads run; the last (b, h) is compared): a schedule or counter
    # error confined to a few units would show here even where sampled rows miss it.
    q, k, v, doc = workload_inputs(w)
    out, lse, _ = run_gpu(w, q, k, v, doc)
    b, h = w.B - 1, w.H - 1
    sl = (slice(b, b + 1), slice(h, h + 1))
    mm = oracle.make_mask_mod(w.mask_kind, window=w.window or None, document_id=doc)
    sm0 = oracle.make_score_mod(w.score_kind, H=w.H, softcap=w.softcap or 30.0)
    sm = (lambda s, bb, hh, qi, ki: sm0(s, bb, h, qi, ki)) if sm0 else None
    O, L = oracle.attention(q[sl].float().numpy(), k[sl].float().numpy(), v[sl].float().numpy(), mm, sm,
                            scale=w.scale)
    compare(out[sl], lse[sl], O, L)


@pytest.mark.parametrize("D,dtype", [(64, torch.float16), (64, torch.bfloat16), (128, torch.bfloat16),
                                     (128, torch.float16)])
def test_window_one_returns_v_exactly(D, dtype):
    fa = fa_module()
    g = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(2, 3, 512, D, generator=g).to(dtype).cuda() for _ in range(3))
    bm = gpu_block_mask(SW, None, None, 512, 512, 1)
    out, lse = fa.flex_attention(q, k, v, bm)
    assert torch.equal(out, v)
    s_ii = (q.double() * k.double()).sum(-1) / np.sqrt(D)
    assert (lse.double() - s_ii).abs().max().item() < 1e-4


def test_keys_outside_the_window_cannot_change_a_row():
    # "The last query cannot read row zero through this single layer."
    fa = fa_module()
    w = wl.WORKLOADS[0]
    q, k, v = (t.cuda() for t in wl.make_qkv(w))
    bm = gpu_block_mask(w.mask_kind, None, None, 512, 512, w.window)
    out, lse = fa.flex_attention(q, k, v, bm, scale=w.scale)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, :256] += 3.0           # rows >= 384 see only keys 257..511
    v2[:, :, :256] -= 5.0
    out2, lse2 = fa.flex_attention(q, k2, v2, bm, scale=w.scale)
    assert torch.equal(out[:, :, 384:], out2[:, :, 384:])
    assert torch.equal(lse[:, :, 384:], lse2[:, :, 384:])
    assert not torch.equal(out[:, :, :256], out2[:, :, :256])


def test_packed_documents_equal_separate_runs():
    fa = fa_module()
    lengths = [256, 384, 128, 256]
    doc = wl.doc_ids_from_lengths(lengths)
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(1, 4, 1024, 128, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    bm = gpu_block_mask(C | DOC, None, None, 1024, 1024, 0, doc)
    out, lse = fa.flex_attention(q, k, v, bm)
    start = 0
    for L in lengths:
        sl = slice(start, start + L)
        bmd = gpu_block_mask(C, None, None, L, L)
        od, ld = fa.flex_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                   v[:, :, sl].contiguous(), bmd)
        assert torch.equal(out[:, :, sl], od)
        assert torch.equal(lse[:, :, sl], ld)
        start += L


@pytest.mark.parametrize("kind,window", [(C, 0), (C | SW, 300), (C | DOC, 0)])
def test_separate_full_blocks_does_not_change_the_result(kind, window):
    # Without separate full blocks every live tile is masked like a partial one (and takes
    # the MUFU exp2 path), so the two results agree to rounding, each within tolerance.
    fa = fa_module()
    doc = wl.doc_ids_from_lengths([700, 900, 448]) if kind & DOC else None
    w = wl.Workload("separate_full", B=1, H=2, S=2048, D=64, dtype="bf16", mask_kind=kind,
                    window=window, seed=6)
    q, k, v = wl.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    a = fa.flex_attention(qd, kd, vd, gpu_block_mask(kind, None, None, 2048, 2048, window, doc, True))
    b = fa.flex_attention(qd, kd, vd, gpu_block_mask(kind, None, None, 2048, 2048, window, doc, False))
    O, L = run_oracle(w, q, k, v, doc)
    compare(a[0], a[1], O, L)
    compare(b[0], b[1], O, L)
    assert (a[0].float() - b[0].float()).abs().max().item() < 1e-2


def test_strided_layout_equals_contiguous():
    fa = fa_module()
    g = torch.Generator().manual_seed(8)
    base = [torch.randn(2, 768, 3, 128, generator=g).to(torch.bfloat16).cuda() for _ in range(3)]
    q, k, v = (t.transpose(1, 2) for t in base)            # (B, H, S, D) views, S stride H*D
    bm = gpu_block_mask(C, None, None, 768, 768)
    out_view = torch.empty(2, 768, 3, 128, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o1, l1 = fa.flex_attention(q, k, v, bm, out=out_view)
    o2, l2 = fa.flex_attention(q.contiguous(), k.contiguous(), v.contiguous(), bm)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_rows_without_live_keys_give_zero_and_minus_inf():
    w = wl.Workload("swa128_q512_kv128", B=1, H=2, S=512, D=64, dtype="bf16",
                    mask_kind=SW, window=128, seed=21)
    fa = fa_module()
    g = torch.Generator().manual_seed(21)
    q = torch.randn(1, 2, 512, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, 128, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 128, 64, generator=g).to(torch.bfloat16)
    bm = gpu_block_mask(SW, None, None, 512, 128, 128)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm)
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)
    assert torch.all(out[:, :, 255:] == 0) and torch.all(torch.isinf(lse[:, :, 255:]))


@pytest.mark.parametrize("Q,KV,kind,window", [(256, 640, C, 0), (640, 256, C, 0), (384, 1024, SW, 200)])
def test_query_and_key_lengths_may_differ(Q, KV, kind, window):
    w = wl.Workload("qkv_lengths", B=1, H=2, S=Q, D=128, dtype="bf16", mask_kind=kind,
                    window=window, seed=22)
    fa = fa_module()
    g = torch.Generator().manual_seed(22)
    q = torch.randn(1, 2, Q, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, KV, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, KV, 128, generator=g).to(torch.bfloat16)
    bm = gpu_block_mask(kind, None, None, Q, KV, window)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm)
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)


RAGGED = [
    (1000, 1000, C, 0, 64, "bf16", wl.SCORE_NONE, None),
    (4097, 4097, C, 0, 128, "bf16", wl.SCORE_NONE, None),
    (300, 700, C, 0, 128, "fp16", wl.SCORE_NONE, None),
    (300, 700, C | SW, 100, 64, "fp16", wl.SCORE_NONE, None),
    (1, 2000, 0, 0, 128, "bf16", wl.SCORE_NONE, None),
    (17, 333, C, 0, 64, "bf16", wl.SCORE_NONE, None),
    (1000, 1000, C | DOC, 0, 128, "bf16", wl.SCORE_NONE, [300, 1, 450, 249]),
    (777, 777, C, 0, 128, "bf16", wl.SCORE_SOFTCAP | wl.SCORE_ALIBI, None),
]


@pytest.mark.parametrize("Q,KV,kind,window,D,dtype,score,doc_lens", RAGGED,
                         ids=[f"q{r[0]}_kv{r[1]}_m{r[2]}_d{r[4]}_{r[5]}_s{r[6]}" for r in RAGGED])
def test_ragged_lengths(Q, KV, kind, window, D, dtype, score, doc_lens):
    # Lengths that are not multiples of 128: the last tile is loaded zero-filled, keys past
    # KV_LEN are masked and rows past Q_LEN are not stored.
    w = wl.Workload("ragged", B=2, H=2, S=Q, D=D, dtype=dtype, mask_kind=kind, window=window,
                    score_kind=score, softcap=30.0, seed=28)
    fa = fa_module()
    g = torch.Generator().manual_seed(28 + Q + KV)
    td = wl.torch_dtype(dtype)
    q = torch.randn(2, 2, Q, D, generator=g).to(td)
    k = torch.randn(2, 2, KV, D, generator=g).to(td)
    v = torch.randn(2, 2, KV, D, generator=g).to(td)
    doc = wl.doc_ids_from_lengths(doc_lens) if doc_lens else None
    bm = gpu_block_mask(kind, None, None, Q, KV, window, doc)
    out = torch.full((2, 2, Q, D), 7.0, dtype=td, device="cuda")   # rows the kernel skips stay 7
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=score, softcap=30.0,
                                 out=out)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    O, L = run_oracle(w, q, k, v, doc)
    compare(out, lse, O, L)


def test_per_head_mask_equals_broadcast_mask():
    fa = fa_module()
    g = torch.Generator().manual_seed(9)
    q, k, v = (torch.randn(2, 3, 1024, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    a = fa.flex_attention(q, k, v, gpu_block_mask(C | SW, None, None, 1024, 1024, 256))
    b = fa.flex_attention(q, k, v, gpu_block_mask(C | SW, 2, 3, 1024, 1024, 256))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("score_kind", [wl.SCORE_SOFTCAP, wl.SCORE_ALIBI, wl.SCORE_SOFTCAP | wl.SCORE_ALIBI])
@pytest.mark.parametrize("D,dtype", [(64, "fp16"), (64, "bf16"), (128, "bf16"), (128, "fp16")])
def test_score_mods(score_kind, D, dtype):
    w = wl.Workload("score_mods", B=1, H=4, S=768, D=D, dtype=dtype, mask_kind=C,
                    score_kind=score_kind, softcap=5.0, seed=23)
    q, k, v = wl.make_qkv(w)
    q = q * 3   # large enough scores for the cap to bend them
    out, lse, _ = run_gpu(w, q, k, v)
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)


@pytest.mark.parametrize("D", [64, 128])
def test_softcap_polynomial_and_mufu_paths_in_one_tile(D):
    # A warp takes tanh from its polynomial when every |s / cap| of its 32 rows in a tile is at
    # most 0.2, else from tanh.approx.  At cap 30 unscaled N(0, 1) scores stay under the bound;
    # query rows scaled by 4 in every other 32-row group push their warps past it, so both paths
    # run side by side in every tile.
    w = wl.Workload("softcap_mix", B=1, H=2, S=1024, D=D, dtype="bf16", mask_kind=C,
                    score_kind=wl.SCORE_SOFTCAP | wl.SCORE_ALIBI, softcap=30.0, seed=29)
    q, k, v = wl.make_qkv(w)
    rows = (torch.arange(w.S) // 32) % 2 == 1
    q[:, :, rows, :] *= 4
    out, lse, _ = run_gpu(w, q, k, v)
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)


def test_explicit_alibi_slopes():
    fa = fa_module()
    w = wl.Workload("alibi_slopes", B=1, H=4, S=512, D=128, dtype="bf16", mask_kind=C,
                    score_kind=wl.SCORE_ALIBI, seed=24)
    q, k, v = wl.make_qkv(w)
    slopes = np.array([0.3, 0.05, 1.0, 0.0], dtype=np.float32)
    bm = gpu_block_mask(C, None, None, 512, 512)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, score_mod=wl.SCORE_ALIBI,
                                 alibi_slopes=torch.from_numpy(slopes).cuda())
    sm = oracle.alibi(slopes.astype(np.float64))
    O, L = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), oracle.causal, sm)
    compare(out, lse, O, L)


def test_lse_may_be_omitted_and_runs_are_deterministic():
    fa = fa_module()
    w = wl.WORKLOADS[1].scaled(S=1024, H=4)
    q, k, v = (t.cuda() for t in wl.make_qkv(w))
    bm = gpu_block_mask(C, None, None, 1024, 1024)
    o1, _ = fa.flex_attention(q, k, v, bm, return_lse=False)
    o2, l2 = fa.flex_attention(q, k, v, bm)
    assert torch.equal(o1, o2)
    o3, l3 = fa.flex_attention(q, k, v, bm)
    assert torch.equal(o2, o3) and torch.equal(l2, l3)


def test_forwards_on_one_mask_from_two_streams():
    # Each launch takes its own pair of the mask's work-distribution counters, so forwards
    # that share a mask may overlap on different streams.
    fa = fa_module()
    g = torch.Generator().manual_seed(12)
    q, k, v = (torch.randn(1, 8, 2048, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    bm = gpu_block_mask(C, None, None, 2048, 2048)
    o_ref, l_ref = fa.flex_attention(q, k, v, bm)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for i in range(8):
        st = streams[i % 2]
        with torch.cuda.stream(st):
            out = torch.empty_like(q)
            lse = torch.empty(1, 8, 2048, device="cuda")
            fa.flex_attention(q, k, v, bm, out=out, lse=lse, stream=st)
            outs.append((out, lse))
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    for out, lse in outs:
        assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)


def test_many_forwards_reuse_the_counters():
    # More launches than the mask has counter pairs: every pair must come back zeroed.
    fa = fa_module()
    w = wl.WORKLOADS[3].scaled(S=1024, H=2)
    q, k, v = (t.cuda() for t in wl.make_qkv(w))
    doc = wl.make_doc_ids(w)
    bm = gpu_block_mask(w.mask_kind, None, None, w.S, w.S, 0, doc)
    o_ref, l_ref = fa.flex_attention(q, k, v, bm)
    for _ in range(70):
        o, l = fa.flex_attention(q, k, v, bm)
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
    assert bm.device_status() == fa.FA_OK


def test_more_forwards_in_flight_than_counter_pairs():
    # Four streams are held back by a sleep kernel while 160 forwards are enqueued on one mask:
    # more than its 64 counter pairs are pending at once.  A forward that would reuse a pair
    # waits on the GPU for the pair's previous user, so every output is still exact.
    fa = fa_module()
    g = torch.Generator().manual_seed(27)
    q, k, v = (torch.randn(1, 4, 1024, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    bm = gpu_block_mask(C, None, None, 1024, 1024)
    o_ref, l_ref = fa.flex_attention(q, k, v, bm)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(4)]
    outs = []
    for st in streams:
        with torch.cuda.stream(st):
            torch.cuda._sleep(20_000_000)          # about 10 ms: the launches below queue up
    for i in range(160):
        st = streams[i % 4]
        with torch.cuda.stream(st):
            out = torch.empty_like(q)
            lse = torch.empty(1, 4, 1024, device="cuda")
            fa.flex_attention(q, k, v, bm, out=out, lse=lse, stream=st)
            outs.append((out, lse))
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    for out, lse in outs:
        assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)


@pytest.mark.parametrize("kind,window,score_kind", [(C, 0, wl.SCORE_NONE),
                                                    (C | SW, 4096, wl.SCORE_SOFTCAP | wl.SCORE_ALIBI)])
def test_long_sequence_sampled_rows(kind, window, score_kind):
    # 131072 positions: 1024 blocks per side, units of up to 1024 entries.
    w = wl.Workload("long", B=1, H=1, S=131072, D=64, dtype="bf16", mask_kind=kind, window=window,
                    score_kind=score_kind, softcap=30.0, seed=25)
    q, k, v = wl.make_qkv(w)
    out, lse, _ = run_gpu(w, q, k, v)
    rows = _sample_rows(w.S, w.seed, n_random=6)
    O, L = run_oracle(w, q, k, v, rows=rows)
    compare(out, lse, O, L, rows=rows)


def test_host_buffers_are_rejected_before_any_launch():
    # The C ABI checks that every buffer is memory of the current device; host memory,
    # pageable or pinned, is an argument error, and the context stays usable.
    fa = fa_module()
    g = torch.Generator().manual_seed(26)
    q, k, v = (torch.randn(1, 2, 256, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bm = gpu_block_mask(C, None, None, 256, 256)
    for bad in (q, q.pin_memory()):
        with pytest.raises((fa.FaError, ValueError)):   # the binding or the C ABI refuses
            fa.flex_attention(bad, kd, vd, bm)
        with pytest.raises(fa.FaError) as info:         # the C ABI on its own
            fa.fa_forward(fa.fa_tensor(bad), fa.fa_tensor(kd), fa.fa_tensor(vd), bm.handle, 0,
                          fa.FaScoreParams(30.0, None), -1.0, fa.fa_tensor(torch.empty_like(qd)),
                          None, None)
        assert info.value.status == fa.FA_ERR_INVALID_ARG
    out_host = torch.empty(1, 2, 256, 64, dtype=torch.bfloat16).pin_memory()
    with pytest.raises(fa.FaError):
        fa.flex_attention(qd, kd, vd, bm, out=out_host)
    lse_host = torch.empty(1, 2, 256, dtype=torch.float32).pin_memory()
    with pytest.raises(ValueError):          # the binding checks what a bare pointer cannot say
        fa.flex_attention(qd, kd, vd, bm, lse=lse_host)
    with pytest.raises(fa.FaError) as info:  # and the C ABI rejects the host pointer itself
        fa.fa_forward(fa.fa_tensor(qd), fa.fa_tensor(kd), fa.fa_tensor(vd), bm.handle, 0,
                      fa.FaScoreParams(30.0, None), -1.0, fa.fa_tensor(torch.empty_like(qd)),
                      lse_host.data_ptr(), None)
    assert info.value.status == fa.FA_ERR_INVALID_ARG
    out, lse = fa.flex_attention(qd, kd, vd, bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    w = wl.Workload("host_check", B=1, H=2, S=256, D=64, dtype="bf16", mask_kind=C, seed=26)
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)


def test_per_batch_sequence_lengths():
    # kv_lens: key kv of batch b exists iff kv < kv_lens[b]; the mask is per batch element.
    fa = fa_module()
    lens = np.array([300, 1000, 129], dtype=np.int32)
    w = wl.Workload("lens", B=3, H=2, S=1000, D=128, dtype="bf16", mask_kind=C, seed=29)
    q, k, v = wl.make_qkv(w)
    bm = fa.create_block_mask(C, 3, None, 1000, 1000, kv_lens=torch.from_numpy(lens).cuda())
    ref = oracle.create_block_mask(oracle.make_mask_mod(C, kv_lens=lens), 3, None, 1000, 1000)
    from gpu_common import assert_block_mask_equal
    assert_block_mask_equal(bm, ref)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm)
    torch.cuda.synchronize()
    mm = oracle.make_mask_mod(C, kv_lens=lens)
    O, L = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), mm, None, scale=w.scale)
    compare(out, lse, O, L)


@pytest.mark.parametrize("Q,D,dtype,score", [(1, 128, "bf16", 0), (3, 64, "fp16", 0), (1, 128, "bf16", 3),
                                             (4, 64, "bf16", 2), (5, 128, "bf16", 0)])
def test_paged_decode_matches_contiguous_and_the_oracle(Q, D, dtype, score):
    # PagedAttention through block indices: K/V in shuffled 128-token pages of one pool.  Up to
    # 4 query rows run the split decode path (checked against the oracle); the tensor-core path
    # over the pages (split_decode=False, and always for more rows) equals the contiguous
    # forward bit for bit.
    fa = fa_module()
    dw = wl.DecodeWorkload("decode_small", B=4, H=4, D=D, lo=130, hi=2500, Q=Q, dtype=dtype, seed=30)
    q, k, v, kp, vp, table, lens = wl.make_decode(dw)
    KV = k.shape[2]
    lens_t = torch.from_numpy(lens).cuda()
    bm = fa.create_block_mask(0, dw.B, None, Q, KV, kv_lens=lens_t)
    qd, kd, vd, kpd, vpd, td = (t.cuda() for t in (q, k, v, kp, vp, table))
    split = fa.flex_attention(qd, kpd, vpd, bm, page_table=td, score_mod=score, softcap=20.0)
    tc = fa.flex_attention(qd, kpd, vpd, bm, page_table=td, score_mod=score, softcap=20.0, split_decode=False)
    contig = fa.flex_attention(qd, kd, vd, bm, score_mod=score, softcap=20.0)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    assert torch.equal(tc[0], contig[0]) and torch.equal(tc[1], contig[1])
    mm = oracle.make_mask_mod(0, kv_lens=lens)
    sm = oracle.make_score_mod(score, H=dw.H, softcap=20.0)
    O, L = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), mm, sm, scale=dw.scale)
    compare(split[0], split[1], O, L)
    compare(tc[0], tc[1], O, L)


def test_paged_page_out_of_range_is_reported():
    fa = fa_module()
    dw = wl.DecodeWorkload("decode_bad", B=2, H=2, D=64, lo=200, hi=300, seed=31)
    q, k, v, kp, vp, table, lens = wl.make_decode(dw)
    table[1, 0] = kp.shape[0] + 5
    bm = fa.create_block_mask(0, dw.B, None, 1, k.shape[2], kv_lens=torch.from_numpy(lens).cuda())
    fa.flex_attention(q.cuda(), kp.cuda(), vp.cuda(), bm, page_table=table.cuda())
    assert bm.device_status() == fa.FA_ERR_INVALID_ARG
    assert bm.device_status() == fa.FA_OK


def test_paged_decode_full_size_every_row():
    # The decode workload the bench times (B = 16, H = 16, one new token, contexts 1k-8k,
    # shuffled 128-token pages), through the split path in the bench's launch configuration
    # (chunks of several tiles each, so chunk boundaries fall inside a sequence), against the
    # float64 oracle on every (b, h) row.
    fa = fa_module()
    dw = wl.DECODE_WORKLOADS[0]
    q, k, v, kp, vp, table, lens = wl.make_decode(dw)
    KV = k.shape[2]
    bm = fa.create_block_mask(0, dw.B, None, dw.Q, KV, kv_lens=torch.from_numpy(lens).cuda())
    out, lse = fa.flex_attention(q.cuda(), kp.cuda(), vp.cuda(), bm, page_table=table.cuda(), scale=dw.scale)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    mm = oracle.make_mask_mod(0, kv_lens=lens)
    O, L = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), mm, None, scale=dw.scale)
    compare(out, lse, O, L)


def test_empty_batches_and_unsupported_head_sizes():
    # Degenerate shapes: an empty batch (B = 0) or no heads is a no-op for the forward, the
    # backward, the masked softmax and the paged decode (nothing launched, status OK); head
    # sizes other than 64 and 128 are refused before any launch; the context stays usable.
    fa = fa_module()
    bm = gpu_block_mask(C, None, None, 256, 256)
    for shape in ((0, 2, 256, 64), (1, 0, 256, 64)):
        q = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        out, lse = fa.flex_attention(q, q, q, bm)
        dq, dk, dv = fa.flex_attention_backward(q, q, q, out, lse, q, bm)
        torch.cuda.synchronize()
        assert out.shape == q.shape and lse.shape == q.shape[:3] and dq.shape == q.shape
        s = torch.zeros(shape[0], shape[1], 256, 256, dtype=torch.bfloat16, device="cuda")
        assert fa.masked_softmax(s).shape == s.shape
    assert bm.device_status() == fa.FA_OK
    for D in (32, 96, 256):
        q = torch.zeros(1, 1, 256, D, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(fa.FaError) as info:
            fa.flex_attention(q, q, q, bm)
        assert info.value.status == fa.FA_ERR_UNSUPPORTED
    # A one-row query against one key (the smallest live problem) still matches the oracle.
    g = torch.Generator().manual_seed(27)
    q, k, v = (torch.randn(1, 1, 1, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    bm1 = gpu_block_mask(C, None, None, 1, 1)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm1)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), v)         # one key: O = V exactly
    assert bm1.device_status() == fa.FA_OK
