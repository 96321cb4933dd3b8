"""The fused causal-masked softmax on the GPU ("Fuse the causal mask into the SDPA fallback
softmax", MLX pull request 3919) against the float64 chain of the oracle, and against itself
run unmasked on where(keep, scores, finfo.min): the page's claim is bit-identity with that
chain, and masked entries must be exactly zero."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def _fa():
    import block_sparse_masked_x128_b200 as fa
    return fa


def _tol(dtype):
    # One rounding to the 16-bit output (half an ulp: at most 2^-8 relative for bf16's 8
    # significant bits, 2^-11 for fp16's 11) plus the float32 exp and sum (about 1e-6
    # relative); absolute terms for fp16's subnormal spacing and for float32 results below
    # its normal range, which the kernel's exp flushes to zero.
    return (2.0 ** -8 * 1.01, 1e-37) if dtype == torch.bfloat16 else (2.0 ** -10, 2.0 ** -24)


def _check_against_oracle(p_gpu, scores, offset, dtype, rows=None):
    name = "bf16" if dtype == torch.bfloat16 else "fp16"
    ref = oracle.masked_softmax(scores.float().numpy(), offset, name, rows=rows)
    got = p_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[..., rows, :]
    zero = ref == 0.0
    assert np.all(got[zero] == 0.0), "a masked entry is not exactly zero"
    rel, ab = _tol(dtype)
    err = np.abs(got - ref)
    assert np.all(err <= rel * np.abs(ref) + ab + 1e-30), float(err.max())
    return float(err.max())


def _chain_input(scores, offset):
    Q, K = scores.shape[2], scores.shape[3]
    keep = torch.from_numpy(oracle.causal_keep(Q, K, offset)).to(scores.device)
    return torch.where(keep, scores, torch.finfo(scores.dtype).min)


CASES = [(1, 2, 64, 512, None), (2, 3, 100, 4096, None), (1, 2, 96, 1024, 0), (1, 1, 40, 2048, -17),
         (1, 2, 33, 8192, 9000), (1, 1, 130, 16384, None), (1, 1, 20, 32768, None), (1, 2, 16, 4104, 4000)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("B,H,Q,K,offset", CASES)
def test_masked_softmax_matches_the_oracle_and_the_unfused_chain(B, H, Q, K, offset, dtype):
    fa = _fa()
    g = torch.Generator().manual_seed(Q * 7 + K)
    scores = (2.0 * torch.randn(B, H, Q, K, generator=g)).to(dtype)
    off = K - Q if offset is None else offset
    sd = scores.cuda()
    p = fa.masked_softmax(sd, off)
    torch.cuda.synchronize()
    _check_against_oracle(p, scores, off, dtype)
    # Bit-identity with the chain: the same kernel, unmasked, on where(keep, s, finfo.min).
    chain = fa.masked_softmax(_chain_input(sd, off), causal=False)
    torch.cuda.synchronize()
    assert torch.equal(p, chain)
    assert fa.fa_masked_softmax_status() == fa.FA_OK


def test_plain_softmax_without_the_mask():
    fa = _fa()
    g = torch.Generator().manual_seed(5)
    s = torch.randn(2, 2, 50, 3000, generator=g).to(torch.bfloat16)
    p = fa.masked_softmax(s.cuda(), causal=False)
    ref = oracle.masked_softmax(s.float().numpy(), 0, "bf16", causal=False)
    err = np.abs(p.float().cpu().numpy() - ref)
    assert np.all(err <= 2.0 ** -8 * 1.01 * ref + 1e-37)


def test_fully_masked_rows_are_uniform():
    fa = _fa()
    s = torch.randn(1, 1, 8, 512, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).cuda()
    p = fa.masked_softmax(s, -5)
    torch.cuda.synchronize()
    assert torch.all(p[0, 0, :5] == 1.0 / 512)
    assert p[0, 0, 5, 0] == 1.0 and torch.all(p[0, 0, 5, 1:] == 0)


def test_in_place_and_strided_views():
    fa = _fa()
    g = torch.Generator().manual_seed(7)
    base = torch.randn(1, 2, 64, 1040, generator=g).to(torch.bfloat16).cuda()
    view = base[..., :1024]                     # rows 1040 apart: a strided (padded) layout
    want = fa.masked_softmax(view.contiguous(), 960)
    got = fa.masked_softmax(view, 960)
    assert torch.equal(got, want)
    tmp = view.contiguous()
    fa.masked_softmax(tmp, 960, out=tmp)
    torch.cuda.synchronize()
    assert torch.equal(tmp, want)


def test_unsupported_shapes_and_host_buffers_are_refused():
    fa = _fa()
    s = torch.zeros(1, 1, 4, 104, dtype=torch.bfloat16, device="cuda")[..., :100]   # K % 8 != 0
    with pytest.raises(fa.FaError) as e:
        fa.masked_softmax(s, out=torch.zeros(1, 1, 4, 104, dtype=torch.bfloat16, device="cuda")[..., :100])
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    s = torch.zeros(1, 1, 2, 32776, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.masked_softmax(s)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    h = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16).pin_memory()
    with pytest.raises(fa.FaError) as e:
        fa.fa_masked_softmax(fa.fa_tensor(h), fa.FA_MASK_CAUSAL, 124, fa.fa_tensor(h.cuda()))
    assert e.value.status == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("w", wl.SOFTMAX_WORKLOADS, ids=[w.name for w in wl.SOFTMAX_WORKLOADS])
def test_full_size_workloads(w):
    fa = _fa()
    scores = wl.make_scores(w)
    sd = scores.cuda()
    p = fa.masked_softmax(sd, w.offset)
    torch.cuda.synchronize()
    # Bit-identity with the unfused chain over the whole tensor.
    chain = fa.masked_softmax(_chain_input(sd, w.offset), causal=False)
    torch.cuda.synchronize()
    assert torch.equal(p, chain)
    del chain
    # Exact zeros past the boundary everywhere; rows sum to one within the output rounding.
    keep = torch.from_numpy(oracle.causal_keep(w.Q, w.K, w.offset)).cuda()
    assert not torch.any(p.masked_select(~keep.expand_as(p)) != 0)
    sums = p.float().sum(-1)
    assert torch.all((sums - 1.0).abs() < 2e-2)
    # Sampled rows against the float64 oracle.
    rows = sorted({0, 1, 511, 512, w.Q - 2, w.Q - 1} | set(np.random.default_rng(w.seed).integers(0, w.Q, 6).tolist()))
    _check_against_oracle(p, scores, w.offset, torch.bfloat16, rows=rows)
    assert fa.fa_masked_softmax_status() == fa.FA_OK
