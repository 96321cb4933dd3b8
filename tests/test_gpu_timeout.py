"""Failure detection on the GPU without a fault: the library's test hook makes the TMA warp
stop before loading any K or V tile, so the MMA warp's bounded wait runs out after about two
seconds.  The kernel must unwind (every role returns, tensor memory is released), the host
must read FA_ERR_TIMEOUT from the mask's status word, and the same context must then run a
normal forward that matches the oracle."""
import time

import pytest
import torch

import workloads as wl
from gpu_common import compare, fa_module, gpu_block_mask, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128])
def test_stalled_loads_time_out_and_the_context_survives(D):
    fa = fa_module()
    w = wl.Workload("timeout", B=1, H=2, S=512, D=D, dtype="bf16", mask_kind=wl.MASK_CAUSAL, seed=31)
    q, k, v = wl.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bm = gpu_block_mask(wl.MASK_CAUSAL, None, None, 512, 512)
    assert bm.device_status() == fa.FA_OK
    fa.fa_debug_set_stall(True)
    try:
        t0 = time.monotonic()
        fa.flex_attention(qd, kd, vd, bm)
        status = bm.device_status()          # synchronises the stream
        elapsed = time.monotonic() - t0
    finally:
        fa.fa_debug_set_stall(False)
    assert status == fa.FA_ERR_TIMEOUT
    assert 1.0 < elapsed < 30.0
    assert bm.device_status() == fa.FA_OK    # reading cleared the word
    out, lse = fa.flex_attention(qd, kd, vd, bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    O, L = run_oracle(w, q, k, v)
    compare(out, lse, O, L)


def test_stalled_backward_times_out_and_the_context_survives():
    fa = fa_module()
    w = wl.Workload("timeout_bwd", B=1, H=2, S=512, D=64, dtype="bf16", mask_kind=wl.MASK_CAUSAL, seed=32)
    q, k, v = (t.cuda() for t in wl.make_qkv(w))
    do = wl.make_dout(w).cuda()
    bm = gpu_block_mask(wl.MASK_CAUSAL, None, None, 512, 512)
    out, lse = fa.flex_attention(q, k, v, bm)
    ref = fa.flex_attention_backward(q, k, v, out, lse, do, bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    fa.fa_debug_set_stall(True)
    try:
        fa.flex_attention_backward(q, k, v, out, lse, do, bm)
        status = bm.device_status()
    finally:
        fa.fa_debug_set_stall(False)
    assert status == fa.FA_ERR_TIMEOUT
    again = fa.flex_attention_backward(q, k, v, out, lse, do, bm)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    assert all(torch.equal(a, b) for a, b in zip(again, ref))


def test_stalled_masked_softmax_times_out_and_the_context_survives():
    fa = fa_module()
    g = torch.Generator().manual_seed(33)
    s = torch.randn(1, 2, 1024, 4096, generator=g).to(torch.bfloat16).cuda()   # > 8 rows per CTA
    ref = fa.masked_softmax(s)
    torch.cuda.synchronize()
    assert fa.fa_masked_softmax_status() == fa.FA_OK
    fa.fa_debug_set_stall(True)
    try:
        fa.masked_softmax(s)
        status = fa.fa_masked_softmax_status()
    finally:
        fa.fa_debug_set_stall(False)
    assert status == fa.FA_ERR_TIMEOUT
    assert fa.fa_masked_softmax_status() == fa.FA_OK
    again = fa.masked_softmax(s)
    torch.cuda.synchronize()
    assert torch.equal(again, ref)
