"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI binding and
the float64 oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as wl

# Tolerances of the float outputs against float64 (fp16/bf16 inputs, fp32 accumulation).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def fa_module():
    import block_sparse_masked_x128_b200 as fa
    return fa


def oracle_mask_mod(kind, window=None, doc=None):
    return oracle.make_mask_mod(kind, window=window, document_id=doc)


def gpu_block_mask(kind, B, H, Q, KV, window=0, doc=None, separate_full=True):
    fa = fa_module()
    doc_t = torch.from_numpy(doc).to("cuda") if doc is not None else None
    return fa.create_block_mask(kind, B, H, Q, KV, window=window, doc_id=doc_t,
                                separate_full_blocks=separate_full)


def assert_block_mask_equal(bm, ref):
    for name in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        got = getattr(bm, name).cpu().numpy()
        want = ref[name]
        assert got.shape == want.shape, (name, got.shape, want.shape)
        if not np.array_equal(got, want):
            bad = np.argwhere(got != want)
            raise AssertionError(f"{name} differs at {len(bad)} places, first {bad[:5].tolist()}: "
                                 f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")


def workload_inputs(w: wl.Workload):
    """q, k, v (CPU, workload dtype) and doc ids for a workload at its stated size."""
    q, k, v = wl.make_qkv(w)
    doc = wl.make_doc_ids(w)
    return q, k, v, doc


def run_gpu(w: wl.Workload, q, k, v, doc=None, separate_full=True, score_kind=None):
    fa = fa_module()
    qd, kd, vd = (t.to("cuda") for t in (q, k, v))
    bm = gpu_block_mask(w.mask_kind, None, None, q.shape[2], k.shape[2], w.window, doc, separate_full)
    sk = w.score_kind if score_kind is None else score_kind
    out, lse = fa.flex_attention(qd, kd, vd, bm, score_mod=sk, softcap=w.softcap or 30.0,
                                 scale=w.scale)
    torch.cuda.synchronize()
    assert bm.device_status() == fa.FA_OK
    return out, lse, bm


def run_oracle(w: wl.Workload, q, k, v, doc=None, rows=None, score_kind=None):
    mm = oracle_mask_mod(w.mask_kind, w.window or None, doc)
    sk = w.score_kind if score_kind is None else score_kind
    sm = oracle.make_score_mod(sk, H=q.shape[1], softcap=w.softcap or 30.0)
    return oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), mm, sm,
                            scale=w.scale, rows=rows)


def compare(out, lse, O_ref, lse_ref, rows=None):
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        o = o[:, :, rows]
        l = l[:, :, rows]
    err = np.abs(o - O_ref)
    finite = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(l), finite), "rows without live keys differ"
    lerr = np.abs(l[finite] - lse_ref[finite]) if finite.any() else np.zeros(1)
    stats = {"o_max": float(err.max()), "o_mean": float(err.mean()), "lse_max": float(lerr.max())}
    assert stats["o_max"] <= O_MAX_ABS, stats
    assert stats["o_mean"] <= O_MEAN_ABS, stats
    assert stats["lse_max"] <= LSE_MAX_ABS, stats
    return stats
