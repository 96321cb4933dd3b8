#!/usr/bin/env python
"""Benchmark: live-position attention forward TFLOP/s of the block-sparse kernel on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one fused forward (``fa_forward``) over one batch of the workload with the block
mask already built: the pages build the mask once and reuse it across forward passes, so the
mask build is timed separately (``mask_build_ms``) and is not part of the metric.  FLOPs are
4 * D * (exact number of live mask positions) * B * H per step; masked positions inside live
tiles and dead tiles do not count.

Under torchrun (N > 1) every rank runs its own independent batch of the workload (data
parallel, weak scaling, no collective on the data path); time is the max over ranks of the
CUDA-event time and ``value`` counts the work of all ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = wl.WORKLOADS[1].name    # 8k dense causal, D = 64, bf16
METRIC = "live-position attention fwd TFLOP/s"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 512 << 20                  # > 126 MB of L2
L2_BYTES = 126 * 1000 * 1000                 # B200 L2
NOMINAL_BF16_TFLOPS = 2250.0


# ---------------------------------------------------------------- work accounting

def live_positions_per_head(w: wl.Workload, doc=None) -> int:
    """Exact count of allowed (q, kv) pairs of one (b, h), from each row's allowed interval.

    Causal and sliding-window rows allow one interval of kv; a document row allows its
    document's run of positions (document ids here form contiguous runs).
    """
    S = w.S
    q = np.arange(S, dtype=np.int64)
    lo = np.zeros(S, dtype=np.int64)
    hi = np.full(S, S - 1, dtype=np.int64)
    if w.mask_kind & (wl.MASK_CAUSAL | wl.MASK_SLIDING_WINDOW):
        hi = np.minimum(hi, q)
    if w.mask_kind & wl.MASK_SLIDING_WINDOW:
        lo = np.maximum(lo, q - w.window + 1)
    if w.mask_kind & wl.MASK_DOCUMENT:
        if doc is None or np.any(np.diff(doc) < 0):
            raise ValueError("document ids must form contiguous ascending runs")
        starts = np.searchsorted(doc, doc, side="left")
        ends = np.searchsorted(doc, doc, side="right") - 1
        lo = np.maximum(lo, starts)
        hi = np.minimum(hi, ends)
    return int(np.clip(hi - lo + 1, 0, None).sum())


def flops_per_step(w: wl.Workload, doc=None) -> float:
    return 4.0 * w.D * live_positions_per_head(w, doc) * w.B * w.H


# ---------------------------------------------------------------- environment helpers

def read_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]), "hbm_gbs": float(d["hbm_gbs"]),
                "source": "measured"}
    return {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "source": "fallback"}


def _strip_c_comments(text: str) -> str:
    """C/C++ source without comments, whitespace runs collapsed (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


# The code of each kernel family: its own sources plus the parameter struct it is launched
# with (extracted from the shared header), so edits elsewhere leave its recorded counters valid.
KERNEL_SOURCES = {
    "forward": (["block_sparse_masked_x128_b200/csrc/attn_fwd.cu",
                 "block_sparse_masked_x128_b200/csrc/fwd_common.cuh",
                 "block_sparse_masked_x128_b200/csrc/sm100_ptx.cuh"], "FwdParams"),
    "backward": (["block_sparse_masked_x128_b200/csrc/attn_bwd.cu",
                  "block_sparse_masked_x128_b200/csrc/fwd_common.cuh",
                  "block_sparse_masked_x128_b200/csrc/sm100_ptx.cuh"], "BwdParams"),
    "masked_softmax": (["block_sparse_masked_x128_b200/csrc/masked_softmax.cu",
                        "block_sparse_masked_x128_b200/csrc/sm100_ptx.cuh"], None),
    "decode": (["block_sparse_masked_x128_b200/csrc/decode.cu",
                "block_sparse_masked_x128_b200/csrc/sm100_ptx.cuh"], "DecodeParams"),
}


def _struct_text(header_text: str, name: str) -> str:
    i = header_text.find("struct %s {" % name)
    if i < 0:
        return ""
    return header_text[i:header_text.find("};", i) + 2]


def kernel_source_sha(family: str = "forward") -> str:
    """Hash of one kernel family's code (comments and layout ignored), to tell whether the
    recorded ncu counters still describe the kernel that runs."""
    files, struct = KERNEL_SOURCES[family]
    h = hashlib.sha256()
    for rel in files:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as fh:
            h.update(_strip_c_comments(fh.read()).encode())
    if struct:
        with open(os.path.join(ROOT, "block_sparse_masked_x128_b200/csrc/fa_internal.h"), encoding="utf-8") as fh:
            h.update(_strip_c_comments(_struct_text(fh.read(), struct)).encode())
    return h.hexdigest()[:16]


def recorded_traffic(name: str, family: str = "forward"):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(name)
    if not e or e.get("kernel_source_sha") != kernel_source_sha(family):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled through NVML while the timed region runs.

    Only reads: nothing here changes a GPU setting.  A thread polls every `period_s`; entering
    the context waits for the first sample, so even a region of a few milliseconds holds
    samples taken while its kernels run.
    """

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int, period_s: float = 0.0005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []          # (sm_mhz, power_w, reasons bitmask)
        self.sm_max = None
        self.error = None
        self._stop = threading.Event()
        self._first = threading.Event()
        self._thread = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _run(self):
        try:
            import pynvml
            h = self._handle()
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            while True:
                sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((sm, pw, rs))
                self._first.set()
                if self._stop.wait(self.period):
                    break
        except Exception as exc:   # no NVML: the summary says so
            self.error = f"{type(exc).__name__}: {exc}"
        finally:
            self._first.set()

    def __enter__(self):
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        self._first.wait(timeout=10)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=10)

    def summary(self) -> dict:
        sm = [x[0] for x in self.samples]
        reasons = set()
        for _, _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
               "sm_mhz_min": min(sm) if sm else None,
               "power_w_max": max(x[1] for x in self.samples) if sm else None,
               "reasons": sorted(reasons), "samples": len(sm), "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- CPU oracle baseline

def oracle_sample_rate(w: wl.Workload, q, k, v, doc, budget_s: float, rows_per_chunk: int = 256,
                       seed: int = 0) -> dict:
    """Time the float64 oracle on random query rows of the workload until budget_s elapses."""
    import oracle
    mm = oracle.make_mask_mod(w.mask_kind, window=w.window or None, document_id=doc)
    sm = oracle.make_score_mod(w.score_kind, H=w.H, softcap=w.softcap or 30.0)
    rng = np.random.default_rng(seed)
    qn, kn, vn = (t.float().numpy() for t in (q, k, v))
    live_row = _live_per_row(w, doc)
    rows_done, live, t_total = 0, 0, 0.0
    while rows_done == 0 or t_total < budget_s:   # at least one chunk
        b = int(rng.integers(0, w.B))
        h = int(rng.integers(0, w.H))
        rows = np.sort(rng.choice(w.S, size=min(rows_per_chunk, w.S), replace=False))
        t0 = time.perf_counter()
        oracle.attention(qn[b:b + 1, h:h + 1], kn[b:b + 1, h:h + 1], vn[b:b + 1, h:h + 1], mm,
                         (lambda s, bb, hh, qi, ki, _h=h: sm(s, 0, _h, qi, ki)) if sm else None,
                         scale=w.scale, rows=rows)
        t_total += time.perf_counter() - t0
        rows_done += len(rows)
        live += int(live_row[rows].sum())
    tflops = 4.0 * w.D * live / t_total / 1e12
    return {"value": tflops, "rows": rows_done, "seconds": t_total, "live_positions": live}


def _live_per_row(w, doc):
    S = w.S
    q = np.arange(S, dtype=np.int64)
    lo = np.zeros(S, dtype=np.int64)
    hi = np.full(S, S - 1, dtype=np.int64)
    if w.mask_kind & (wl.MASK_CAUSAL | wl.MASK_SLIDING_WINDOW):
        hi = np.minimum(hi, q)
    if w.mask_kind & wl.MASK_SLIDING_WINDOW:
        lo = np.maximum(lo, q - w.window + 1)
    if w.mask_kind & wl.MASK_DOCUMENT:
        lo = np.maximum(lo, np.searchsorted(doc, doc, side="left"))
        hi = np.minimum(hi, np.searchsorted(doc, doc, side="right") - 1)
    return np.clip(hi - lo + 1, 0, None)


def cores_used() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        if blas:
            return int(max(blas))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------- arms

def rank_plan(w: wl.Workload, world: int, rank: int) -> dict:
    """What rank `rank` of `world` runs: its own batch of the workload (data parallel, weak
    scaling), drawn from its own seed, with no exchange on the data path."""
    return {"seed": w.seed + 1000 * rank, "global_batch": w.B * world,
            "parallelism": f"dp{world}"}


def config_dict(w: wl.Workload, world: int) -> dict:
    mask = []
    if w.mask_kind & wl.MASK_CAUSAL:
        mask.append("causal")
    if w.mask_kind & wl.MASK_SLIDING_WINDOW:
        mask.append(f"sliding_window(W={w.window})")
    if w.mask_kind & wl.MASK_DOCUMENT:
        mask.append(f"document({w.n_docs} seeded docs)")
    score = []
    if w.score_kind & wl.SCORE_SOFTCAP:
        score.append(f"softcap({w.softcap:g})")
    if w.score_kind & wl.SCORE_ALIBI:
        score.append("alibi(2^(-8(h+1)/H))")
    plan = rank_plan(w, world, 0)
    return {"workload": w.name, "B": w.B, "H": w.H, "Q_LEN": w.S, "KV_LEN": w.S, "head_dim": w.D,
            "BLOCK_SIZE": 128, "mask_mod": " & ".join(mask) or "none",
            "score_mod": " then ".join(score) or "none", "global_batch": plan["global_batch"],
            "seq_len": w.S, "parallelism": plan["parallelism"],
            "l2": f"flushed ({L2_FLUSH_BYTES >> 20} MiB write) before every timed step"}


def time_forward(w: wl.Workload, steps: int, warmup: int, world: int, rank: int, dev) -> dict:
    """Build the mask (timed apart), then time `steps` forwards with CUDA events on the
    launching stream, L2 flushed before each, clocks sampled during the timed region."""
    import torch
    import block_sparse_masked_x128_b200 as fa

    q, k, v = wl.make_qkv(w, seed=rank_plan(w, world, rank)["seed"])
    doc = wl.make_doc_ids(w)
    flops = flops_per_step(w, doc)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    doc_d = torch.from_numpy(doc).to(dev) if doc is not None else None
    stream = torch.cuda.current_stream()

    # Mask build: CUDA events around the whole call (its one device allocation, the copies and
    # the kernels), every mask kept alive until all are timed so that no free (which
    # synchronises the device) falls inside a timed build.
    build_ms = []
    masks = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        masks.append(fa.create_block_mask(w.mask_kind, None, None, w.S, w.S, window=w.window, doc_id=doc_d))
        e1.record(stream)
        torch.cuda.synchronize()
        build_ms.append(e0.elapsed_time(e1))
    bm = masks.pop()
    del masks
    out = torch.empty_like(qd)
    lse = torch.empty(w.B, w.H, w.S, device=dev, dtype=torch.float32)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd():
        fa.flex_attention(qd, kd, vd, bm, score_mod=w.score_kind, softcap=w.softcap or 30.0,
                          scale=w.scale, out=out, lse=lse)

    for _ in range(warmup):
        flush.zero_()
        fwd()
    torch.cuda.synchronize()
    if bm.device_status() != fa.FA_OK:
        raise RuntimeError("a device-side wait timed out during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        t_wall0 = time.perf_counter()
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            fwd()
            ends[i].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall0
    barrier(world)
    if bm.device_status() != fa.FA_OK:
        raise RuntimeError("a device-side wait timed out during the timed steps")
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    t_max_ms = max_over_ranks(sum(per), world, dev)
    ck = clocks.summary()
    return {"flops": flops, "per_ms": per, "t_max_ms": t_max_ms,
            "value": world * flops * steps / (t_max_ms * 1e-3) / 1e12,
            "achieved": flops / (statistics.mean(per) * 1e-3) / 1e12,
            "mask_build_ms": statistics.median(build_ms[1:]), "clocks": ck, "wall_s": t_wall,
            "q": q, "k": k, "v": v, "doc": doc, "qd": qd, "kd": kd, "vd": vd, "out": out,
            "lse": lse, "bm": bm}


def softmax_bytes(w: wl.SoftmaxWorkload) -> int:
    """Algorithmic bytes of one fused masked softmax: the live scores read once (scores past
    the causal boundary are never needed) and every probability written once, 2 bytes each."""
    q = np.arange(w.Q, dtype=np.int64)
    live = np.clip(q + w.offset + 1, 0, w.K).sum()
    return int(2 * w.B * w.H * (live + w.Q * w.K))


def time_masked_softmax(w: wl.SoftmaxWorkload, steps: int, warmup: int, world: int, dev) -> dict:
    """Time the fused causal-masked softmax (CUDA events on the launching stream) and report its
    HBM roofline.  The scores are several times the L2, so steps run back to back with no flush,
    like the copy that measured the peak (a flush would leave its own dirty lines in L2 for the
    kernel to write back)."""
    import torch
    import block_sparse_masked_x128_b200 as fa

    scores = wl.make_scores(w).to(dev)
    out = torch.empty_like(scores)
    assert scores.numel() * scores.element_size() > 4 * L2_BYTES
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fa.masked_softmax(scores, w.offset, out=out)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    with ClockSampler(dev.index) as clocks:
        for i in range(steps):
            starts[i].record(stream)
            fa.masked_softmax(scores, w.offset, out=out)
            ends[i].record(stream)
        torch.cuda.synchronize()
    if fa.fa_masked_softmax_status() != fa.FA_OK:
        raise RuntimeError("a masked-softmax wait timed out")
    per = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    t_max = max_over_ranks(sum(per), world, dev)
    nbytes = softmax_bytes(w)
    peaks = read_peaks()
    achieved = nbytes / (statistics.mean(per) * 1e-3) / 1e9
    return {"metric": "fused causal-masked softmax GB/s (live scores read + probabilities written)",
            "value": world * nbytes * steps / (t_max * 1e-3) / 1e9, "unit": "GB/s",
            "ms_per_step": t_max / steps, "bytes_per_step": nbytes, "gpu_launches": steps,
            "config": {"workload": w.name, "B": w.B, "H": w.H, "Q": w.Q, "K": w.K,
                       "offset": w.offset, "dtype": w.dtype,
                       "l2": f"no flush: the scores ({scores.numel() * 2 >> 20} MiB) exceed the L2 four times over"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": recorded_traffic(w.name, "masked_softmax"),
                         "peak_source": peaks["source"] + " hbm_gbs",
                         "kernel": "masked_softmax_kernel"},
            "clocks": clocks.summary()}


def time_backward(w: wl.Workload, steps: int, warmup: int, world: int, rank: int, dev) -> dict:
    """Time fa_backward (pre-pass, dK/dV pass, dQ pass) on one workload, L2 flushed before each
    step.  Algorithmic FLOPs are 2.5 times the forward's (five 4*D-per-position matmul pairs
    halved: 10 * D per live position); the kernels execute 14 * D (S and dP are formed in both
    passes, which keeps every sum on one CTA)."""
    import torch
    import block_sparse_masked_x128_b200 as fa

    q, k, v = (t.to(dev) for t in wl.make_qkv(w, seed=rank_plan(w, world, rank)["seed"]))
    do = wl.make_dout(w, seed=rank_plan(w, world, rank)["seed"]).to(dev)
    doc = wl.make_doc_ids(w)
    doc_d = torch.from_numpy(doc).to(dev) if doc is not None else None
    bm = fa.create_block_mask(w.mask_kind, None, None, w.S, w.S, window=w.window, doc_id=doc_d)
    out, lse = fa.flex_attention(q, k, v, bm, score_mod=w.score_kind, softcap=w.softcap or 30.0,
                                 scale=w.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_backward_workspace_bytes(w.B, w.H, w.S), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def bwd():
        fa.flex_attention_backward(q, k, v, out, lse, do, bm, score_mod=w.score_kind,
                                   softcap=w.softcap or 30.0, scale=w.scale, dq=dq, dk=dk, dv=dv,
                                   workspace=ws)

    for _ in range(warmup):
        flush.zero_()
        bwd()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    with ClockSampler(dev.index) as clocks:
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            bwd()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if bm.device_status() != fa.FA_OK:
        raise RuntimeError("a device-side wait timed out in the backward")
    per = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    t_max = max_over_ranks(sum(per), world, dev)
    flops = 2.5 * flops_per_step(w, doc)
    peaks = read_peaks()
    achieved = flops / (statistics.mean(per) * 1e-3) / 1e12
    return {"metric": "live-position attention bwd TFLOP/s (2.5x forward FLOPs)",
            "value": world * flops * steps / (t_max * 1e-3) / 1e12, "unit": UNIT,
            "ms_per_step": t_max / steps, "algorithmic_gflop_per_step": flops / 1e9,
            "executed_gflop_per_step": flops * 1.4 / 1e9, "gpu_launches": 3 * steps,
            "config": {"workload": w.name, "dtype": w.dtype},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "traffic": recorded_traffic("backward_" + w.name, "backward"),
                         "peak_source": peaks["source"] + " bf16_tflops (burst)",
                         "kernel": "attn_bwd_kernel (dK/dV and dQ passes) + pre-pass"},
            "clocks": clocks.summary()}


def decode_bytes(w: wl.DecodeWorkload) -> int:
    """Algorithmic bytes of one paged decode step: every live key and value read once (the
    tokens of each sequence, all heads), q read and out written once, lse written once."""
    toks = int(w.lengths().astype(np.int64).sum())
    return int(toks * w.H * w.D * 2 * 2 + 2 * w.B * w.H * w.Q * w.D * 2 + w.B * w.H * w.Q * 4)


def time_decode(w: wl.DecodeWorkload, steps: int, warmup: int, world: int, dev) -> dict:
    """Time one paged decode step (fa_forward_paged over the shuffled page pool); HBM roofline
    over the bytes decode_bytes counts.  The live K/V pages are several times the L2 and are
    streamed in the same order every step, so steps run back to back with no flush (as the
    copy that measured the peak did)."""
    import torch
    import block_sparse_masked_x128_b200 as fa

    q, k, v, kp, vp, table, lens = wl.make_decode(w)
    del k, v
    q, kp, vp, table = q.to(dev), kp.to(dev), vp.to(dev), table.to(dev)
    bm = fa.create_block_mask(0, w.B, None, w.Q, w.kv_len, kv_lens=torch.from_numpy(lens).to(dev))
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.Q, device=dev, dtype=torch.float32)
    assert decode_bytes(w) > 4 * L2_BYTES
    stream = torch.cuda.current_stream()

    def step():
        fa.flex_attention(q, kp, vp, bm, page_table=table, scale=w.scale, out=out, lse=lse)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    with ClockSampler(dev.index) as clocks:
        for i in range(steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if bm.device_status() != fa.FA_OK:
        raise RuntimeError("the paged decode reported a timeout or a page out of range")
    per = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    t_max = max_over_ranks(sum(per), world, dev)
    nbytes = decode_bytes(w)
    peaks = read_peaks()
    achieved = nbytes / (statistics.mean(per) * 1e-3) / 1e9
    return {"metric": "paged decode attention GB/s (live K/V read once)",
            "value": world * nbytes * steps / (t_max * 1e-3) / 1e9, "unit": "GB/s",
            "ms_per_step": t_max / steps, "bytes_per_step": nbytes, "gpu_launches": steps,
            "config": {"workload": w.name, "B": w.B, "H": w.H, "D": w.D, "Q": w.Q,
                       "context_lengths": f"seeded in [{w.lo}, {w.hi}]", "dtype": w.dtype,
                       "pages": int(sum(-(-int(n) // 128) for n in lens)),
                       "l2": f"no flush: the live K/V ({decode_bytes(w) >> 20} MiB) exceed the L2 four times over"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": recorded_traffic(w.name, "decode"),
                         "peak_source": peaks["source"] + " hbm_gbs",
                         "kernel": "decode_split_kernel + decode_merge_kernel"},
            "clocks": clocks.summary()}


def run_ours(args, w: wl.Workload, world: int, rank: int, local: int) -> dict:
    import torch
    import block_sparse_masked_x128_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = read_peaks()
    tf = time_forward(w, args.steps, args.warmup, world, rank, dev)
    flops, out, lse, bm = tf["flops"], tf["out"], tf["lse"], tf["bm"]
    stream = torch.cuda.current_stream()

    # End to end through the public API from pinned host buffers: every step copies its q, k,
    # v in, runs the forward and copies out and lse back.  Two device buffer sets and three
    # streams (copy in, compute, copy out) let step i's forward overlap step i+1's input copy
    # and step i-1's output copy, as a user streaming batches would run it.
    e2e = None
    if not args.no_e2e:
        q, k, v = tf["q"], tf["k"], tf["v"]
        qd, kd, vd = tf["qd"], tf["kd"], tf["vd"]
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        e2e_steps = max(3, min(args.steps, args.e2e_steps))
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        bufs = []
        for _ in range(2):
            bufs.append({"q": torch.empty_like(qd), "k": torch.empty_like(kd), "v": torch.empty_like(vd),
                         "out": torch.empty_like(out), "lse": torch.empty_like(lse),
                         "oh": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                         "lh": torch.empty(lse.shape, dtype=lse.dtype).pin_memory(),
                         "in": torch.cuda.Event(), "comp": torch.cuda.Event(), "done": torch.cuda.Event()})

        def e2e_run(n):
            for i in range(n):
                b = bufs[i % 2]
                if i >= 2:
                    s_in.wait_event(b["comp"])          # the forward of step i-2 read these
                with torch.cuda.stream(s_in):
                    b["q"].copy_(qh, non_blocking=True)
                    b["k"].copy_(kh, non_blocking=True)
                    b["v"].copy_(vh, non_blocking=True)
                    b["in"].record(s_in)
                stream.wait_event(b["in"])
                if i >= 2:
                    stream.wait_event(b["done"])        # step i-2's results are on the host
                fa.flex_attention(b["q"], b["k"], b["v"], bm, score_mod=w.score_kind,
                                  softcap=w.softcap or 30.0, scale=w.scale, out=b["out"],
                                  lse=b["lse"], stream=stream)
                b["comp"].record(stream)
                s_out.wait_event(b["comp"])
                with torch.cuda.stream(s_out):
                    b["oh"].copy_(b["out"], non_blocking=True)
                    b["lh"].copy_(b["lse"], non_blocking=True)
                    b["done"].record(s_out)
            for b in bufs:
                stream.wait_event(b["done"])

        e2e_run(2)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(e2e_steps)
        e1.record(stream)
        torch.cuda.synchronize()
        if not torch.equal(bufs[(e2e_steps - 1) % 2]["oh"], out.cpu()):
            raise RuntimeError("end-to-end output differs from the device-resident run")
        t_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
        barrier(world)
        e2e = {"value": world * flops * e2e_steps / (t_e2e * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in (q, k, v))),
               "d2h_bytes_per_step": int(out.numel() * out.element_size() + lse.numel() * 4),
               "steps": e2e_steps, "pipelined": "copy-in / forward / copy-out on three streams"}

    traffic = recorded_traffic(w.name)
    ck = tf["clocks"]
    ms_step = tf["t_max_ms"] / args.steps
    res = {
        "metric": METRIC, "value": tf["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": config_dict(w, world),
        "pct_of_peak": 100.0 * tf["value"] / world / peaks["bf16_tflops"],
        "pct_of_nominal_2250": 100.0 * tf["value"] / world / NOMINAL_BF16_TFLOPS,
        "live_gflop_per_step": flops / 1e9,
        "mask_build_ms": tf["mask_build_ms"],
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "achieved": tf["achieved"], "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tf["achieved"] / peaks["bf16_tflops"],
                     "traffic": traffic, "peak_source": peaks["source"] + " bf16_tflops (burst)",
                     "kernel": "attn_fwd_kernel"},
        "clocks": ck,
        "ms_x_sm_mhz": ms_step * ck["sm_mhz"] if ck.get("sm_mhz") else None,
        "wall_s_timed_region": tf["wall_s"],
    }
    if e2e is not None:
        res["e2e"] = e2e
    del tf

    # The other workloads, measured the same way in the same process (the 32k soft-cap + ALiBi
    # one is the second headline configuration).
    if not args.no_per_workload:
        per = {}
        for other in wl.WORKLOADS:
            if other.name == w.name:
                continue
            o = time_forward(other, args.steps, args.warmup, world, rank, dev)
            oms = o["t_max_ms"] / args.steps
            per[other.name] = {
                "value": o["value"], "unit": UNIT, "ms_per_step": oms,
                "frac": o["achieved"] / peaks["bf16_tflops"],
                "live_gflop_per_step": o["flops"] / 1e9, "mask_build_ms": o["mask_build_ms"],
                "traffic": recorded_traffic(other.name), "clocks": o["clocks"],
                "ms_x_sm_mhz": oms * o["clocks"]["sm_mhz"] if o["clocks"].get("sm_mhz") else None,
                "gpu_launches": args.steps}
            del o
            torch.cuda.empty_cache()
        res["per_workload"] = per

    # The rows after the forward: each timed on its own headline workload.
    if not args.no_per_workload:
        res["next_rows"] = {
            "masked_softmax": time_masked_softmax(wl.SOFTMAX_WORKLOADS[0], args.steps, args.warmup,
                                                  world, dev)}
        torch.cuda.empty_cache()
        res["next_rows"]["decode_paged"] = time_decode(wl.DECODE_WORKLOADS[0], args.steps,
                                                       args.warmup, world, dev)
        torch.cuda.empty_cache()
        for bw in (wl.WORKLOADS[1], wl.WORKLOADS[4]):
            res["next_rows"]["backward_" + bw.name] = time_backward(bw, args.steps, args.warmup,
                                                                     world, rank, dev)
            torch.cuda.empty_cache()

    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        q, k, v = wl.make_qkv(w, seed=rank_plan(w, world, rank)["seed"])
        doc = wl.make_doc_ids(w)
        cb = oracle_sample_rate(w, q, k, v, doc, args.cpu_seconds)
        res["cpu_baseline"] = {"value": cb["value"], "unit": UNIT, "cores": cores_used(),
                               "kind": "oracle",
                               "sample": f"{cb['rows']} random query rows of {w.name} "
                                         f"({cb['seconds']:.1f} s of float64 oracle time)"}
    return res


def run_reference(args, w: wl.Workload, world: int, rank: int) -> dict:
    """The oracle as the reference arm: each step is a bounded sample of query rows."""
    q, k, v = wl.make_qkv(w)
    doc = wl.make_doc_ids(w)
    per_step = max(0.02, args.reference_budget_s / max(1, args.steps + args.warmup))
    rows = 256
    oracle_sample_rate(w, q, k, v, doc, 0.0, rows_per_chunk=rows)  # warm the imports
    for _ in range(args.warmup):
        oracle_sample_rate(w, q, k, v, doc, 0.0, rows_per_chunk=rows)
    t0 = time.perf_counter()
    tot_live, tot_t, tot_rows = 0, 0.0, 0
    for i in range(args.steps):
        r = oracle_sample_rate(w, q, k, v, doc, per_step, rows_per_chunk=rows, seed=i)
        tot_live += r["live_positions"]
        tot_t += r["seconds"]
        tot_rows += r["rows"]
        if time.perf_counter() - t0 > per_step * args.steps + 60:
            break
    value = 4.0 * w.D * tot_live / tot_t / 1e12
    cores = cores_used()
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": dict(config_dict(w, world), l2="host cores: the float64 oracle, no GPU cache involved"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{tot_rows} query rows of {w.name} in {rows}-row chunks, about {per_step:.2g} s per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=[x.name for x in wl.WORKLOADS])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only --workload (skip the per_workload and next_rows sections)")
    ap.add_argument("--only", choices=["masked_softmax", "decode", "backward"],
                    help="time only this row and print its line (for profiling one kernel); "
                         "backward runs on --workload")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-budget-s", type=float, default=60.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = wl.BY_NAME[args.workload]
    world, rank, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, w, world, rank)))
        return 0

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)   # one GPU per rank, bound before NCCL starts
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        if args.only:
            import torch
            torch.cuda.set_device(local)
            dev = torch.device("cuda", local)
            if args.only == "masked_softmax":
                res = time_masked_softmax(wl.SOFTMAX_WORKLOADS[0], args.steps, args.warmup, world, dev)
            elif args.only == "decode":
                res = time_decode(wl.DECODE_WORKLOADS[0], args.steps, args.warmup, world, dev)
            else:
                res = time_backward(w, args.steps, args.warmup, world, rank, dev)
            res.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                        "higher_is_better": True, "scaling": "weak", "data": "synthetic"})
        else:
            res = run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
