"""Host-side logic of bench.py on the CPU: the live-position accounting behind the metric
(checked against the oracle's dense-mask count), the max-over-ranks timing reduction with
two gloo ranks, clock-sample parsing and the peak / traffic bookkeeping."""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import oracle
import workloads as wl


@pytest.mark.parametrize("w", [wl.WORKLOADS[0], wl.WORKLOADS[1].scaled(S=1024),
                               wl.WORKLOADS[2].scaled(S=2048), wl.WORKLOADS[3].scaled(S=2048),
                               wl.WORKLOADS[4].scaled(S=1024)], ids=lambda w: w.name + f"_{w.S}")
def test_live_positions_match_the_oracle_count(w):
    doc = wl.make_doc_ids(w)
    mm = oracle.make_mask_mod(w.mask_kind, window=w.window or None, document_id=doc)
    assert bench.live_positions_per_head(w, doc) == oracle.live_positions(mm, w.S, w.S)


def test_flops_of_the_stated_workloads():
    # 4 * D * live positions * B * H, live counts as the closed forms give them.
    assert bench.flops_per_step(wl.WORKLOADS[1]) == 4 * 64 * (8192 * 8193 // 2) * 16
    assert bench.flops_per_step(wl.WORKLOADS[4]) == 4 * 128 * (32768 * 32769 // 2) * 8
    w = wl.WORKLOADS[2]
    live = sum(min(q + 1, 1024) for q in range(8192))
    assert bench.flops_per_step(w) == 4 * 128 * live * 32


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (world, rank, rank)
        # The per-rank partition bench.py runs: each rank draws its own batch from its own seed.
        w = wl.WORKLOADS[1].scaled(S=256, H=2)
        plan = bench.rank_plan(w, world, rank)
        q, k, v = wl.make_qkv(w, seed=plan["seed"])
        sums = torch.tensor([float(q.float().sum()), float(plan["seed"])], dtype=torch.float64)
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, sums)
        cfg = bench.config_dict(w, world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        out[rank] = {"t": t, "plan": plan, "cfg": (cfg["global_batch"], cfg["parallelism"]),
                     "gathered": [g.tolist() for g in gathered]}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_partition_the_work_and_take_the_max_time():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0["t"] == r1["t"] == 15.0                     # max over ranks, on every rank
    assert r0["plan"]["seed"] != r1["plan"]["seed"]       # independent batches
    assert r0["plan"]["seed"] == wl.WORKLOADS[1].seed and r1["plan"]["seed"] == wl.WORKLOADS[1].seed + 1000
    assert r0["gathered"] == r1["gathered"]
    (s0, seed0), (s1, seed1) = r0["gathered"]
    assert s0 != s1 and (seed0, seed1) == (r0["plan"]["seed"], r1["plan"]["seed"])
    assert r0["cfg"] == r1["cfg"] == (2, "dp2")           # global batch = B * world
    assert r0["plan"]["global_batch"] == 2 and r0["plan"]["parallelism"] == "dp2"


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_clock_sample_summary():
    c = bench.ClockSampler(0)
    c.sm_max = 1965.0
    c.samples = [(1965.0, 700.5, 0x0), (1800.0, 990.1, 0x4), (1900.0, 950.0, 0x4 | 0x1)]
    s = c.summary()
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965 and s["sm_mhz_min"] == 1800
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3 and s["power_w_max"] == 990.1
    c.samples = [(1500.0, 500.0, 0x8 | 0x40 | 0x20)]
    assert c.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_sampler_reports_why_it_has_no_samples():
    # No GPU here: NVML cannot start, and the summary says so instead of inventing clocks.
    with bench.ClockSampler(0, period_s=0.001) as c:
        pass
    s = c.summary()
    if s["samples"] == 0:
        assert s["sm_mhz"] is None and "error" in s


def test_peaks_and_recorded_traffic(tmp_path, monkeypatch):
    peaks = bench.read_peaks()
    assert peaks["bf16_tflops"] > 0 and peaks["source"] in ("measured", "fallback")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_peaks()["source"] == "fallback"
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "kernel_source_sha", lambda family="forward": "abc")
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(
        {"w1": {"kernel_source_sha": "abc", "dram_bytes_per_launch": 123},
         "w2": {"kernel_source_sha": "old", "dram_bytes_per_launch": 456}}))
    assert bench.recorded_traffic("w1") == 123
    assert bench.recorded_traffic("w2") is None
    assert bench.recorded_traffic("w3") is None


def test_config_names_the_workload():
    c = bench.config_dict(wl.WORKLOADS[4], 2)
    assert c["workload"] == wl.WORKLOADS[4].name and c["parallelism"] == "dp2"
    assert "softcap" in c["score_mod"] and "alibi" in c["score_mod"]
    assert c["global_batch"] == 2


def test_reference_arm_times_bounded_oracle_samples():
    import argparse
    args = argparse.Namespace(steps=2, warmup=3, reference_budget_s=0.5)
    w = wl.WORKLOADS[1].scaled(S=1024)
    r = bench.run_reference(args, w, 1, 0)
    assert r["impl"] == "reference" and r["value"] > 0 and r["dtype"] == "f64"
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["value"] == r["value"]
    assert r["e2e"]["value"] == r["value"] and r["e2e"]["h2d_bytes_per_step"] == 0
    assert r["steps"] == 2 and r["warmup"] == 3


def test_oracle_sample_rate_runs_at_least_one_chunk():
    w = wl.WORKLOADS[0]
    q, k, v = wl.make_qkv(w)
    r = bench.oracle_sample_rate(w, q, k, v, None, 0.0, rows_per_chunk=8)
    assert r["rows"] == 8 and r["value"] > 0


def test_kernel_hash_ignores_comments_and_layout():
    a = 'int x = 1; // note\n/* block\n comment */ asm volatile("ld.x // not a comment");\n'
    b = 'int  x = 1;\n\nasm volatile("ld.x // not a comment"); // other words\n'
    assert bench._strip_c_comments(a) == bench._strip_c_comments(b)
    assert "not a comment" in bench._strip_c_comments(a)
    assert bench._strip_c_comments("int x = 1;") != bench._strip_c_comments("int x = 2;")
    assert len(bench.kernel_source_sha()) == 16
    assert {len(bench.kernel_source_sha(f)) for f in bench.KERNEL_SOURCES} == {16}
    assert len({bench.kernel_source_sha(f) for f in bench.KERNEL_SOURCES}) == len(bench.KERNEL_SOURCES)
    # Only a kernel's own struct enters its hash: the forward's ignores BwdParams.
    text = "struct FwdParams { int a; };\nstruct BwdParams { int b; };"
    assert bench._struct_text(text, "BwdParams") == "struct BwdParams { int b; };"
