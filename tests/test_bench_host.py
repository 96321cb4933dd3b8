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
    import torch.distributed as dist
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (world, rank, rank)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 15.0


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_clock_sample_summary():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active",
               "0, 1800, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1900, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
               "garbage"]
    s = c.summary()
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3


def test_peaks_and_recorded_traffic(tmp_path, monkeypatch):
    peaks = bench.read_peaks()
    assert peaks["bf16_tflops"] > 0 and peaks["source"] in ("measured", "fallback")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_peaks()["source"] == "fallback"
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "abc")
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
