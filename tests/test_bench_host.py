"""Host-side logic of bench.py, on CPU: the max-over-ranks timing across two
gloo ranks, the roofline denominator choice, the recorded ncu traffic lookup,
and the oracle reference arm (alone and under torchrun with two ranks, where
only rank 0 works and prints)."""

import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        v = bench.max_over_ranks(10.0 + rank * 2.5, dist, "cpu")
        out[rank] = v
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: 12.5, 1: 12.5}
    assert bench.max_over_ranks(3.0, None, "cpu") == 3.0


def test_peak_choice():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0}
    # A kernel timed in a sub-second region is compared with the burst figure (timed the same
    # way), one timed over seconds with the power-capped sustained figure.
    assert bench.pick_peak(peaks, 0.7, "tensor")[0] == 1650.0
    assert bench.pick_peak(peaks, 0.7, "tensor")[1].startswith("burst")
    assert bench.pick_peak(peaks, 1.99, "tensor")[0] == 1650.0
    assert bench.pick_peak(peaks, 2.0, "tensor")[0] == 1400.0
    assert bench.pick_peak(peaks, 30.0, "tensor")[1].startswith("sustained")
    assert bench.pick_peak(peaks, 30.0, "hbm")[0] == 6500.0


def test_rows_report_measured_and_nominal_fractions():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0}
    r = bench.part_row("fwd", 8.25e12, 0, 10.0, peaks, 1650.0)  # 825 TFLOP/s
    assert r["frac_bf16"] == 0.5 and r["frac_bf16_nominal"] == round(825 / 2250, 4)
    b = bench.part_row("bwd", 8.25e12, 0, 10.0, peaks, 1650.0)
    assert b["frac_bf16_8d"] == 0.4
    d = bench.part_row("decode", 0, 4e9, 1.0, peaks, 1650.0)  # 4000 GB/s
    assert d["frac_hbm"] == round(4000 / 6500, 4) and d["frac_hbm_nominal"] == 0.5


def test_recorded_traffic_is_tied_to_kernel_sources(tmp_path, monkeypatch):
    assert bench.recorded_traffic("no such part", "step32k") is None
    with open(bench.TRAFFIC_FILE) as f:
        table = json.load(f)
    keys = [(e["part"], w) for e in table for w in e["workloads"]]
    assert len(keys) == len(set(keys)), "one entry per part and workload"
    for n, e in enumerate(table):
        assert set(e) >= {"part", "workloads", "sources", "sources_sha256", "dram_bytes_per_launch", "capture"}
        fresh = bench.sources_sha256(e["sources"]) == e["sources_sha256"]
        for w in e["workloads"]:
            bench.workload(w)  # a known workload
            assert bench.recorded_traffic(e["part"], w) == (e["dram_bytes_per_launch"] if fresh else None)
        # a stale hash reads as "no capture for this kernel"
        bad = [dict(x) for x in table]
        bad[n]["sources_sha256"] = "0" * 64
        p = tmp_path / "t.json"
        p.write_text(json.dumps(bad))
        monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
        assert bench.recorded_traffic(e["part"], e["workloads"][0]) is None
        monkeypatch.setattr(bench, "TRAFFIC_FILE", os.path.join(ROOT, "profiles", "kernel_traffic.json"))
    # the same part name in another workload (another launch shape) has no figure of its own
    assert bench.recorded_traffic("bwd sink+window", "bwd128k") is None or any(
        e["part"] == "bwd sink+window" and "bwd128k" in e["workloads"] for e in table)


def test_workloads_and_useful_work():
    w = bench.workload("step32k")
    assert w["prefill"]["S"] == 32768 and w["decode"]["L"] == 4160
    assert bench.pairs_of(bench.SINK_WINDOW, 32768) == 126763008
    assert bench.pairs_of(bench.FULL, 32768) == 32768 * 32769 // 2
    assert bench.pairs_of(bench.BLOCK_SPARSE, 131072) == 398032896
    import attention_sink_long_b200 as lg

    bs = bench.workload("blocksparse128k")
    assert bs["decode"]["L"] == lg.lg_kv_compact_rows(bench.BLOCK_SPARSE, bs["prefill"]["S"])
    ho = bench.workload("handoff")["handoff"]
    assert lg.lg_kv_compact_rows(ho["pattern"], ho["S"]) == 4096
    pg = bench.workload("decode_paged")["paged"]
    assert lg.lg_kv_compact_rows(pg["pattern"], pg["S"]) + pg["appended"] == pg["L"] == 4160
    assert bench.work_unit(bench.workload("decode_paged"))[0] == "GB/s"
    assert bench.work_unit(bench.workload("step32k"))[0] == "TFLOP/s"


def _run(cmd, timeout=240):
    return subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout,
                          env=dict(os.environ, MASTER_ADDR="127.0.0.1"))


def test_reference_arm_prints_one_line():
    r = _run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    r = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
              "--master-addr", "127.0.0.1", "--master-port", "29533", "bench.py", "--impl", "reference",
              "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2
