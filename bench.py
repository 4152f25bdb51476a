#!/usr/bin/env python3
"""Benchmark of the LongGen sparse-attention hot path on B200.

One step = one pass of every kernel of the path over the Llama-2-7B-shaped 32K
workload (B=1, H=Hkv=32, D=128, bf16, 64-token blocks):
  * prefill forward, sink+window pattern {64, 1, 64, 0} (64 sink + 4096 window tokens);
  * prefill forward, full causal pattern (the middle-layer dense case);
  * training backward of the sink+window layer (preprocess, main, dQ convert);
  * decode of one sparse layer over its reduced cache: batch 32, 32 heads,
    4160 cached rows (64 sink + 4096 window), split-KV with the LSE merge.
The block iterator (pattern expansion) runs inside the kernels.

value = useful FLOPs of the whole step (unmasked pairs only: 4*D per pair
forward, 10*D per pair backward, 4*D per cached row decode) / device time.
Per-kernel rows (TFLOP/s, GB/s and roofline fractions) are in "rows".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload step32k|fwd128k|bwd128k|decode]

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
device (weak scaling, independent replicas -- the path has no exchange step);
the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn fwd/bwd useful TFLOP/s & decode GB/s; % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The B200 data-sheet figures (dense bf16, HBM3e), reported beside the measured
# peaks for context; the measured fractions are the headline.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
SINK_WINDOW = (64, 1, 64, 0)
FULL = (64, 0, 2**31 - 1, 0)
BLOCK_SPARSE = (64, 1, 16, 32)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", choices=["step32k", "fwd128k", "bwd128k", "decode", "handoff", "blocksparse128k",
                                           "varlen", "decode_paged", "gqa32k", "fp8qk32k", "decode_gqa", "d64_32k",
                                           "pair32k"],
                    default="step32k")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end loop")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the 128K / 32-layer / head-dim-64 rows the default step32k run adds")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline")
    return ap.parse_args(argv)


def max_over_ranks(value: float, dist, device) -> float:
    """The largest value over all ranks (identity without a process group)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


SUSTAINED_REGION_S = 2.0  # a timed region this long runs at the power-capped sustained rate


def pick_peak(peaks, region_s, bound):
    """Roofline denominator: the measured burst figure for a kernel timed in a
    short region (the cuBLAS burst it is compared with is timed the same way),
    the sustained figure once the timed region lasts seconds."""
    if bound == "hbm":
        return peaks["hbm_gbs"], "copy bandwidth"
    if region_s >= SUSTAINED_REGION_S:
        return peaks["bf16_tflops_sustained"], f"sustained (timed region {region_s:.2f} s)"
    return peaks["bf16_tflops"], f"burst (timed region {region_s:.2f} s)"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "kernel_traffic.json")


def sources_sha256(files):
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(part_name, workload_name):
    """DRAM bytes per launch of this part of this workload (the same launch
    shape) from the committed ncu capture, or None when there is none or the
    kernel's sources changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            table = json.load(f)
    except Exception:
        return None
    for e in table:
        if e["part"] == part_name and workload_name in e["workloads"]:
            if sources_sha256(e["sources"]) != e["sources_sha256"]:
                return None
            return int(e["dram_bytes_per_launch"])
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# Workload description (shared by both arms)
# ----------------------------------------------------------------------------

def workload(name):
    D = 128
    if name == "step32k":
        return {
            "workload": "llama2-7b-shaped 32K step: fwd sink+window + fwd dense + bwd sink+window + sparse-layer decode",
            "prefill": {"B": 1, "S": 32768, "H": 32, "Hkv": 32, "D": D},
            "fwd": [("sink+window", SINK_WINDOW), ("dense", FULL)],
            "bwd": [("sink+window", SINK_WINDOW)],
            "decode": {"B": 32, "H": 32, "Hkv": 32, "D": D, "L": 4160},
        }
    if name == "fwd128k":
        return {"workload": "128K block-sparse prefill forward {64,1,16,32}",
                "prefill": {"B": 1, "S": 131072, "H": 32, "Hkv": 32, "D": D},
                "fwd": [("block-sparse", BLOCK_SPARSE)], "bwd": [], "decode": None}
    if name == "decode_gqa":
        return {"workload": "grouped-query decode over the sink+window cache: B32 H32 Hkv8 D128, 4160 rows",
                "prefill": None, "fwd": [], "bwd": [], "decode": {"B": 32, "H": 32, "Hkv": 8, "D": D, "L": 4160}}
    if name == "fp8qk32k":
        # Throughput experiment (no fp8 claim on the pages): Q and K arrive in fp8 e4m3 with
        # dequantisation scales, S runs on the fp8 tensor-core path, P V in bf16.
        return {"workload": "fp8 Q/K forward 32K (S on the fp8 path, P V bf16): sink+window + dense, "
                            "B1 H32 D128",
                "prefill": {"B": 1, "S": 32768, "H": 32, "Hkv": 32, "D": D},
                "fwd": [("sink+window fp8qk", SINK_WINDOW), ("dense fp8qk", FULL)], "bwd": [], "decode": None,
                "fp8qk": True}
    if name == "gqa32k":
        return {"workload": "grouped-query 32K: fwd + training bwd sink+window {64,1,64,0}, H32 Hkv8 D128",
                "prefill": {"B": 1, "S": 32768, "H": 32, "Hkv": 8, "D": D},
                "fwd": [("sink+window", SINK_WINDOW)], "bwd": [("sink+window", SINK_WINDOW)], "decode": None}
    if name == "pair32k":
        # The CTA-pair forward (lg_sparse_attn_fwd_pair: 256-row cta_group::2 MMAs) beside the default one.
        return {"workload": "CTA-pair forward vs the default forward, 32K dense and sink+window, B1 H32 D128",
                "prefill": {"B": 1, "S": 32768, "H": 32, "Hkv": 32, "D": D},
                "fwd": [("dense pair", FULL), ("dense", FULL), ("sink+window pair", SINK_WINDOW),
                        ("sink+window", SINK_WINDOW)], "bwd": [], "decode": None, "pair_parts": ["dense pair",
                                                                                                 "sink+window pair"]}
    if name == "d64_32k":
        return {"workload": "head dim 64 sink+window 32K: fwd + training bwd {64,1,64,0}, B1 H32 D64",
                "prefill": {"B": 1, "S": 32768, "H": 32, "Hkv": 32, "D": 64},
                "fwd": [("sink+window d64", SINK_WINDOW)], "bwd": [("sink+window d64", SINK_WINDOW)],
                "decode": None}
    if name == "bwd128k":
        return {"workload": "128K sink+window training backward {64,1,64,0}",
                "prefill": {"B": 1, "S": 131072, "H": 32, "Hkv": 32, "D": D},
                "fwd": [], "bwd": [("sink+window", SINK_WINDOW)], "decode": None}
    if name == "decode":
        return {"workload": "32-layer hybrid decode step: 21 sparse layers (4160 rows) + 11 full layers (131072 rows)",
                "prefill": None, "fwd": [], "bwd": [],
                "decode": {"B": 32, "H": 32, "Hkv": 32, "D": D, "L": 4160, "L_full": 131072}}
    if name == "blocksparse128k":
        # 5056 = the block-sparse reduced cache of a 128K prompt (lg_kv_compact_rows).
        return {"workload": "128K block-sparse {64,1,16,32}: prefill forward + training backward + "
                            "decode over the reduced cache (5056 rows, B32)",
                "prefill": {"B": 1, "S": 131072, "H": 32, "Hkv": 32, "D": D},
                "fwd": [("block-sparse", BLOCK_SPARSE)], "bwd": [("block-sparse", BLOCK_SPARSE)],
                "decode": {"B": 32, "H": 32, "Hkv": 32, "D": D, "L": 5056}}
    if name == "varlen":
        return {"workload": "variable-length sink+window forward + training backward: 8 packed sequences of "
                            "32K..512 tokens (64K rows), H32 D128",
                "prefill": None, "fwd": [], "bwd": [], "decode": None,
                "varlen": {"lens": [32768, 16384, 8192, 4096, 2048, 1024, 512, 512], "H": 32, "Hkv": 32, "D": D,
                           "pattern": SINK_WINDOW}}
    if name == "decode_paged":
        # The spec sparse-layer cache (64 sink + 4096 window rows = 4160) reached the way a
        # server reaches it: hand-off of an 8K prompt into pages, then 64 appended tokens.
        return {"workload": "paged decode over the sink+window ring cache: B32 H32 D128, 4160 rows per sequence in "
                            "64-row pages of a shuffled pool (hand-off of 8K prompts + 64 appended tokens)",
                "prefill": None, "fwd": [], "bwd": [], "decode": None,
                "paged": {"B": 32, "H": 32, "Hkv": 32, "D": D, "S": 8192, "appended": 64, "L": 4160,
                          "pattern": SINK_WINDOW}}
    if name == "handoff":
        return {"workload": "prefill->decode hand-off: reduced sink+window KV cache of 32K-token prompts, "
                            "B32 Hkv32 D128",
                "prefill": None, "fwd": [], "bwd": [], "decode": None,
                "handoff": {"B": 32, "S": 32768, "Hkv": 32, "D": D, "pattern": SINK_WINDOW}}
    raise ValueError(name)


def pairs_of(pattern, S):
    """Unmasked pairs per head, from the library's host expansion (closed form)."""
    import attention_sink_long_b200 as lg

    return lg.lg_pattern_pairs(pattern, S)


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# CUDA arm
# ----------------------------------------------------------------------------

class CudaStep:
    """Device buffers and the launch sequence of one step."""

    def __init__(self, wl, device):
        import torch

        import attention_sink_long_b200 as lg
        import synthetic_inputs as si

        self.lg, self.torch, self.wl, self.dev = lg, torch, wl, device
        self.stream = torch.cuda.current_stream(device)
        self.parts = []  # (name, kind, useful_flops, useful_bytes, launches)
        pf = wl["prefill"]
        if pf is not None:
            B, S, H, Hkv, D = pf["B"], pf["S"], pf["H"], pf["Hkv"], pf["D"]
            self.scale = 1.0 / math.sqrt(D)
            self.q, self.k, self.v, self.do = si.prefill_inputs_device(B, S, H, Hkv, D, device, with_dout=True)
            if wl.get("fp8qk"):
                # caller-side quantisation (outside the timed step): e4m3 with scales 4 and 2
                self.q8 = (self.q.float() * 4.0).to(torch.float8_e4m3fn)
                self.k8 = (self.k.float() * 2.0).to(torch.float8_e4m3fn)
            self.o = {n: torch.empty_like(self.q) for n, _ in wl["fwd"]}
            self.lse = {n: torch.empty(B, H, S, dtype=torch.float32, device=device) for n, _ in wl["fwd"]}
            for n, p in wl["fwd"]:
                self.parts.append((f"fwd {n}", "fwd_fp8qk" if wl.get("fp8qk") else "fwd",
                                   4 * D * pairs_of(p, S) * B * H, None, 1))
            if wl["bwd"]:
                self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
                self.bwd_ws = torch.empty(max(lg.lg_sparse_attn_bwd_workspace(wl["bwd"][0][1], B, S, H, Hkv, D), 1),
                                          dtype=torch.uint8, device=device)
                for n, p in wl["bwd"]:
                    if n not in self.o:  # the backward needs O and LSE of its own forward
                        self.o[n] = torch.empty_like(self.q)
                        self.lse[n] = torch.empty(B, H, S, dtype=torch.float32, device=device)
                        lg.lg_sparse_attn_fwd(p, self.q, self.k, self.v, self.o[n], self.lse[n], self.scale)
                    self.parts.append((f"bwd {n}", "bwd", 10 * D * pairs_of(p, S) * B * H, None, 3))
        dc = wl["decode"]
        if dc is not None:
            B, H, Hkv, D, L = dc["B"], dc["H"], dc["Hkv"], dc["D"], dc["L"]
            self.dq_in, self.kc, self.vc, self.lens = si.decode_inputs_device(B, H, Hkv, D, L, device)
            self.do_out = torch.empty(B, H, D, dtype=torch.bfloat16, device=device)
            self.dlse = torch.empty(B, H, dtype=torch.float32, device=device)
            self.dws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, L), 1), dtype=torch.uint8,
                                   device=device)
            nbytes = 2 * B * L * Hkv * D * 2 + 2 * B * H * D * 2
            name = "decode sparse layer" if Hkv == H else f"decode sparse layer, {H // Hkv} query heads per KV head"
            self.parts.append((name, "decode", 4 * D * L * B * H, nbytes, 1))
            if "L_full" in dc:
                Lf = dc["L_full"]
                self.fq, self.fkc, self.fvc, self.flens = si.decode_inputs_device(B, H, Hkv, D, Lf, device, seed=2000)
                self.fws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, Lf), 1), dtype=torch.uint8,
                                       device=device)
                fbytes = 2 * B * Lf * Hkv * D * 2 + 2 * B * H * D * 2
                self.parts.append(("decode full layer", "decode_full", 4 * D * Lf * B * H, fbytes, 1))
        vl = wl.get("varlen")
        if vl is not None:
            lens, H, Hkv, D = vl["lens"], vl["H"], vl["Hkv"], vl["D"]
            total = sum(lens)
            self.scale = 1.0 / math.sqrt(D)
            self.vq = si.device_normal((total, H, D), si.SEED_BASE + 0, device)
            self.vk = si.device_normal((total, Hkv, D), si.SEED_BASE + 1, device)
            self.vv = si.device_normal((total, Hkv, D), si.SEED_BASE + 2, device)
            self.vo = torch.empty_like(self.vq)
            self.vlse = torch.empty(H, total, dtype=torch.float32, device=device)
            cu = [0]
            for n in lens:
                cu.append(cu[-1] + n)
            self.vcu = torch.tensor(cu, dtype=torch.int32, device=device)
            flops = sum(4 * D * pairs_of(vl["pattern"], n) * H for n in lens)
            self.parts.append(("fwd varlen sink+window", "fwd", flops, None, 1))
            self.vdo = si.device_normal((total, H, D), si.SEED_BASE + 3, device)
            self.vdq, self.vdk, self.vdv = (torch.empty_like(self.vq), torch.empty_like(self.vk),
                                            torch.empty_like(self.vv))
            self.vws = torch.empty(lg.lg_sparse_attn_bwd_workspace(vl["pattern"], 1, total, H, Hkv, D),
                                   dtype=torch.uint8, device=device)
            self.parts.append(("bwd varlen sink+window", "bwd", 10 * flops // 4, None, 3))
        pg = wl.get("paged")
        if pg is not None:
            self._setup_paged(pg, device)
        ho = wl.get("handoff")
        if ho is not None:
            B, S, Hkv, D = ho["B"], ho["S"], ho["Hkv"], ho["D"]
            self.hk = si.device_normal((B, S, Hkv, D), si.SEED_BASE + 1, device)
            self.hv = si.device_normal((B, S, Hkv, D), si.SEED_BASE + 2, device)
            rows = lg.lg_kv_compact_rows(ho["pattern"], S)
            self.hkc = torch.empty(B, rows + 64, Hkv, D, dtype=torch.bfloat16, device=device)
            self.hvc = torch.empty_like(self.hkc)
            self.hlens = torch.empty(B, dtype=torch.int32, device=device)
            nbytes = 2 * 2 * B * rows * Hkv * D * 2  # K and V, each row read once and written once
            self.parts.append(("handoff sink+window", "copy", 0, nbytes, 1))

    def _setup_paged(self, pg, device):
        """Paged ring cache in the state a decode server reaches: lg_kv_compact_paged of a prompt, then
        lg_kv_append_paged of `appended` tokens; the timed part is lg_sparse_decode_paged."""
        lg, torch = self.lg, self.torch
        import synthetic_inputs as si

        B, H, Hkv, D, S, A = pg["B"], pg["H"], pg["Hkv"], pg["D"], pg["S"], pg["appended"]
        rows = lg.lg_kv_compact_rows(pg["pattern"], S)
        MB = rows // 64 + 2
        P = B * MB + B
        perm = torch.randperm(P, generator=torch.Generator().manual_seed(7))[: B * MB]
        self.ptable = perm.view(B, MB).to(torch.int32).to(device)
        self.pids = torch.empty(B, MB, dtype=torch.int32, device=device)
        self.plens = torch.empty(B, dtype=torch.int32, device=device)
        self.ppos = torch.empty(B, dtype=torch.int32, device=device)
        self.kpool = torch.empty(P, 64, Hkv, D, dtype=torch.bfloat16, device=device)
        self.vpool = torch.empty_like(self.kpool)
        state = (self.kpool, self.vpool, self.ptable, self.pids, self.plens, self.ppos)
        k = si.device_normal((B, S + A, Hkv, D), si.SEED_BASE + 1, device)
        v = si.device_normal((B, S + A, Hkv, D), si.SEED_BASE + 2, device)
        lg.lg_kv_compact_paged(pg["pattern"], k[:, :S].contiguous(), v[:, :S].contiguous(), *state)
        for t in range(S, S + A):
            lg.lg_kv_append_paged(pg["pattern"], k[:, t].contiguous(), v[:, t].contiguous(), *state)
        del k, v
        torch.cuda.synchronize()
        assert int(self.plens.min()) == int(self.plens.max()) == pg["L"], self.plens
        self.pq = si.device_normal((B, H, D), si.SEED_BASE + 0, device)
        self.po = torch.empty(B, H, D, dtype=torch.bfloat16, device=device)
        self.plse = torch.empty(B, H, dtype=torch.float32, device=device)
        self.pws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, 64 * MB), 1), dtype=torch.uint8,
                               device=device)
        L = pg["L"]
        nbytes = 2 * B * L * Hkv * D * 2 + 2 * B * H * D * 2
        self.parts.append(("decode paged sink+window", "decode", 4 * D * L * B * H, nbytes, 1))

    def run(self, events=None):
        """Launch one step; if events is given, record one event after each part."""
        lg, wl = self.lg, self.wl
        i = 0
        for n, p in wl["fwd"]:
            if wl.get("fp8qk"):
                lg.lg_sparse_attn_fwd_fp8qk(p, self.q8, self.k8, self.v, 0.25, 0.5, self.o[n], self.lse[n],
                                            self.scale)
            elif n in wl.get("pair_parts", ()):
                lg.lg_sparse_attn_fwd_pair(p, self.q, self.k, self.v, self.o[n], self.lse[n], self.scale)
            else:
                lg.lg_sparse_attn_fwd(p, self.q, self.k, self.v, self.o[n], self.lse[n], self.scale)
            if events is not None:
                events[i].record(self.stream)
            i += 1
        for n, p in wl["bwd"]:
            lg.lg_sparse_attn_bwd(p, self.q, self.k, self.v, self.o[n], self.do, self.lse[n], self.dq, self.dk,
                                  self.dv, self.scale, self.bwd_ws)
            if events is not None:
                events[i].record(self.stream)
            i += 1
        if wl["decode"] is not None:
            lg.lg_sparse_decode(self.dq_in, self.kc, self.vc, self.lens, self.do_out, self.dlse, self.scale_dec(),
                                workspace=self.dws)
            if events is not None:
                events[i].record(self.stream)
            i += 1
            if "L_full" in wl["decode"]:
                lg.lg_sparse_decode(self.fq, self.fkc, self.fvc, self.flens, self.do_out, self.dlse,
                                    self.scale_dec(), workspace=self.fws)
                if events is not None:
                    events[i].record(self.stream)
                i += 1
        if wl.get("varlen") is not None:
            vl = wl["varlen"]
            lg.lg_sparse_attn_fwd_varlen(vl["pattern"], self.vq, self.vk, self.vv, self.vo, self.vlse, self.vcu,
                                         max(vl["lens"]), self.scale)
            if events is not None:
                events[i].record(self.stream)
            i += 1
            lg.lg_sparse_attn_bwd_varlen(vl["pattern"], self.vq, self.vk, self.vv, self.vo, self.vdo, self.vlse,
                                         self.vdq, self.vdk, self.vdv, self.vcu, max(vl["lens"]), self.scale,
                                         self.vws)
            if events is not None:
                events[i].record(self.stream)
            i += 1
        if wl.get("paged") is not None:
            lg.lg_sparse_decode_paged(self.pq, self.kpool, self.vpool, self.ptable, self.plens, self.po, self.plse,
                                      1.0 / math.sqrt(wl["paged"]["D"]), workspace=self.pws)
            if events is not None:
                events[i].record(self.stream)
            i += 1
        if wl.get("handoff") is not None:
            lg.lg_kv_compact(wl["handoff"]["pattern"], self.hk, self.hv, self.hkc, self.hvc, self.hlens)
            if events is not None:
                events[i].record(self.stream)
            i += 1

    def scale_dec(self):
        return 1.0 / math.sqrt(self.wl["decode"]["D"])

    def e2e_parts(self):
        """Indices of the parts the end-to-end loop runs: all of them, except in the 32-layer decode step,
        where only the sparse-layer call runs end to end (its full-layer caches, 69 GB, stay on the device;
        uploading them every step is not what a decode server does)."""
        if self.wl["workload"].startswith("32-layer"):
            return [0]
        return list(range(len(self.parts)))

    def run_e2e(self):
        if self.wl["workload"].startswith("32-layer"):
            self.lg.lg_sparse_decode(self.dq_in, self.kc, self.vc, self.lens, self.do_out, self.dlse,
                                     self.scale_dec(), workspace=self.dws)
        else:
            self.run()

    def launches_per_step(self):
        return sum(p[4] for p in self.parts)

    def step_weights(self):
        """How many times each part counts per reported step (decode: 21 sparse + 11 full layers)."""
        if self.wl["workload"].startswith("32-layer"):
            return [21 if p[2] and p[1] == "decode" else 11 for p in self.parts]
        return [1] * len(self.parts)


def host_buffers(step):
    """Pinned host copies of the step's inputs and outputs, for the end-to-end loop."""
    torch = step.torch
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t.cpu())  # noqa: E731
    ins, outs = [], []
    names = ("q8", "k8", "v") if step.wl.get("fp8qk") else ("q", "k", "v", "do")
    for name in names + ("dq_in", "kc", "vc", "lens", "hk", "hv", "vq", "vk", "vv", "vdo", "pq", "kpool",
                 "vpool", "ptable", "plens"):
        if hasattr(step, name):
            ins.append((name, getattr(step, name), pin(getattr(step, name))))
    for d in ("o", "lse"):
        if hasattr(step, d):
            for t in getattr(step, d).values():
                outs.append((t, torch.empty(t.shape, dtype=t.dtype, pin_memory=True)))
    for name in ("dq", "dk", "dv", "do_out", "dlse", "hkc", "hvc", "hlens", "vo", "vlse", "vdq", "vdk", "vdv", "po", "plse"):
        if hasattr(step, name):
            t = getattr(step, name)
            outs.append((t, torch.empty(t.shape, dtype=t.dtype, pin_memory=True)))
    return ins, outs


def e2e_steps(step, ins, outs, nsteps):
    """nsteps end-to-end steps: upload inputs, run, download outputs. Inputs have two device sets used in
    turn, so step k+1's upload runs while step k computes; uploads and downloads run on their own streams,
    so step k's download overlaps step k+1's upload. Events keep each buffer's uses in order: an input set is
    overwritten only after the kernels of the step before last read it, outputs only after the previous
    step's download. Returns device ms from the first upload to the last download."""
    torch = step.torch
    comp = step.stream
    s_in = torch.cuda.Stream(device=step.dev)
    s_out = torch.cuda.Stream(device=step.dev)
    sets = [{name: d for name, d, _ in ins}, {name: torch.empty_like(d) for name, d, _ in ins}]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    free_set, free_out = [e0, e0], e0
    for k in range(nsteps):
        cur = sets[k % 2]
        s_in.wait_event(free_set[k % 2])
        with torch.cuda.stream(s_in):
            for name, _, h in ins:
                cur[name].copy_(h, non_blocking=True)
        ready = torch.cuda.Event()
        ready.record(s_in)
        comp.wait_event(ready)
        comp.wait_event(free_out)
        for name, t in cur.items():
            setattr(step, name, t)
        step.run_e2e()
        done = torch.cuda.Event()
        done.record(comp)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            for d, h in outs:
                h.copy_(d, non_blocking=True)
        downloaded = torch.cuda.Event()
        downloaded.record(s_out)
        free_set[k % 2], free_out = done, downloaded
    comp.wait_event(free_out)
    e1.record(comp)
    torch.cuda.synchronize()
    for name, t in sets[0].items():  # the step keeps its original input tensors
        setattr(step, name, t)
    return e0.elapsed_time(e1)


def cuda_arm(args, rank, world, dist):
    import torch

    import attention_sink_long_b200 as lg
    from attention_sink_long_b200 import build as lgbuild

    lgbuild.build()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = workload(args.workload)
    step = CudaStep(wl, device)
    wl = step.wl
    # Skip parts the library does not provide (e.g. a kernel not built yet): probe once.
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    assert lg.lg_device_status(local) == 0, "a bounded device wait ran out during warm-up"

    nparts = len(step.parts)
    per_part_ms = [[] for _ in range(nparts)]
    clocks = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nparts)] for _ in range(args.steps)]
    t0.record(step.stream)
    for k in range(args.steps):
        step.run(evs[k])
    t1.record(step.stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    for k in range(args.steps):
        prev = t0 if k == 0 else evs[k - 1][-1]
        for i in range(nparts):
            per_part_ms[i].append(prev.elapsed_time(evs[k][i]))
            prev = evs[k][i]
    assert lg.lg_device_status(local) == 0, "a bounded device wait ran out during the timed region"

    total_ms = max_over_ranks(total_ms, dist, device)

    weights = step.step_weights()
    step_flops = sum(w * p[2] for w, p in zip(weights, step.parts))
    ms_per_step = total_ms / args.steps
    if wl["workload"].startswith("32-layer"):
        # Reported decode step: 21 sparse-layer + 11 full-layer calls, from the per-call times.
        ms_per_step = sum(w * statistics.mean(per_part_ms[i]) for i, w in enumerate(weights))
    # A workload of HBM-bound parts only (decode, the hand-off copy) reports bytes moved per second.
    step_bytes = sum(w * (p[3] or 0) for w, p in zip(weights, step.parts))
    by_bytes = work_unit(wl)[0] == "GB/s"
    unit = "GB/s" if by_bytes else "TFLOP/s"
    value = world * (step_bytes / (ms_per_step * 1e-3) / 1e9 if by_bytes else
                     step_flops / (ms_per_step * 1e-3) / 1e12)

    peaks, peak_src = load_peaks()
    tensor_peak, tensor_kind = pick_peak(peaks, total_ms * 1e-3, "tensor")
    rows = {}
    dominant = None
    for i, (name, kind, flops, nbytes, nl) in enumerate(step.parts):
        ms = statistics.mean(per_part_ms[i])
        rows[name] = part_row(kind, flops, nbytes, ms, peaks, tensor_peak)
        if dominant is None or ms * weights[i] > dominant[1]:
            dominant = (i, ms * weights[i])
    di = dominant[0]
    dname, dkind, dflops, dbytes, _ = step.parts[di]
    dms = statistics.mean(per_part_ms[di])
    if dkind.startswith("decode") or dkind == "copy":
        achieved = dbytes / (dms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4)}
        roof["peak_source"] = f"{peak_src} (copy bandwidth)"
        roof["frac_nominal"] = round(achieved / NOMINAL_PEAKS["hbm_gbs"], 4)
    else:
        achieved = dflops / (dms * 1e-3) / 1e12
        pk = tensor_peak * 4 / 3 if dkind == "fwd_fp8qk" else tensor_peak
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(pk, 1), "unit": "TFLOP/s",
                "frac": round(achieved / pk, 4)}
        roof["peak_source"] = f"{peak_src} bf16 dense, {tensor_kind}" + (
            "; x 4/3: S (half the FLOPs) on the fp8 path at twice the bf16 rate (nominal ratio)"
            if dkind == "fwd_fp8qk" else "")
        # The same kernel against the other measured figure, for context.
        other = peaks["bf16_tflops_sustained"] if pk == peaks["bf16_tflops"] else peaks["bf16_tflops"]
        roof["frac_" + ("sustained" if pk == peaks["bf16_tflops"] else "burst")] = round(achieved / other, 4)
        nom = NOMINAL_PEAKS["bf16_tflops"] * (4 / 3 if dkind == "fwd_fp8qk" else 1)
        roof["frac_nominal"] = round(achieved / nom, 4)
    roof["traffic"] = recorded_traffic(dname, args.workload)
    roof["kernel"] = dname

    # End-to-end through the public API with pinned host buffers.
    e2e = None
    if not args.no_e2e:
        ins, outs = host_buffers(step)
        bi = sum(h.numel() * h.element_size() for _, _, h in ins)
        bo = sum(h.numel() * h.element_size() for _, h in outs)
        e2e_steps(step, ins, outs, 1)  # warm-up
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        # As many steps as the device-timed region: the first upload and the last
        # download have nothing to overlap with, and over a few steps that fill
        # and drain would dominate what is a steady-state rate.
        ek = max(1, args.steps)
        ems = max_over_ranks(e2e_steps(step, ins, outs, ek) / ek, dist, device)
        idx = step.e2e_parts()
        e_flops = sum(step.parts[i][2] for i in idx)
        e_bytes = sum(step.parts[i][3] or 0 for i in idx)
        e2e_v = e_bytes / (ems * 1e-3) / 1e9 if by_bytes else e_flops / (ems * 1e-3) / 1e12
        e2e = {"value": round(world * e2e_v, 3), "unit": unit,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(ems, 3), "steps": ek,
               "copies": "every step uploads all its inputs and downloads all its outputs (pinned host memory); "
                         "inputs alternate between two device sets and uploads / downloads run on their own "
                         "streams, so step k+1's upload overlaps step k's compute and download"}
        if len(idx) < len(step.parts):
            e2e["scope"] = "the sparse-layer decode call end to end (cache, query up; output, LSE down); the " \
                           "full-layer caches stay on the device"

    # The metric's other configurations (128K forward and backward, the 32-layer
    # decode step, head dim 64), each timed alone after the step: one GPU only.
    others = None
    if world == 1 and args.workload == "step32k" and not args.no_other_workloads:
        others = other_workload_rows(device, steps=10, warmup=3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    launches = args.steps * step.launches_per_step()
    pf = wl["prefill"]
    config = {"workload": wl["workload"], "l2": "inputs larger than L2 (126 MB), no flush",
              "parallelism": f"dp{world} (independent replicas, no collective)"}
    if pf:
        config.update({"prefill_shape": pf, "patterns": {n: list(p) for n, p in wl["fwd"] + wl["bwd"]}})
    if wl["decode"]:
        config["decode_shape"] = wl["decode"]
    if wl.get("varlen"):
        config["varlen_shape"] = {k: (list(v) if k == "pattern" else v) for k, v in wl["varlen"].items()}
    if wl.get("paged"):
        config["paged_shape"] = {k: (list(v) if k == "pattern" else v) for k, v in wl["paged"].items()}
    if wl.get("handoff"):
        config["handoff_shape"] = {k: (list(v) if k == "pattern" else v) for k, v in wl["handoff"].items()}
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; no dataset, no weights)",
        "config": config, "roofline": roof, "rows": rows, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches, "clocks": clk,
    }
    if others is not None:
        line["rows_other_workloads"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)


def part_row(kind, flops, nbytes, ms, peaks, tensor_peak):
    """Per-part figures: useful TFLOP/s (and GB/s for HBM-bound parts) with their roofline fractions."""
    r = {"ms": round(ms, 4), "useful_tflops": round(flops / (ms * 1e-3) / 1e12, 2)}
    if kind.startswith("decode") or kind == "copy":
        r["gbs"] = round(nbytes / (ms * 1e-3) / 1e9, 1)
        r["frac_hbm"] = round(r["gbs"] / peaks["hbm_gbs"], 4)
        r["frac_hbm_nominal"] = round(r["gbs"] / NOMINAL_PEAKS["hbm_gbs"], 4)
    elif kind == "fwd_fp8qk":
        # half of the FLOPs (S) at the fp8 rate, twice bf16: the mixed peak is 4/3 of bf16's
        r["frac_mixed_fp8_bf16_peak"] = round(r["useful_tflops"] / (tensor_peak * 4 / 3), 4)
    else:
        r["frac_bf16"] = round(r["useful_tflops"] / tensor_peak, 4)
        r["frac_bf16_sustained"] = round(r["useful_tflops"] / peaks["bf16_tflops_sustained"], 4)
        r["frac_bf16_nominal"] = round(r["useful_tflops"] / NOMINAL_PEAKS["bf16_tflops"], 4)
        if kind == "bwd":
            # 10 D FLOP per pair counts the five GEMMs (S recomputed); 8 D leaves the recompute out.
            r["useful_tflops_8d"] = round(0.8 * r["useful_tflops"], 2)
            r["frac_bf16_8d"] = round(0.8 * r["useful_tflops"] / tensor_peak, 4)
    return r


# The other configurations of the metric, timed in the default run beside the
# 32K step (each alone, CUDA events, after warm-up): the 128K block-sparse
# forward, the 128K sink+window backward, the full-layer decode and the
# 32-layer decode step it makes with the sparse layer, the head-dim-64
# sink+window forward + backward at 32K, and the CTA-pair forward beside the
# default one.
OTHER_WORKLOADS = ["fwd128k", "bwd128k", "decode", "d64_32k", "pair32k"]


def other_workload_rows(device, steps, warmup):
    import torch

    peaks, _ = load_peaks()
    out = {}
    for name in OTHER_WORKLOADS:
        wl = workload(name)
        step = CudaStep(wl, device)
        for _ in range(warmup):
            step.run()
        torch.cuda.synchronize()
        nparts = len(step.parts)
        t0 = torch.cuda.Event(enable_timing=True)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nparts)] for _ in range(steps)]
        t0.record(step.stream)
        for k in range(steps):
            step.run(evs[k])
        torch.cuda.synchronize()
        per = [[] for _ in range(nparts)]
        for k in range(steps):
            prev = t0 if k == 0 else evs[k - 1][-1]
            for i in range(nparts):
                per[i].append(prev.elapsed_time(evs[k][i]))
                prev = evs[k][i]
        region_s = t0.elapsed_time(evs[-1][-1]) * 1e-3
        tensor_peak, kind_s = pick_peak(peaks, region_s, "tensor")
        rows = {}
        for i, (pname, kind, flops, nbytes, _) in enumerate(step.parts):
            rows[pname] = part_row(kind, flops, nbytes, statistics.mean(per[i]), peaks, tensor_peak)
        entry = {"workload": wl["workload"], "steps": steps, "tensor_peak": kind_s, "rows": rows}
        if name == "decode":
            w = step.step_weights()
            ms = sum(wi * statistics.mean(per[i]) for i, wi in enumerate(w))
            gb = sum(wi * p[3] for wi, p in zip(w, step.parts)) / 1e9
            entry["step_32_layers"] = {"ms": round(ms, 3), "gbs": round(gb / (ms * 1e-3), 1),
                                       "frac_hbm": round(gb / (ms * 1e-3) / peaks["hbm_gbs"], 4),
                                       "composition": "21 sparse-layer + 11 full-layer calls, from per-call times"}
        assert step.lg.lg_device_status(device.index or 0) == 0, f"a bounded device wait ran out in {name}"
        out[name] = entry
        del step
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------
# Oracle on the host: the CPU baseline and the reference arm
# ----------------------------------------------------------------------------

def oracle_sample(wl, budget_s, seed=11):
    """Runs the fp64 oracle on a bounded sample of the workload for about
    budget_s seconds; returns (useful_flops, seconds, description)."""
    import numpy as np

    import oracle
    import synthetic_inputs as si

    rng = np.random.default_rng(seed)
    flops = 0.0
    t_used = 0.0
    desc = []
    pf = wl["prefill"]
    jobs = []
    if pf:
        S, D = pf["S"], pf["D"]
        B, H = pf["B"], pf["H"]
        nqb = S // 64
        # One head's inputs drawn on the host with the same seeds (head 0 of a 1-head draw).
        q, k, v, do = si.prefill_inputs(1, S, 1, 1, D, with_dout=True)
        qh, kh, vh, doh = (t[0, :, 0].double().numpy() for t in (q, k, v, do))
        scale = 1.0 / math.sqrt(D)
        for n, p in wl["fwd"]:
            jobs.append(("fwd " + n, "fwd", p))
        for n, p in wl["bwd"]:
            jobs.append(("bwd " + n, "bwd", p))
    by_bytes = work_unit(wl)[0] == "GB/s"
    if wl["decode"]:
        jobs.append(("decode", "decode", None))
    if wl.get("paged"):
        jobs.append(("decode paged", "decode", None))
    vl = wl.get("varlen")
    if vl:
        # Forward rows of the longest sequence (the pattern acts inside each sequence alone).
        S, D = max(vl["lens"]), vl["D"]
        nqb = S // 64
        q, k, v, do = si.prefill_inputs(1, S, 1, 1, D, with_dout=True)
        qh, kh, vh, doh = (t[0, :, 0].double().numpy() for t in (q, k, v, do))
        scale = 1.0 / math.sqrt(D)
        jobs.append(("fwd varlen", "fwd", vl["pattern"]))
        jobs.append(("bwd varlen", "bwd", vl["pattern"]))
    ho = wl.get("handoff")
    if ho:
        # One KV head of one prompt, drawn on the host with the same seed as head 0.
        _, hk, hv = si.prefill_inputs(1, ho["S"], 1, 1, ho["D"])
        hk, hv = hk.double().numpy(), hv.double().numpy()
        jobs.append(("handoff", "handoff", oracle.Pattern(*ho["pattern"])))
    per_job = budget_s / max(1, len(jobs))
    for name, kind, p in jobs:
        t_start = time.perf_counter()
        n_done = 0
        job_flops = 0.0
        while time.perf_counter() - t_start < per_job:
            if kind in ("fwd", "bwd"):
                blk = int(rng.integers(0, nqb))
                rows = np.arange(blk * 64, blk * 64 + 64)
                op = oracle.Pattern(*p)
                pairs = int(oracle.allowed(rows[:, None], np.arange(S)[None, :], op).sum())
                if kind == "fwd":
                    oracle.attention_rows(qh, kh, vh, rows, op, scale)
                    job_flops += 4 * D * pairs
                else:
                    # dQ rows of a query block (S, dP, dQ: 6 D per pair), then dK / dV
                    # rows of a KV block (the dV and dK products: 4 D per pair), so the
                    # backward is credited the same 10 D per pair as the GPU arm.
                    oracle.attention_backward_rows(qh, kh, vh, doh, rows, op, scale)
                    job_flops += 6 * D * pairs
                    kblk = int(rng.integers(0, nqb))
                    krows = np.arange(kblk * 64, kblk * 64 + 64)
                    kpairs = int(oracle.allowed(np.arange(S)[:, None], krows[None, :], op).sum())
                    oracle.attention_backward_kv_rows(qh, kh, vh, doh, krows, op, scale)
                    job_flops += 4 * D * kpairs
            elif kind == "handoff":
                kc, vc, rws = oracle.reduced_cache(hk, hv, ho["S"], p)
                job_flops += 2 * 2 * len(rws) * ho["D"] * 2  # bytes: K and V rows read and written (bf16)
            else:
                dc = wl["decode"] or wl["paged"]
                L, D2 = dc["L"], dc["D"]
                qq, kc, vc, cl = si.decode_inputs(1, 1, 1, D2, L, seed=1000 + int(rng.integers(0, 1000)))
                oracle.decode(qq, kc, vc, cl.numpy(), 1.0 / math.sqrt(D2))
                job_flops += 2 * L * D2 * 2 if by_bytes else 4 * D2 * L  # K and V rows of one head (bf16)
            n_done += 1
        dt = time.perf_counter() - t_start
        flops += job_flops
        t_used += dt
        what = {"decode": "(b,h) rows", "handoff": "one-head prompt compactions",
                "bwd": "query blocks (dQ) + KV blocks (dK, dV) of one head"}.get(kind, "query blocks of one head")
        desc.append(f"{name}: {n_done} {what}")
    return flops, t_used, "; ".join(desc)


def work_unit(wl):
    """(unit, scale) of the work count: FLOPs, or bytes for workloads of HBM-bound parts only
    (decode, the hand-off copy)."""
    hbm_only = not (wl["prefill"] or wl.get("varlen")) and bool(wl["decode"] or wl.get("paged") or wl.get("handoff"))
    return ("GB/s", 1e9) if hbm_only else ("TFLOP/s", 1e12)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s):
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=cpu_cores()):
        flops, secs, desc = oracle_sample(wl, budget_s)
    unit, sc = work_unit(wl)
    return {"value": round(flops / secs / sc, 6), "unit": unit, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"fp64 numpy oracle, {secs:.1f} s: {desc}; useful FLOPs credited 4D/pair fwd, "
                      f"10D/pair bwd (6D for the sampled dQ rows + 4D for the sampled dK/dV rows, as the GPU "
                      f"arm's 10D), 4D/row decode; decode-only and hand-off workloads credited their bf16 "
                      f"bytes"}


def reference_arm(args, rank, world):
    if rank != 0:
        return
    wl = workload(args.workload)
    per_step = 1.5
    for _ in range(args.warmup):
        oracle_sample(wl, per_step / 3)
    tot_f, tot_s, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        f, s, desc = oracle_sample(wl, per_step)
        tot_f += f
        tot_s += s
    unit, sc = work_unit(wl)
    value = tot_f / tot_s / sc
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 upcast to f64)",
        "config": {"workload": wl["workload"], "sample": "bounded oracle sample per step (see cpu_baseline)"},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return 0
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        cuda_arm(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
