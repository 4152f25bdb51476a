"""Small single-kernel cases for profilers (ncu): each runs one kernel of the
path three times on seeded synthetic inputs a few GB in size at most, so a
capture of one launch (``ncu -k regex:<kernel> -s 1 -c 1 ...``) ends quickly.

    python -m attention_sink_long_b200.profile_cases <case>

Cases and the bench launch each stands for (DRAM bytes scale with rows x
heads for the prefill kernels and with the batch for decode and hand-off):
  fwd_dense    B1 H16 S16384 D128 full causal          (1/4 of the 32K H32 dense forward)
  fwd_sw       B1 H16 S16384 D128 sink+window          (1/4 of the 32K H32 sink+window forward)
  fwd_bs       B1 H8 S131072 D128 block-sparse         (1/4 of the 128K H32 block-sparse forward)
  fwd_pair     B1 H16 S16384 D128 full causal, on the CTA-pair forward (lg_sparse_attn_fwd_pair)
  bwd_sw       B1 H8 S32768 D128 sink+window backward  (1/4 of the 32K H32 backward)
  bwd_gqa      B1 H8 Hkv2 S32768 D128 sink+window      (1/4 of the 32K H32 Hkv8 backward)
  fwd_d64      B1 H16 S16384 D64 sink+window           (1/4 of the 32K H32 head-dim-64 forward)
  bwd_d64      B1 H8 S32768 D64 sink+window backward   (1/4 of the 32K H32 head-dim-64 backward)
  decode       B32 H32 D128, 4160 cached rows          (the sparse-layer decode itself)
  decode_full  B1 H32 D128, 131072 cached rows         (1/32 of the full-layer decode)
  decode_gqa   B32 H32 Hkv8 D128, 4160 cached rows     (the grouped-query decode itself)
  handoff      B8 S32768 Hkv32 D128 prompts            (1/4 of the hand-off of 32 prompts)
"""

import math
import sys

import torch

import attention_sink_long_b200 as lg
import synthetic_inputs as si

SW, FULL, BS = (64, 1, 64, 0), (64, 0, 2**31 - 1, 0), (64, 1, 16, 32)
CASES = ("fwd_dense", "fwd_sw", "fwd_bs", "fwd_pair", "fwd_d64", "bwd_sw", "bwd_gqa", "bwd_d64", "decode", "decode_full",
         "decode_gqa", "handoff")


def run(case: str) -> None:
    d = torch.device("cuda")
    D = 64 if case.endswith("_d64") else 128
    sc = 1 / math.sqrt(D)
    if case.startswith("fwd"):
        pat = {"fwd_dense": FULL, "fwd_sw": SW, "fwd_bs": BS, "fwd_pair": FULL, "fwd_d64": SW}[case]
        S, H = (131072, 8) if case == "fwd_bs" else (16384, 16)
        q, k, v = si.prefill_inputs_device(1, S, H, H, D, d)
        o = torch.empty_like(q)
        lse = torch.empty(1, H, S, device=d)
        fwd = lg.lg_sparse_attn_fwd_pair if case == "fwd_pair" else lg.lg_sparse_attn_fwd
        for _ in range(3):
            fwd(pat, q, k, v, o, lse, sc)
    elif case in ("bwd_sw", "bwd_gqa", "bwd_d64"):
        H, Hkv = (8, 2) if case == "bwd_gqa" else (8, 8)
        q, k, v, do = si.prefill_inputs_device(1, 32768, H, Hkv, D, d, with_dout=True)
        o = torch.empty_like(q)
        lse = torch.empty(1, H, 32768, device=d)
        lg.lg_sparse_attn_fwd(SW, q, k, v, o, lse, sc)
        g = [torch.empty_like(t) for t in (q, k, v)]
        w = torch.empty(lg.lg_sparse_attn_bwd_workspace(SW, 1, 32768, H, Hkv, D), dtype=torch.uint8, device=d)
        for _ in range(3):
            lg.lg_sparse_attn_bwd(SW, q, k, v, o, do, lse, *g, sc, w)
    elif case.startswith("decode"):
        B, Hkv, L = {"decode": (32, 32, 4160), "decode_full": (1, 32, 131072), "decode_gqa": (32, 8, 4160)}[case]
        q, kc, vc, cl = si.decode_inputs_device(B, 32, Hkv, 128, L, d)
        o = torch.empty_like(q)
        lse = torch.empty(B, 32, device=d)
        w = torch.empty(max(lg.lg_sparse_decode_workspace(B, 32, Hkv, 128, L), 1), dtype=torch.uint8, device=d)
        for _ in range(3):
            lg.lg_sparse_decode(q, kc, vc, cl, o, lse, sc, workspace=w)
    elif case == "handoff":
        k = si.device_normal((8, 32768, 32, 128), si.SEED_BASE + 1, d)
        v = si.device_normal((8, 32768, 32, 128), si.SEED_BASE + 2, d)
        rows = lg.lg_kv_compact_rows(SW, 32768)
        kc = torch.empty(8, rows + 64, 32, 128, dtype=torch.bfloat16, device=d)
        vc = torch.empty_like(kc)
        lens = torch.empty(8, dtype=torch.int32, device=d)
        for _ in range(3):
            lg.lg_kv_compact(SW, k, v, kc, vc, lens)
    else:
        raise SystemExit(f"unknown case {case!r}; cases: {', '.join(CASES)}")
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0, "a bounded device wait ran out"
    print("ok", case)


if __name__ == "__main__":
    run(sys.argv[1] if len(sys.argv) > 1 else "")
