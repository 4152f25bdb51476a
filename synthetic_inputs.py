"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no attention arithmetic: it only draws i.i.d. N(0, 1)
values from a CPU ``torch.Generator`` and rounds them to bf16 (round to
nearest even). Both sides read the same bf16 values; the oracle upcasts them
exactly to float64.

Seeds: 1000 + {Q: 0, K: 1, V: 2, dO: 3} for prefill, and the same offsets for
decode's q / k_cache / v_cache. The workloads stand in for the pages' Llama-2-7B
128K shapes (32 heads x 128 dims); no dataset or model weights are used.
"""

from __future__ import annotations

import torch

SEED_BASE = 1000


def _normal(shape, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)


def prefill_inputs(B: int, S: int, H: int, Hkv: int, D: int, seed: int = SEED_BASE,
                   with_dout: bool = False):
    """q [B,S,H,D], k/v [B,S,Hkv,D] (and dO [B,S,H,D]) as CPU bf16 tensors."""
    q = _normal((B, S, H, D), seed + 0)
    k = _normal((B, S, Hkv, D), seed + 1)
    v = _normal((B, S, Hkv, D), seed + 2)
    if with_dout:
        return q, k, v, _normal((B, S, H, D), seed + 3)
    return q, k, v


def decode_inputs(B: int, H: int, Hkv: int, D: int, Lmax: int, seed: int = SEED_BASE,
                  lens=None):
    """q [B,H,D], k_cache/v_cache [B,Lmax,Hkv,D] bf16 and cache_lens [B] int32.

    ``lens`` defaults to a full cache (Lmax rows for every sequence).
    """
    q = _normal((B, H, D), seed + 0)
    kc = _normal((B, Lmax, Hkv, D), seed + 1)
    vc = _normal((B, Lmax, Hkv, D), seed + 2)
    if lens is None:
        lens = [Lmax] * B
    cache_lens = torch.tensor(lens, dtype=torch.int32)
    return q, kc, vc, cache_lens


def ragged_lens(B: int, Lmax: int, seed: int = SEED_BASE + 7):
    """Seeded per-sequence cache lengths in [1, Lmax] (a length mix for edge cases)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randint(1, Lmax + 1, (B,), generator=g, dtype=torch.int64).tolist()
