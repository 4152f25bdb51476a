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


def device_normal(shape, seed: int, device, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, 1) drawn by torch's generator on ``device`` (used for inputs too large
    to draw on the host, e.g. the 128K prefill and the 131072-row decode caches;
    the oracle reads the sampled slices it needs back from the device)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(*shape, dtype=dtype, device=device)
    chunk = 1 << 28  # elements per draw: bounds the fp32 temporary to 1 GiB
    flat = out.view(-1)
    for i, s in enumerate(range(0, flat.numel(), chunk)):
        n = min(chunk, flat.numel() - s)
        flat[s:s + n] = torch.randn(n, generator=g, device=device, dtype=torch.float32).to(dtype)
    return out


def prefill_inputs_device(B: int, S: int, H: int, Hkv: int, D: int, device, seed: int = SEED_BASE,
                          with_dout: bool = False):
    q = device_normal((B, S, H, D), seed + 0, device)
    k = device_normal((B, S, Hkv, D), seed + 1, device)
    v = device_normal((B, S, Hkv, D), seed + 2, device)
    if with_dout:
        return q, k, v, device_normal((B, S, H, D), seed + 3, device)
    return q, k, v


def decode_inputs_device(B: int, H: int, Hkv: int, D: int, Lmax: int, device, seed: int = SEED_BASE, lens=None):
    q = device_normal((B, H, D), seed + 0, device)
    kc = device_normal((B, Lmax, Hkv, D), seed + 1, device)
    vc = device_normal((B, Lmax, Hkv, D), seed + 2, device)
    if lens is None:
        lens = [Lmax] * B
    return q, kc, vc, torch.tensor(lens, dtype=torch.int32, device=device)
