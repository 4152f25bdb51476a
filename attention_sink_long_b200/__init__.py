"""Python binding of liblgattn.so -- the LongGen sparse-attention hot path on B200.

Argument marshalling only: every function below checks tensor dtypes, shapes
and devices, converts them to raw pointers and calls the C entry point of the
same name (include/lg_attn.h). All computation happens in the CUDA kernels of
the library; there is no fallback. Importing works without a GPU; any call
into the library raises if ``liblgattn.so`` has not been built.

Method: "A Little Goes a Long Way: Efficient Long Context Training and
Inference with Partial Contexts" (LongGen, arXiv 2410.01485) -- sparse layers
with attention-sink / window / strided-block static patterns, full-attention
middle layers, decode over the reduced KV cache.
"""

from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblgattn.so")
INT32_MAX = 2**31 - 1

__all__ = [
    "LgError", "Pattern", "lib", "lg_strerror", "lg_version",
    "lg_pattern_expand", "lg_pattern_expand_t", "lg_pattern_pairs", "lg_pattern_iterate_device",
    "lg_sparse_attn_fwd_workspace", "lg_sparse_attn_fwd", "lg_sparse_attn_fwd_varlen", "lg_sparse_attn_fwd_fp8qk",
    "lg_sparse_attn_fwd_pair", "lg_sparse_attn_bwd_workspace", "lg_sparse_attn_bwd", "lg_sparse_attn_bwd_varlen",
    "lg_sparse_decode_splits", "lg_sparse_decode_workspace", "lg_sparse_decode",
    "lg_sparse_decode_noalloc", "lg_kv_compact_rows", "lg_kv_compact", "lg_kv_compact_paged", "lg_kv_append_paged",
    "lg_sparse_decode_paged", "lg_exp2_device", "lg_wait_selftest", "lg_device_status", "EXPORTED_SYMBOLS",
]

EXPORTED_SYMBOLS = (
    "lg_strerror", "lg_version", "lg_pattern_expand", "lg_pattern_expand_t", "lg_pattern_pairs",
    "lg_pattern_iterate_device", "lg_sparse_attn_fwd_workspace", "lg_sparse_attn_fwd", "lg_sparse_attn_fwd_varlen",
    "lg_sparse_attn_fwd_fp8qk", "lg_sparse_attn_fwd_pair",
    "lg_sparse_attn_bwd_workspace", "lg_sparse_attn_bwd", "lg_sparse_attn_bwd_varlen", "lg_sparse_decode_splits",
    "lg_sparse_decode_workspace", "lg_sparse_decode", "lg_sparse_decode_noalloc", "lg_kv_compact_rows",
    "lg_kv_compact", "lg_kv_compact_paged", "lg_kv_append_paged", "lg_sparse_decode_paged", "lg_exp2_device",
    "lg_wait_selftest", "lg_device_status",
)


class Pattern(NamedTuple):
    """{block_size, sink_blocks, local_blocks, stride}; stride 0 = no strided term."""

    block_size: int
    sink_blocks: int
    local_blocks: int
    stride: int = 0

    @staticmethod
    def full(block_size: int = 64) -> "Pattern":
        return Pattern(block_size, 0, INT32_MAX, 0)


class _lg_pattern_t(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int32), ("sink_blocks", ctypes.c_int32),
                ("local_blocks", ctypes.c_int32), ("stride", ctypes.c_int32)]


class LgError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lg_strerror(status)} (status {status})")


_c_i32, _c_i64, _c_sz, _c_vp, _c_f = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
_P = ctypes.POINTER
_SIGS = {
    "lg_strerror": (ctypes.c_char_p, [_c_i32]),
    "lg_version": (_c_i32, []),
    "lg_pattern_expand": (_c_i32, [_P(_lg_pattern_t), _c_i32, _P(_c_i32), _P(_c_i32), _c_i64, _P(_c_i64)]),
    "lg_pattern_expand_t": (_c_i32, [_P(_lg_pattern_t), _c_i32, _P(_c_i32), _P(_c_i32), _c_i64, _P(_c_i64)]),
    "lg_pattern_pairs": (_c_i32, [_P(_lg_pattern_t), _c_i32, _P(_c_i64)]),
    "lg_pattern_iterate_device": (_c_i32, [_P(_lg_pattern_t), _c_i32, _c_i32, _c_i32, _c_vp, _c_i32, _c_vp]),
    "lg_sparse_attn_fwd_workspace": (_c_i32, [_P(_lg_pattern_t)] + [_c_i32] * 5 + [_P(_c_sz)]),
    "lg_sparse_attn_fwd": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_vp] + [_c_i32] * 5
                           + [_c_f, _c_vp, _c_sz, _c_vp]),
    "lg_sparse_attn_fwd_varlen": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_vp, _c_vp]
                                  + [_c_i32] * 6 + [_c_f, _c_vp]),
    "lg_sparse_attn_fwd_fp8qk": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp, _c_vp, _c_f, _c_f, _c_vp, _c_i32, _c_vp]
                                 + [_c_i32] * 5 + [_c_f, _c_vp]),
    "lg_sparse_attn_fwd_pair": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_vp] + [_c_i32] * 5
                                + [_c_f, _c_vp]),
    "lg_sparse_attn_bwd_workspace": (_c_i32, [_P(_lg_pattern_t)] + [_c_i32] * 5 + [_P(_c_sz)]),
    "lg_sparse_attn_bwd": (_c_i32, [_P(_lg_pattern_t)] + [_c_vp] * 4 + [_c_i32] + [_c_vp] * 5 + [_c_i32] * 6
                           + [_c_f, _c_vp, _c_sz, _c_vp]),
    "lg_sparse_attn_bwd_varlen": (_c_i32, [_P(_lg_pattern_t)] + [_c_vp] * 4 + [_c_i32] + [_c_vp] * 5 + [_c_i32]
                                  + [_c_vp] + [_c_i32] * 6 + [_c_f, _c_vp, _c_sz, _c_vp]),
    "lg_sparse_decode_splits": (_c_i32, [_c_i32] * 6 + [_P(_c_i32)]),
    "lg_sparse_decode_workspace": (_c_i32, [_c_i32] * 6 + [_P(_c_sz)]),
    "lg_sparse_decode": (_c_i32, [_c_vp] * 5 + [_c_i32, _c_vp] + [_c_i32] * 6 + [_c_f, _c_vp, _c_sz, _c_vp]),
    "lg_sparse_decode_noalloc": (_c_i32, [_c_vp] * 5 + [_c_i32, _c_vp] + [_c_i32] * 6 + [_c_f, _c_vp]),
    "lg_kv_compact_rows": (_c_i32, [_P(_lg_pattern_t), _c_i32, _P(_c_i32)]),
    "lg_kv_compact": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp] + [_c_i32] * 4 + [_c_vp, _c_vp, _c_i32, _c_vp, _c_vp]),
    "lg_kv_compact_paged": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp] + [_c_i32] * 4
                            + [_c_vp, _c_vp, _c_i64, _c_vp, _c_vp, _c_i32, _c_vp, _c_vp, _c_vp]),
    "lg_kv_append_paged": (_c_i32, [_P(_lg_pattern_t), _c_vp, _c_vp] + [_c_i32] * 3
                           + [_c_vp, _c_vp, _c_i64, _c_vp, _c_vp, _c_i32, _c_vp, _c_vp, _c_vp]),
    "lg_sparse_decode_paged": (_c_i32, [_c_vp, _c_vp, _c_vp, _c_i64, _c_vp, _c_i32, _c_vp, _c_vp, _c_i32, _c_vp]
                               + [_c_i32] * 5 + [_c_f, _c_vp, _c_sz, _c_vp]),
    "lg_exp2_device": (_c_i32, [_c_vp, _c_vp, _c_i64, _c_i32, _c_vp]),
    "lg_wait_selftest": (_c_i32, [_c_i64, _c_vp]),
    "lg_device_status": (_c_i32, [_c_i32, _P(ctypes.c_uint32)]),
}

_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m attention_sink_long_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise LgError(status, where)


def _pat(p) -> _lg_pattern_t:
    return _lg_pattern_t(int(p[0]), int(p[1]), int(p[2]), int(p[3]) if len(p) > 3 else 0)


def _stream(stream) -> int:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return int(getattr(stream, "cuda_stream", stream))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _expect(t, name, dtype, shape, device=None):
    import torch

    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    return torch


def lg_strerror(status: int) -> str:
    return lib().lg_strerror(int(status)).decode()


def lg_version() -> int:
    return int(lib().lg_version())


# ---------------------------------------------------------------- pattern
def lg_pattern_expand(pattern, seqlen: int):
    """CSR (row_ptr, col) as int32 numpy arrays."""
    import numpy as np

    p = _pat(pattern)
    nnz = _c_i64(0)
    _check(lib().lg_pattern_expand(ctypes.byref(p), seqlen, None, None, 0, ctypes.byref(nnz)), "lg_pattern_expand")
    nqb = seqlen // p.block_size
    row_ptr = np.zeros(nqb + 1, dtype=np.int32)
    col = np.zeros(max(nnz.value, 1), dtype=np.int32)
    _check(lib().lg_pattern_expand(ctypes.byref(p), seqlen, row_ptr.ctypes.data_as(_P(_c_i32)),
                                   col.ctypes.data_as(_P(_c_i32)), col.size, ctypes.byref(nnz)), "lg_pattern_expand")
    return row_ptr, col[: nnz.value]


def lg_pattern_expand_t(pattern, seqlen: int):
    """CSC (col_ptr, row) as int32 numpy arrays."""
    import numpy as np

    p = _pat(pattern)
    nnz = _c_i64(0)
    _check(lib().lg_pattern_expand_t(ctypes.byref(p), seqlen, None, None, 0, ctypes.byref(nnz)),
           "lg_pattern_expand_t")
    nqb = seqlen // p.block_size
    col_ptr = np.zeros(nqb + 1, dtype=np.int32)
    row = np.zeros(max(nnz.value, 1), dtype=np.int32)
    _check(lib().lg_pattern_expand_t(ctypes.byref(p), seqlen, col_ptr.ctypes.data_as(_P(_c_i32)),
                                     row.ctypes.data_as(_P(_c_i32)), row.size, ctypes.byref(nnz)),
           "lg_pattern_expand_t")
    return col_ptr, row[: nnz.value]


def lg_pattern_pairs(pattern, seqlen: int) -> int:
    p = _pat(pattern)
    out = _c_i64(0)
    _check(lib().lg_pattern_pairs(ctypes.byref(p), seqlen, ctypes.byref(out)), "lg_pattern_pairs")
    return out.value


def lg_pattern_iterate_device(pattern, seqlen: int, tile_blocks: int, mode: int, out, cap: int, stream=None):
    """Runs the kernels' block iterators on the device into ``out`` (int32 CUDA
    tensor); mode 0/1 forward/backward unions, 2 the forward's chunked walk,
    3 the backward's paired KV tiles (see include/lg_attn.h)."""
    p = _pat(pattern)
    _check(lib().lg_pattern_iterate_device(ctypes.byref(p), seqlen, tile_blocks, mode, out.data_ptr(), cap,
                                           _stream(stream)), "lg_pattern_iterate_device")


# ---------------------------------------------------------------- forward
def lg_sparse_attn_fwd_workspace(pattern, B, S, H, Hkv, D) -> int:
    p = _pat(pattern)
    n = _c_sz(0)
    _check(lib().lg_sparse_attn_fwd_workspace(ctypes.byref(p), B, S, H, Hkv, D, ctypes.byref(n)),
           "lg_sparse_attn_fwd_workspace")
    return n.value


def _dtype_code(t, name):
    import torch

    if t.dtype == torch.bfloat16:
        return 0
    if t.dtype == torch.float32:
        return 1
    raise TypeError(f"{name}: expected bfloat16 or float32, got {t.dtype}")


def lg_sparse_attn_fwd(pattern, q, k, v, o, lse, scale: float, workspace=None, stream=None):
    """q [B,S,H,D], k/v [B,S,Hkv,D] bf16 CUDA tensors; o [B,S,H,D] bf16 or fp32
    (written); lse [B,H,S] fp32 or None."""
    import torch

    B, S, H, D = q.shape
    Hkv = k.shape[2]
    _expect(q, "q", torch.bfloat16, (B, S, H, D))
    _expect(k, "k", torch.bfloat16, (B, S, Hkv, D), q.device)
    _expect(v, "v", torch.bfloat16, (B, S, Hkv, D), q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, S, H, D), q.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, H, S), q.device)
    p = _pat(pattern)
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lg_sparse_attn_fwd(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), odt,
                                    _ptr(lse), B, S, H, Hkv, D, float(scale), _ptr(workspace), ws, _stream(stream)),
           "lg_sparse_attn_fwd")


def lg_sparse_attn_fwd_pair(pattern, q, k, v, o, lse, scale: float, stream=None):
    """lg_sparse_attn_fwd computed by CTA pairs sharing 256-row MMAs (head dim 128):
    q [B,S,H,128], k/v [B,S,Hkv,128] bf16; o bf16 or fp32 (written); lse [B,H,S] fp32 or None."""
    import torch

    B, S, H, D = q.shape
    Hkv = k.shape[2]
    _expect(q, "q", torch.bfloat16, (B, S, H, D))
    _expect(k, "k", torch.bfloat16, (B, S, Hkv, D), q.device)
    _expect(v, "v", torch.bfloat16, (B, S, Hkv, D), q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, S, H, D), q.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, H, S), q.device)
    _check(lib().lg_sparse_attn_fwd_pair(ctypes.byref(_pat(pattern)), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         o.data_ptr(), odt, _ptr(lse), B, S, H, Hkv, D, float(scale),
                                         _stream(stream)), "lg_sparse_attn_fwd_pair")


def lg_sparse_attn_fwd_varlen(pattern, q, k, v, o, lse, cu_seqlens, max_seqlen: int, scale: float, stream=None):
    """Packed sequences: q [total,H,D], k/v [total,Hkv,D] bf16; o [total,H,D] bf16
    or fp32 (written); lse [H,total] fp32 or None; cu_seqlens [B+1] int32 on the
    device; max_seqlen the longest sequence (a multiple of 64)."""
    import torch

    total, H, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    _expect(q, "q", torch.bfloat16, (total, H, D))
    _expect(k, "k", torch.bfloat16, (total, Hkv, D), q.device)
    _expect(v, "v", torch.bfloat16, (total, Hkv, D), q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (total, H, D), q.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (H, total), q.device)
    _expect(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), q.device)
    _check(lib().lg_sparse_attn_fwd_varlen(ctypes.byref(_pat(pattern)), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           o.data_ptr(), odt, _ptr(lse), cu_seqlens.data_ptr(), B, total,
                                           int(max_seqlen), H, Hkv, D, float(scale), _stream(stream)),
           "lg_sparse_attn_fwd_varlen")


def lg_sparse_attn_fwd_fp8qk(pattern, q8, k8, v, q_descale: float, k_descale: float, o, lse, scale: float,
                             stream=None):
    """q8 [B,S,H,128], k8 [B,S,Hkv,128] torch.float8_e4m3fn; v bf16; o bf16 or fp32; lse [B,H,S] or None.
    S = q8 k8^T * q_descale * k_descale on the fp8 tensor-core path."""
    import torch

    B, S, H, D = q8.shape
    Hkv = k8.shape[2]
    _expect(q8, "q8", torch.float8_e4m3fn, (B, S, H, D))
    _expect(k8, "k8", torch.float8_e4m3fn, (B, S, Hkv, D), q8.device)
    _expect(v, "v", torch.bfloat16, (B, S, Hkv, D), q8.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, S, H, D), q8.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, H, S), q8.device)
    _check(lib().lg_sparse_attn_fwd_fp8qk(ctypes.byref(_pat(pattern)), q8.data_ptr(), k8.data_ptr(), v.data_ptr(),
                                          float(q_descale), float(k_descale), o.data_ptr(), odt, _ptr(lse), B, S, H,
                                          Hkv, D, float(scale), _stream(stream)), "lg_sparse_attn_fwd_fp8qk")


# ---------------------------------------------------------------- backward
def lg_sparse_attn_bwd_workspace(pattern, B, S, H, Hkv, D) -> int:
    p = _pat(pattern)
    n = _c_sz(0)
    _check(lib().lg_sparse_attn_bwd_workspace(ctypes.byref(p), B, S, H, Hkv, D, ctypes.byref(n)),
           "lg_sparse_attn_bwd_workspace")
    return n.value


def lg_sparse_attn_bwd(pattern, q, k, v, o, dout, lse, dq, dk, dv, scale: float, workspace, stream=None):
    """Gradients into dq/dk/dv (shaped like q/k/v; all bf16, or all fp32 for the
    unrounded accumulators). o is the forward output (bf16 or fp32); workspace
    is a CUDA uint8 tensor."""
    import torch

    B, S, H, D = q.shape
    Hkv = k.shape[2]
    for name, t, shp in (("q", q, (B, S, H, D)), ("dout", dout, (B, S, H, D)),
                         ("k", k, (B, S, Hkv, D)), ("v", v, (B, S, Hkv, D))):
        _expect(t, name, torch.bfloat16, shp, q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, S, H, D), q.device)
    gdt = _dtype_code(dq, "dq")
    for name, t, shp in (("dq", dq, (B, S, H, D)), ("dk", dk, (B, S, Hkv, D)), ("dv", dv, (B, S, Hkv, D))):
        _expect(t, name, dq.dtype, shp, q.device)
    _expect(lse, "lse", torch.float32, (B, H, S), q.device)
    p = _pat(pattern)
    ws = workspace.numel() * workspace.element_size()
    _check(lib().lg_sparse_attn_bwd(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), odt,
                                    dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), gdt,
                                    B, S, H, Hkv, D, float(scale), workspace.data_ptr(), ws, _stream(stream)),
           "lg_sparse_attn_bwd")


def lg_sparse_attn_bwd_varlen(pattern, q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens, max_seqlen: int, scale: float,
                              workspace, stream=None):
    """Packed sequences (see lg_sparse_attn_fwd_varlen): q, dout, dq [total,H,D];
    k, v, dk, dv [total,Hkv,D]; o [total,H,D] bf16 or fp32; lse [H,total];
    workspace of lg_sparse_attn_bwd_workspace(pattern, 1, total, H, Hkv, D) bytes."""
    import torch

    total, H, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    for name, t, shp in (("q", q, (total, H, D)), ("dout", dout, (total, H, D)),
                         ("k", k, (total, Hkv, D)), ("v", v, (total, Hkv, D))):
        _expect(t, name, torch.bfloat16, shp, q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (total, H, D), q.device)
    gdt = _dtype_code(dq, "dq")
    for name, t, shp in (("dq", dq, (total, H, D)), ("dk", dk, (total, Hkv, D)), ("dv", dv, (total, Hkv, D))):
        _expect(t, name, dq.dtype, shp, q.device)
    _expect(lse, "lse", torch.float32, (H, total), q.device)
    _expect(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), q.device)
    ws = workspace.numel() * workspace.element_size()
    _check(lib().lg_sparse_attn_bwd_varlen(ctypes.byref(_pat(pattern)), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           o.data_ptr(), odt, dout.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                                           dk.data_ptr(), dv.data_ptr(), gdt, cu_seqlens.data_ptr(), B, total,
                                           int(max_seqlen), H, Hkv, D, float(scale), workspace.data_ptr(), ws,
                                           _stream(stream)), "lg_sparse_attn_bwd_varlen")


# ---------------------------------------------------------------- decode
def lg_sparse_decode_splits(B, H, Hkv, D, Lmax, num_splits=0) -> int:
    n = _c_i32(0)
    _check(lib().lg_sparse_decode_splits(B, H, Hkv, D, Lmax, num_splits, ctypes.byref(n)), "lg_sparse_decode_splits")
    return n.value


def lg_sparse_decode_workspace(B, H, Hkv, D, Lmax, num_splits=0) -> int:
    n = _c_sz(0)
    _check(lib().lg_sparse_decode_workspace(B, H, Hkv, D, Lmax, num_splits, ctypes.byref(n)),
           "lg_sparse_decode_workspace")
    return n.value


def lg_sparse_decode(q, k_cache, v_cache, cache_lens, o, lse, scale: float, num_splits: int = 0, workspace=None,
                     stream=None):
    """q [B,H,D] bf16, caches [B,Lmax,Hkv,D] bf16, cache_lens [B] int32, o [B,H,D] bf16 or fp32 (the
    unrounded result), lse [B,H] fp32 or None."""
    import torch

    B, H, D = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    _expect(q, "q", torch.bfloat16, (B, H, D))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, Lmax, Hkv, D), q.device)
    _expect(v_cache, "v_cache", torch.bfloat16, (B, Lmax, Hkv, D), q.device)
    _expect(cache_lens, "cache_lens", torch.int32, (B,), q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, H, D), q.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, H), q.device)
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lg_sparse_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cache_lens.data_ptr(),
                                  o.data_ptr(), odt, _ptr(lse), B, H, Hkv, D, Lmax, int(num_splits), float(scale),
                                  _ptr(workspace), ws, _stream(stream)), "lg_sparse_decode")


def lg_kv_compact_rows(pattern, S) -> int:
    """Rows of the reduced cache lg_kv_compact writes for a prompt of S tokens."""
    n = _c_i32(0)
    _check(lib().lg_kv_compact_rows(ctypes.byref(_pat(pattern)), int(S), ctypes.byref(n)), "lg_kv_compact_rows")
    return n.value


def lg_kv_compact(pattern, k, v, k_cache, v_cache, cache_lens, stream=None):
    """k, v [B,S,Hkv,D] bf16 (prompt); k_cache, v_cache [B,Lmax,Hkv,D] bf16 and
    cache_lens [B] int32 (written): the reduced cache for decoding token S."""
    import torch

    B, S, Hkv, D = k.shape
    Lmax = k_cache.shape[1]
    _expect(k, "k", torch.bfloat16, (B, S, Hkv, D))
    _expect(v, "v", torch.bfloat16, (B, S, Hkv, D), k.device)
    _expect(k_cache, "k_cache", torch.bfloat16, (B, Lmax, Hkv, D), k.device)
    _expect(v_cache, "v_cache", torch.bfloat16, (B, Lmax, Hkv, D), k.device)
    _expect(cache_lens, "cache_lens", torch.int32, (B,), k.device)
    _check(lib().lg_kv_compact(ctypes.byref(_pat(pattern)), k.data_ptr(), v.data_ptr(), B, S, Hkv, D,
                               k_cache.data_ptr(), v_cache.data_ptr(), Lmax, cache_lens.data_ptr(), _stream(stream)),
           "lg_kv_compact")


def _expect_paged(k_pool, v_pool, block_table, block_ids, cache_lens, positions, Hkv=None, D=None):
    import torch

    P = k_pool.shape[0]
    Hkv = k_pool.shape[2] if Hkv is None else Hkv
    D = k_pool.shape[3] if D is None else D
    B, MB = block_table.shape
    dev = k_pool.device
    _expect(k_pool, "k_pool", torch.bfloat16, (P, 64, Hkv, D), dev)
    _expect(v_pool, "v_pool", torch.bfloat16, (P, 64, Hkv, D), dev)
    _expect(block_table, "block_table", torch.int32, (B, MB), dev)
    if block_ids is not None:
        _expect(block_ids, "block_ids", torch.int32, (B, MB), dev)
    _expect(cache_lens, "cache_lens", torch.int32, (B,), dev)
    if positions is not None:
        _expect(positions, "positions", torch.int32, (B,), dev)
    return P, B, MB, Hkv, D


def lg_kv_compact_paged(pattern, k, v, k_pool, v_pool, block_table, block_ids, cache_lens, positions, stream=None):
    """The reduced cache of each prompt (k, v [B,S,Hkv,D] bf16) into pages:
    k_pool, v_pool [P,64,Hkv,D] bf16; block_table, block_ids [B,max_blocks],
    cache_lens, positions [B] int32 (see include/lg_attn.h)."""
    import torch

    B, S, Hkv, D = k.shape
    _expect(k, "k", torch.bfloat16, (B, S, Hkv, D))
    _expect(v, "v", torch.bfloat16, (B, S, Hkv, D), k.device)
    P, Bt, MB, _, _ = _expect_paged(k_pool, v_pool, block_table, block_ids, cache_lens, positions, Hkv, D)
    if Bt != B:
        raise ValueError(f"block_table has {Bt} rows, expected {B}")
    _check(lib().lg_kv_compact_paged(ctypes.byref(_pat(pattern)), k.data_ptr(), v.data_ptr(), B, S, Hkv, D,
                                     k_pool.data_ptr(), v_pool.data_ptr(), P, block_table.data_ptr(),
                                     block_ids.data_ptr(), MB, cache_lens.data_ptr(), positions.data_ptr(),
                                     _stream(stream)), "lg_kv_compact_paged")


def lg_kv_append_paged(pattern, k_new, v_new, k_pool, v_pool, block_table, block_ids, cache_lens, positions,
                       stream=None):
    """Append one token per sequence (k_new, v_new [B,Hkv,D] bf16) to a paged cache."""
    import torch

    B, Hkv, D = k_new.shape
    _expect(k_new, "k_new", torch.bfloat16, (B, Hkv, D))
    _expect(v_new, "v_new", torch.bfloat16, (B, Hkv, D), k_new.device)
    P, Bt, MB, _, _ = _expect_paged(k_pool, v_pool, block_table, block_ids, cache_lens, positions, Hkv, D)
    if Bt != B:
        raise ValueError(f"block_table has {Bt} rows, expected {B}")
    _check(lib().lg_kv_append_paged(ctypes.byref(_pat(pattern)), k_new.data_ptr(), v_new.data_ptr(), B, Hkv, D,
                                    k_pool.data_ptr(), v_pool.data_ptr(), P, block_table.data_ptr(),
                                    block_ids.data_ptr(), MB, cache_lens.data_ptr(), positions.data_ptr(),
                                    _stream(stream)), "lg_kv_append_paged")


def lg_sparse_decode_paged(q, k_pool, v_pool, block_table, cache_lens, o, lse, scale: float, num_splits: int = 0,
                           workspace=None, stream=None):
    """lg_sparse_decode over a paged cache; workspace as lg_sparse_decode_workspace(..., Lmax=64*max_blocks)."""
    import torch

    B, H, D = q.shape
    _expect(q, "q", torch.bfloat16, (B, H, D))
    P, Bt, MB, Hkv, _ = _expect_paged(k_pool, v_pool, block_table, None, cache_lens, None, None, D)
    if Bt != B:
        raise ValueError(f"block_table has {Bt} rows, expected {B}")
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, H, D), q.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, H), q.device)
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lg_sparse_decode_paged(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), P,
                                        block_table.data_ptr(), MB, cache_lens.data_ptr(), o.data_ptr(), odt,
                                        _ptr(lse),
                                        B, H, Hkv, D, int(num_splits), float(scale), _ptr(workspace), ws,
                                        _stream(stream)), "lg_sparse_decode_paged")


def lg_sparse_decode_noalloc(q, k_cache, v_cache, cache_lens, o, lse, scale: float, num_splits: int = 0,
                             stream=None):
    """lg_sparse_decode for callers that cannot allocate device memory: no
    workspace argument; the library's fixed 16 MiB device scratch array holds
    the split partials. Calls that overlap on the GPU share that array and race,
    so serialise them. The first call on a device resolves the array's address;
    make it before any stream capture. The tensors must live on the current
    device: that device's array is the one the call uses."""
    import torch

    B, H, D = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    if q.device.type != "cuda" or q.device.index != torch.cuda.current_device():
        raise ValueError(f"q: expected the current device cuda:{torch.cuda.current_device()}, got {q.device}")
    _expect(q, "q", torch.bfloat16, (B, H, D))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, Lmax, Hkv, D), q.device)
    _expect(v_cache, "v_cache", torch.bfloat16, (B, Lmax, Hkv, D), q.device)
    _expect(cache_lens, "cache_lens", torch.int32, (B,), q.device)
    odt = _dtype_code(o, "o")
    _expect(o, "o", o.dtype, (B, H, D), q.device)
    if lse is not None:
        _expect(lse, "lse", torch.float32, (B, H), q.device)
    _check(lib().lg_sparse_decode_noalloc(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                          cache_lens.data_ptr(), o.data_ptr(), odt, _ptr(lse), B, H, Hkv, D, Lmax,
                                          int(num_splits), float(scale), _stream(stream)),
           "lg_sparse_decode_noalloc")


# ---------------------------------------------------------------- numerics
def lg_exp2_device(x, y, method: int, stream=None):
    """y = 2^x on the device with the softmax's exponential (method 0: ex2.approx)."""
    import torch

    _expect(x, "x", torch.float32, tuple(x.shape))
    _expect(y, "y", torch.float32, tuple(x.shape), x.device)
    _check(lib().lg_exp2_device(x.data_ptr(), y.data_ptr(), x.numel(), int(method), _stream(stream)),
           "lg_exp2_device")


# ---------------------------------------------------------------- diagnostics
def lg_wait_selftest(limit_cycles: int, stream=None):
    """Run the bounded-wait failure path once (sets device error bit 5)."""
    _check(lib().lg_wait_selftest(int(limit_cycles), _stream(stream)), "lg_wait_selftest")

def lg_device_status(device: int = 0) -> int:
    """Reads and clears the device error flags (synchronises the device)."""
    f = ctypes.c_uint32(0)
    _check(lib().lg_device_status(int(device), ctypes.byref(f)), "lg_device_status")
    return f.value
