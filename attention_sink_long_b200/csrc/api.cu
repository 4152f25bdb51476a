// api.cu -- the extern "C" boundary (include/lg_attn.h): argument validation,
// workspace sizing, TMA tensor-map construction and kernel launches.
// Nothing here allocates or frees device memory or synchronises a stream,
// except lg_device_status, which says so.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "lg_kernels.h"
#include "lg_pattern.cuh"

// Device error word written by bounded waits that ran out (see lg_device_status).
__device__ unsigned int g_lg_error_word;

namespace {

using lg::imax;
using lg::imin;

constexpr int kMaxDevices = 64;

lg_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? LG_OK : LG_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lg_status_t check_pattern(const lg_pattern_t* p) {
  if (p == nullptr) return LG_ERR_INVALID_ARG;
  if (p->block_size <= 0 || p->sink_blocks < 0 || p->local_blocks < 1 || p->stride < 0) return LG_ERR_INVALID_ARG;
  return LG_OK;
}

lg_status_t check_prefill_shape(const lg_pattern_t* p, int B, int S, int H, int Hkv, int D) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (B <= 0 || S <= 0 || H <= 0 || Hkv <= 0 || D <= 0) return LG_ERR_INVALID_ARG;
  if (H % Hkv != 0) return LG_ERR_INVALID_ARG;
  if (p->block_size != 64) return LG_ERR_UNSUPPORTED;
  if (S % 64 != 0) return LG_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return LG_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || (long long)((S + 127) / 128) * H > 2147483647LL) return LG_ERR_UNSUPPORTED;
  return LG_OK;
}

// Device error word address, resolved once per device with that device current.
unsigned int* error_word(lg_status_t* st) {
  static std::mutex mu;
  static unsigned int* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = LG_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lg_error_word) != cudaSuccess) {
      *st = LG_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = static_cast<unsigned int*>(p);
  }
  *st = LG_OK;
  return addr[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 4-D bf16 tensor map over a contiguous [B, S, Hx, D] tensor: dims {D, Hx, S, B};
// box {64, 1, rows, 1} with 128-byte swizzle, i.e. one [rows x 64] panel.
lg_status_t make_map(CUtensorMap* m, const void* base, int B, int S, int Hx, int D, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return LG_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hx, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hx * D * 2, (cuuint64_t)S * Hx * D * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LG_OK : LG_ERR_CUDA;
}

// The same over a byte tensor (fp8 e4m3 Q or K, head dim 128): box {128, 1, rows, 1},
// one 128-byte panel per row.
lg_status_t make_map_u8(CUtensorMap* m, const void* base, int B, int S, int Hx, int D, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return LG_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hx, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D, (cuuint64_t)Hx * D, (cuuint64_t)S * Hx * D};
  const cuuint32_t box[4] = {128, 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LG_OK : LG_ERR_CUDA;
}

// Decode split rule: about 256 KB of K+V per CTA, more splits when there are
// too few (b, kv head) rows to fill the GPU.
void decode_split_rule(int B, int H, int Hkv, int D, int Lmax, int requested, int* ns_out, int* rps_out) {
  int rps, ns;
  if (requested > 0) {
    ns = imin(requested, Lmax);
    rps = (Lmax + ns - 1) / ns;
  } else if (H / Hkv >= 2) {
    // Query-head groups (the staged tensor-core kernel, three CTAs per SM).
    // Many (b, kv head) pairs: about 1024 cache rows per CTA -- shorter
    // pieces lose more to each CTA's pipeline ramp and merge than they gain
    // in balance (B32 x 4160 rows, 8 KV heads: 5.9 TB/s with 5 pieces
    // against 5.65 with 9; 64K rows: 6.7 against 6.5). At most 128 pairs:
    // about 256 CTAs in one wave, which measured best from 16 to 128 pairs
    // (e.g. 32 pairs: 3.5 TB/s with 8 pieces against 2.9-3.0 with 5; 128
    // pairs: 5.4-5.7 with 2 against 4.5-5.0 with 5).
    const long long pairs = (long long)B * Hkv;
    if (pairs <= 128) {
      ns = (int)((256 + pairs / 2) / pairs);
      ns = imax(1, imin(ns, (Lmax + 63) / 64));
    } else {
      ns = (Lmax + 1023) / 1024;
    }
    rps = (Lmax + ns - 1) / ns;
  } else {
    rps = (D == 128) ? 512 : 1024;
    ns = (Lmax + rps - 1) / rps;
    while (rps > 64 && (long long)B * Hkv * ns < 148LL * 8) {
      rps /= 2;
      ns = (Lmax + rps - 1) / rps;
    }
  }
  if (ns < 1) ns = 1;
  rps = (Lmax + ns - 1) / ns;
  ns = (Lmax + rps - 1) / rps;
  *ns_out = ns;
  *rps_out = rps;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

const char* lg_strerror(lg_status_t s) {
  switch (s) {
    case LG_OK: return "ok";
    case LG_ERR_INVALID_ARG: return "invalid argument";
    case LG_ERR_UNSUPPORTED: return "unsupported shape, pattern or alignment";
    case LG_ERR_WORKSPACE: return "workspace missing or too small";
    case LG_ERR_CUDA: return "CUDA error";
    case LG_ERR_INTERNAL: return "internal error";
    case LG_ERR_CAPACITY: return "output capacity too small";
  }
  return "unknown status";
}

int32_t lg_version(void) { return (2 << 16) | 1; }

// ---------------------------------------------------------------- pattern (host)
lg_status_t lg_pattern_expand(const lg_pattern_t* p, int32_t seqlen, int32_t* row_ptr, int32_t* col, int64_t cap,
                              int64_t* nnz) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (nnz == nullptr || seqlen <= 0 || seqlen % p->block_size != 0) return LG_ERR_INVALID_ARG;
  const int nqb = seqlen / p->block_size;
  int64_t total = 0;
  for (int i = 0; i < nqb; ++i) total += lg::KvIter(*p, i, i).count();
  *nnz = total;
  if (col == nullptr) return LG_OK;
  if (row_ptr == nullptr) return LG_ERR_INVALID_ARG;
  if (cap < total) return LG_ERR_CAPACITY;
  int64_t e = 0;
  for (int i = 0; i < nqb; ++i) {
    row_ptr[i] = (int32_t)e;
    const lg::KvIter it(*p, i, i);
    for (int j = it.first(); j >= 0; j = it.next(j)) col[e++] = j;
  }
  row_ptr[nqb] = (int32_t)e;
  return e == total ? LG_OK : LG_ERR_INTERNAL;
}

lg_status_t lg_pattern_expand_t(const lg_pattern_t* p, int32_t seqlen, int32_t* col_ptr, int32_t* row, int64_t cap,
                                int64_t* nnz) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (nnz == nullptr || seqlen <= 0 || seqlen % p->block_size != 0) return LG_ERR_INVALID_ARG;
  const int nqb = seqlen / p->block_size;
  int64_t total = 0;
  for (int j = 0; j < nqb; ++j) total += lg::QIter(*p, j, j, nqb).count();
  *nnz = total;
  if (row == nullptr) return LG_OK;
  if (col_ptr == nullptr) return LG_ERR_INVALID_ARG;
  if (cap < total) return LG_ERR_CAPACITY;
  int64_t e = 0;
  for (int j = 0; j < nqb; ++j) {
    col_ptr[j] = (int32_t)e;
    const lg::QIter it(*p, j, j, nqb);
    for (int i = it.first_blk; i <= it.last_blk; ++i) row[e++] = i;
  }
  col_ptr[nqb] = (int32_t)e;
  return e == total ? LG_OK : LG_ERR_INTERNAL;
}

lg_status_t lg_pattern_pairs(const lg_pattern_t* p, int32_t seqlen, int64_t* pairs) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (pairs == nullptr || seqlen <= 0 || seqlen % p->block_size != 0) return LG_ERR_INVALID_ARG;
  const int64_t b = p->block_size;
  const int nqb = seqlen / p->block_size;
  int64_t total = 0;
  // Every listed block below the diagonal is fully visible; the diagonal is causal.
  for (int i = 0; i < nqb; ++i) total += (int64_t)(lg::KvIter(*p, i, i).count() - 1) * b * b + b * (b + 1) / 2;
  *pairs = total;
  return LG_OK;
}

lg_status_t lg_pattern_iterate_device(const lg_pattern_t* p, int32_t seqlen, int32_t tile_blocks, int32_t mode,
                                      int32_t* out, int32_t cap, lg_stream_t stream) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (out == nullptr || seqlen <= 0 || seqlen % p->block_size != 0 || cap < 0) return LG_ERR_INVALID_ARG;
  if (mode < 0 || mode > 3) return LG_ERR_INVALID_ARG;
  if (p->block_size != 64) return LG_ERR_UNSUPPORTED;
  const bool ok_tiles = (mode == 0 && (tile_blocks == 1 || tile_blocks == 2 || tile_blocks == 4 || tile_blocks == 8)) ||
                        (mode == 1 && (tile_blocks == 1 || tile_blocks == 2)) ||
                        (mode == 2 && (tile_blocks == 4 || tile_blocks == 8)) || (mode == 3 && tile_blocks == 2);
  if (!ok_tiles) return LG_ERR_UNSUPPORTED;
  if (seqlen / 64 >= (1 << 23)) return LG_ERR_UNSUPPORTED;  // block << 8 must fit an int32
  return cuda_status(
      lg::launch_pattern_iterate(*p, seqlen, tile_blocks, mode, out, cap, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- forward
lg_status_t lg_sparse_attn_fwd_workspace(const lg_pattern_t* p, int32_t B, int32_t S, int32_t H, int32_t Hkv,
                                         int32_t D, size_t* bytes) {
  lg_status_t st = check_prefill_shape(p, B, S, H, Hkv, D);
  if (st != LG_OK) return st;
  if (bytes == nullptr) return LG_ERR_INVALID_ARG;
  *bytes = 0;
  return LG_OK;
}

lg_status_t lg_sparse_attn_fwd(const lg_pattern_t* p, const void* q, const void* k, const void* v, void* o,
                               int32_t o_dtype, float* lse, int32_t B, int32_t S, int32_t H, int32_t Hkv, int32_t D,
                               float scale, void* workspace, size_t workspace_bytes, lg_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  lg_status_t st = check_prefill_shape(p, B, S, H, Hkv, D);
  if (st != LG_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return LG_ERR_INVALID_ARG;
  if (o_dtype != LG_BF16 && o_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return LG_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return LG_ERR_UNSUPPORTED;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  CUtensorMap tq, tk, tv, to;
  if ((st = make_map(&tq, q, B, S, H, D, 128)) != LG_OK) return st;
  if ((st = make_map(&tk, k, B, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tv, v, B, S, Hkv, D, 64)) != LG_OK) return st;
  // With an fp32 O the kernel stores rows directly; the bf16 map is then built
  // over q only to have a valid (unused) descriptor.
  if ((st = make_map(&to, o_dtype == LG_F32 ? q : o, B, S, H, D, 64)) != LG_OK) return st;
  lg::FwdParams prm;
  prm.pat = *p;
  prm.lse = lse;
  prm.o_f32 = o_dtype == LG_F32 ? static_cast<float*>(o) : nullptr;
  prm.S = S;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.nqb = S / 64;
  prm.nqt = (S + 255) / 256;  // 256-row query spans (two 128-row tiles per CTA)
  prm.cu_seqlens = nullptr;
  prm.max_len = S;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = err;
  return cuda_status(lg::launch_fwd(D, tq, tk, tv, to, prm, B, static_cast<cudaStream_t>(stream)));
}

lg_status_t lg_sparse_attn_fwd_pair(const lg_pattern_t* p, const void* q, const void* k, const void* v, void* o,
                                    int32_t o_dtype, float* lse, int32_t B, int32_t S, int32_t H, int32_t Hkv,
                                    int32_t D, float scale, lg_stream_t stream) {
  lg_status_t st = check_prefill_shape(p, B, S, H, Hkv, D);
  if (st != LG_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return LG_ERR_INVALID_ARG;
  if (o_dtype != LG_BF16 && o_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return LG_ERR_INVALID_ARG;
  if (D != 128) return LG_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return LG_ERR_UNSUPPORTED;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  CUtensorMap tq, tk, tv, to;
  if ((st = make_map(&tq, q, B, S, H, D, 128)) != LG_OK) return st;
  if ((st = make_map(&tk, k, B, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tv, v, B, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&to, o_dtype == LG_F32 ? q : o, B, S, H, D, 64)) != LG_OK) return st;
  lg::FwdParams prm;
  prm.pat = *p;
  prm.lse = lse;
  prm.o_f32 = o_dtype == LG_F32 ? static_cast<float*>(o) : nullptr;
  prm.S = S;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.nqb = S / 64;
  prm.nqt = (S + 511) / 512;  // 512-row spans, one per CTA pair
  prm.cu_seqlens = nullptr;
  prm.max_len = S;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = err;
  return cuda_status(lg::launch_fwd2(tq, tk, tv, to, prm, B, static_cast<cudaStream_t>(stream)));
}

lg_status_t lg_sparse_attn_fwd_fp8qk(const lg_pattern_t* p, const void* q8, const void* k8, const void* v,
                                     float q_descale, float k_descale, void* o, int32_t o_dtype, float* lse, int32_t B,
                                     int32_t S, int32_t H, int32_t Hkv, int32_t D, float scale, lg_stream_t stream) {
  lg_status_t st = check_prefill_shape(p, B, S, H, Hkv, D);
  if (st != LG_OK) return st;
  if (q8 == nullptr || k8 == nullptr || v == nullptr || o == nullptr) return LG_ERR_INVALID_ARG;
  if (o_dtype != LG_BF16 && o_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  const float sc = scale * q_descale * k_descale;
  if (!(scale > 0.f) || !(q_descale > 0.f) || !(k_descale > 0.f) || !isfinite(sc) || !(sc > 0.f))
    return LG_ERR_INVALID_ARG;
  if (D != 128) return LG_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return LG_ERR_UNSUPPORTED;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  CUtensorMap tq, tk, tv, to;
  if ((st = make_map_u8(&tq, q8, B, S, H, D, 128)) != LG_OK) return st;
  if ((st = make_map_u8(&tk, k8, B, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tv, v, B, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&to, o_dtype == LG_F32 ? v : o, B, S, H, D, 64)) != LG_OK) return st;
  lg::FwdParams prm;
  prm.pat = *p;
  prm.lse = lse;
  prm.o_f32 = o_dtype == LG_F32 ? static_cast<float*>(o) : nullptr;
  prm.S = S;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.nqb = S / 64;
  prm.nqt = (S + 255) / 256;
  prm.cu_seqlens = nullptr;
  prm.max_len = S;
  prm.scale_log2 = sc * 1.4426950408889634f;  // the dequantisation scales fold into the softmax scale
  prm.err = err;
  return cuda_status(lg::launch_fwd_fp8qk(tq, tk, tv, to, prm, B, static_cast<cudaStream_t>(stream)));
}

lg_status_t lg_sparse_attn_fwd_varlen(const lg_pattern_t* p, const void* q, const void* k, const void* v, void* o,
                                      int32_t o_dtype, float* lse, const int32_t* cu_seqlens, int32_t B,
                                      int32_t total, int32_t max_seqlen, int32_t H, int32_t Hkv, int32_t D,
                                      float scale, lg_stream_t stream) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || cu_seqlens == nullptr)
    return LG_ERR_INVALID_ARG;
  if (B <= 0 || total <= 0 || max_seqlen <= 0 || H <= 0 || Hkv <= 0 || D <= 0 || H % Hkv != 0)
    return LG_ERR_INVALID_ARG;
  if (o_dtype != LG_BF16 && o_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return LG_ERR_INVALID_ARG;
  if (p->block_size != 64 || max_seqlen % 64 != 0 || (D != 64 && D != 128)) return LG_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || max_seqlen > total) return LG_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
    return LG_ERR_UNSUPPORTED;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  // Packed tensors are one batch of `total` rows to the tensor maps.
  CUtensorMap tq, tk, tv, to;
  if ((st = make_map(&tq, q, 1, total, H, D, 128)) != LG_OK) return st;
  if ((st = make_map(&tk, k, 1, total, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tv, v, 1, total, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&to, o_dtype == LG_F32 ? q : o, 1, total, H, D, 64)) != LG_OK) return st;
  lg::FwdParams prm;
  prm.pat = *p;
  prm.lse = lse;
  prm.o_f32 = o_dtype == LG_F32 ? static_cast<float*>(o) : nullptr;
  prm.S = total;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.nqb = total / 64;
  prm.nqt = (max_seqlen + 255) / 256;
  prm.cu_seqlens = cu_seqlens;
  prm.max_len = max_seqlen;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = err;
  return cuda_status(lg::launch_fwd(D, tq, tk, tv, to, prm, B, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- backward
namespace {

// Heavy KV tiles of the backward (query-list length above twice the median,
// e.g. the sink tile, seen by every query; at most 128), and, when a head has
// exactly one, how its walk splits into chunks about as long as a median tile.
struct HeavyPlan {
  int n_heavy = 0;
  int heavy[128];
  int n_chunks = 0;     // 0: not split
  int chunk_steps = 0;  // 128-row query steps per chunk
};

HeavyPlan heavy_plan(const lg_pattern_t& p, int nqb, int nkt) {
  HeavyPlan hp;
  std::vector<int> counts(nkt);
  const lg::BlockPairing bp(p, nqb);
  for (int t = 0; t < nkt; ++t) {
    int x, y;
    bp.pair(t, &x, &y);
    const int first = y >= 0 ? imin(x, y) : x;
    const int last = y >= 0 ? imax(bp.reach(x), bp.reach(y)) : bp.reach(x);
    counts[t] = last - first + 1;
  }
  std::vector<int> sorted_counts(counts);
  std::nth_element(sorted_counts.begin(), sorted_counts.begin() + nkt / 2, sorted_counts.end());
  const int median = sorted_counts[nkt / 2];
  for (int t = 0; t < nkt && hp.n_heavy < 128; ++t)
    if (counts[t] > 2 * median) hp.heavy[hp.n_heavy++] = t;
  if (hp.n_heavy == 1) {
    const int steps = (counts[hp.heavy[0]] + 1) / 2;
    const int ch = imax((median + 1) / 2, 16);
    if (steps > ch) {
      hp.chunk_steps = ch;
      hp.n_chunks = (steps + ch - 1) / ch;
    }
  }
  return hp;
}

// Bytes of the split heavy tile's partials and tickets for a (B, S) call.
size_t heavy_part_bytes(const lg_pattern_t& p, int B, int S, int Hkv, int D) {
  const HeavyPlan hp = heavy_plan(p, S / 64, (S + 127) / 128);
  if (hp.n_chunks == 0) return 0;
  return round256((size_t)B * Hkv * hp.n_chunks * 2 * 128 * D * sizeof(float)) +
         round256((size_t)B * Hkv * sizeof(unsigned int));
}

}  // namespace

lg_status_t lg_sparse_attn_bwd_workspace(const lg_pattern_t* p, int32_t B, int32_t S, int32_t H, int32_t Hkv,
                                         int32_t D, size_t* bytes) {
  lg_status_t st = check_prefill_shape(p, B, S, H, Hkv, D);
  if (st != LG_OK) return st;
  if (bytes == nullptr) return LG_ERR_INVALID_ARG;
  *bytes = round256((size_t)B * H * S * D * sizeof(float)) + 2 * round256((size_t)B * H * S * sizeof(float)) +
           heavy_part_bytes(*p, B, S, Hkv, D);
  return LG_OK;
}

// The backward of one (B, S) batch, or of B packed sequences (cu_seqlens given:
// S = total rows, every tensor one batch of S rows, max_len the longest sequence).
static lg_status_t bwd_common(const lg_pattern_t* p, const void* q, const void* k, const void* v, const void* o,
                              int32_t o_dtype, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int32_t grad_dtype, const int32_t* cu_seqlens, int32_t B, int32_t S, int32_t max_len,
                              int32_t H, int32_t Hkv, int32_t D, float scale, void* workspace, size_t workspace_bytes,
                              lg_stream_t stream) {
  const bool varlen = cu_seqlens != nullptr;
  const int Bm = varlen ? 1 : B;  // batches of the tensors
  lg_status_t st = LG_OK;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return LG_ERR_INVALID_ARG;
  if (grad_dtype != LG_BF16 && grad_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  if (o_dtype != LG_BF16 && o_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  const int grad_f32 = grad_dtype == LG_F32;
  if (!(scale > 0.f) || !isfinite(scale)) return LG_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return LG_ERR_UNSUPPORTED;
  size_t need = 0;
  lg_sparse_attn_bwd_workspace(p, Bm, S, H, Hkv, D, &need);
  if (workspace == nullptr || workspace_bytes < need) return LG_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LG_ERR_UNSUPPORTED;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* dq_acc = static_cast<float*>(workspace);
  float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + round256((size_t)Bm * H * S * D * 4));
  float* lse2 = reinterpret_cast<float*>(reinterpret_cast<char*>(delta) + round256((size_t)Bm * H * S * 4));

  // The 128-row-step kernel's KV tiles are two separately placed 64-row
  // blocks (BlockPairing), each moved as its own 64-row box.
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if ((st = make_map(&tq, q, Bm, S, H, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tk, k, Bm, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tv, v, Bm, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tdo, dout, Bm, S, H, D, 64)) != LG_OK) return st;
  // With fp32 gradients the kernel stores dK / dV directly; the bf16 maps are
  // then built over K / V only to have valid (unused) descriptors.
  if ((st = make_map(&tdk, grad_f32 ? k : dk, Bm, S, Hkv, D, 64)) != LG_OK) return st;
  if ((st = make_map(&tdv, grad_f32 ? v : dv, Bm, S, Hkv, D, 64)) != LG_OK) return st;

  st = cuda_status(lg::launch_bwd_pre(o, o_dtype == LG_F32, dout, delta, dq_acc, lse, lse2, Bm, S, H, D, s));
  if (st != LG_OK) return st;
  lg::BwdParams prm;
  prm.pat = *p;
  prm.lse = lse;
  prm.delta = delta;
  prm.lse2 = lse2;
  prm.dq_acc = dq_acc;
  prm.S = S;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.D = D;
  prm.nqb = max_len / 64;  // the launch order is laid out for the longest sequence
  prm.nkt = (max_len + 127) / 128;
  prm.cu_seqlens = cu_seqlens;
  prm.max_len = max_len;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  // Heavy KV tiles (see heavy_plan); with one per head, in a fixed-length
  // batch, its walk is split into chunks (the packed-sequence call, whose
  // workspace query cannot size per-sequence partials, keeps one CTA).
  {
    const HeavyPlan hp = heavy_plan(*p, prm.nqb, prm.nkt);
    prm.n_heavy = hp.n_heavy;
    for (int t = 0; t < hp.n_heavy; ++t) prm.heavy[t] = hp.heavy[t];
    if (!varlen && hp.n_chunks > 0) {
      prm.n_chunks = hp.n_chunks;
      prm.chunk_steps = hp.chunk_steps;
      char* w = reinterpret_cast<char*>(lse2) + round256((size_t)Bm * H * S * 4);
      prm.hk_part = reinterpret_cast<float*>(w);
      w += round256((size_t)Bm * Hkv * hp.n_chunks * 2 * 128 * D * sizeof(float));
      prm.hk_ticket = reinterpret_cast<unsigned int*>(w);
      st = cuda_status(cudaMemsetAsync(prm.hk_ticket, 0, (size_t)Bm * Hkv * sizeof(unsigned int), s));
      if (st != LG_OK) return st;
    }
  }
  // dK and dV of a KV head sum over its H / Hkv query heads, so their size
  // grows with the group; the bf16 residuals of P and dS then keep the bf16
  // rounding of those operands out of dV and dK.
  prm.split_lo = (H / Hkv) > 1;
  prm.grad_f32 = grad_f32;
  prm.dk_f32 = grad_f32 ? static_cast<float*>(dk) : nullptr;
  prm.dv_f32 = grad_f32 ? static_cast<float*>(dv) : nullptr;
  prm.err = err;
  st = cuda_status(lg::launch_bwd(D, tq, tk, tv, tdo, tdk, tdv, prm, B, s));
  if (st != LG_OK) return st;
  return cuda_status(lg::launch_bwd_dq(dq_acc, dq, grad_f32, scale, Bm, S, H, D, s));
}

lg_status_t lg_sparse_attn_bwd(const lg_pattern_t* p, const void* q, const void* k, const void* v, const void* o,
                               int32_t o_dtype, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               int32_t grad_dtype, int32_t B, int32_t S, int32_t H, int32_t Hkv, int32_t D,
                               float scale, void* workspace, size_t workspace_bytes, lg_stream_t stream) {
  lg_status_t st = check_prefill_shape(p, B, S, H, Hkv, D);
  if (st != LG_OK) return st;
  return bwd_common(p, q, k, v, o, o_dtype, dout, lse, dq, dk, dv, grad_dtype, nullptr, B, S, S, H, Hkv, D, scale,
                    workspace, workspace_bytes, stream);
}

lg_status_t lg_sparse_attn_bwd_varlen(const lg_pattern_t* p, const void* q, const void* k, const void* v,
                                      const void* o, int32_t o_dtype, const void* dout, const float* lse, void* dq,
                                      void* dk, void* dv, int32_t grad_dtype, const int32_t* cu_seqlens, int32_t B,
                                      int32_t total, int32_t max_seqlen, int32_t H, int32_t Hkv, int32_t D,
                                      float scale, void* workspace, size_t workspace_bytes, lg_stream_t stream) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (cu_seqlens == nullptr) return LG_ERR_INVALID_ARG;
  if (B <= 0 || total <= 0 || max_seqlen <= 0 || H <= 0 || Hkv <= 0 || D <= 0 || H % Hkv != 0)
    return LG_ERR_INVALID_ARG;
  if (p->block_size != 64 || max_seqlen % 64 != 0 || total % 4 != 0 || (D != 64 && D != 128))
    return LG_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || max_seqlen > total) return LG_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return LG_ERR_UNSUPPORTED;
  return bwd_common(p, q, k, v, o, o_dtype, dout, lse, dq, dk, dv, grad_dtype, cu_seqlens, B, total, max_seqlen, H,
                    Hkv, D, scale, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- prefill -> decode hand-off
lg_status_t lg_kv_compact_rows(const lg_pattern_t* p, int32_t S, int32_t* rows) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (rows == nullptr || S <= 0) return LG_ERR_INVALID_ARG;
  if (p->block_size != 64 || S % 64 != 0) return LG_ERR_UNSUPPORTED;
  *rows = 64 * lg::compact_blocks(*p, S);
  return LG_OK;
}

lg_status_t lg_kv_compact(const lg_pattern_t* p, const void* k, const void* v, int32_t B, int32_t S, int32_t Hkv,
                          int32_t D, void* k_cache, void* v_cache, int32_t Lmax, int32_t* cache_lens,
                          lg_stream_t stream) {
  int32_t rows = 0;
  lg_status_t st = lg_kv_compact_rows(p, S, &rows);
  if (st != LG_OK) return st;
  if (!k || !v || !k_cache || !v_cache || !cache_lens) return LG_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0) return LG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return LG_ERR_UNSUPPORTED;
  if (B > 65535) return LG_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return LG_ERR_UNSUPPORTED;
  if (Lmax < rows) return LG_ERR_CAPACITY;
  lg::CompactParams prm;
  prm.pat = *p;
  prm.S = S;
  prm.Lmax = Lmax;
  prm.row_chunks = (long long)Hkv * D / 8;
  return cuda_status(lg::launch_compact(k, v, k_cache, v_cache, cache_lens, prm, B, static_cast<cudaStream_t>(stream)));
}

// Paged cache arguments shared by the paged hand-off, append and decode calls.
static lg_status_t check_paged(const void* k_pool, const void* v_pool, int64_t num_pages, const int32_t* block_table,
                               int32_t max_blocks, const int32_t* cache_lens, int32_t B, int32_t Hkv, int32_t D) {
  if (!k_pool || !v_pool || !block_table || !cache_lens) return LG_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || D <= 0 || num_pages <= 0 || max_blocks <= 0) return LG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return LG_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535 || max_blocks > (1 << 24)) return LG_ERR_UNSUPPORTED;
  if (num_pages > ((int64_t)1 << 31) - 1) return LG_ERR_UNSUPPORTED;
  if (!aligned16(k_pool) || !aligned16(v_pool) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(cache_lens) & 3u))
    return LG_ERR_UNSUPPORTED;
  return LG_OK;
}

static lg_status_t paged_state(const lg_pattern_t* p, void* k_pool, void* v_pool, int64_t num_pages,
                               int32_t* block_table, int32_t* block_ids, int32_t max_blocks, int32_t* cache_lens,
                               int32_t* positions, int32_t B, int32_t Hkv, int32_t D, lg::PagedCache* pc) {
  lg_status_t st = check_pattern(p);
  if (st != LG_OK) return st;
  if (p->block_size != 64) return LG_ERR_UNSUPPORTED;
  st = check_paged(k_pool, v_pool, num_pages, block_table, max_blocks, cache_lens, B, Hkv, D);
  if (st != LG_OK) return st;
  if (!block_ids || !positions) return LG_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_ids) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u))
    return LG_ERR_UNSUPPORTED;
  pc->k_pool = k_pool;
  pc->v_pool = v_pool;
  pc->num_pages = num_pages;
  pc->block_table = block_table;
  pc->block_ids = block_ids;
  pc->max_blocks = max_blocks;
  pc->cache_lens = cache_lens;
  pc->positions = positions;
  pc->row_chunks = (long long)Hkv * D / 8;
  pc->err = nullptr;
  return LG_OK;
}

lg_status_t lg_kv_compact_paged(const lg_pattern_t* p, const void* k, const void* v, int32_t B, int32_t S,
                                int32_t Hkv, int32_t D, void* k_pool, void* v_pool, int64_t num_pages,
                                int32_t* block_table, int32_t* block_ids, int32_t max_blocks, int32_t* cache_lens,
                                int32_t* positions, lg_stream_t stream) {
  int32_t rows = 0;
  lg_status_t st = lg_kv_compact_rows(p, S, &rows);
  if (st != LG_OK) return st;
  if (!k || !v) return LG_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return LG_ERR_UNSUPPORTED;
  lg::PagedCache pc;
  st = paged_state(p, k_pool, v_pool, num_pages, block_table, block_ids, max_blocks, cache_lens, positions, B, Hkv, D,
                   &pc);
  if (st != LG_OK) return st;
  if (rows / 64 > max_blocks) return LG_ERR_CAPACITY;
  pc.err = error_word(&st);
  if (st != LG_OK) return st;
  return cuda_status(lg::launch_compact_paged(k, v, *p, S, pc, B, static_cast<cudaStream_t>(stream)));
}

lg_status_t lg_kv_append_paged(const lg_pattern_t* p, const void* k_new, const void* v_new, int32_t B, int32_t Hkv,
                               int32_t D, void* k_pool, void* v_pool, int64_t num_pages, int32_t* block_table,
                               int32_t* block_ids, int32_t max_blocks, int32_t* cache_lens, int32_t* positions,
                               lg_stream_t stream) {
  if (!k_new || !v_new) return LG_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return LG_ERR_UNSUPPORTED;
  lg::PagedCache pc;
  lg_status_t st = paged_state(p, k_pool, v_pool, num_pages, block_table, block_ids, max_blocks, cache_lens, positions,
                               B, Hkv, D, &pc);
  if (st != LG_OK) return st;
  pc.err = error_word(&st);
  if (st != LG_OK) return st;
  return cuda_status(lg::launch_append_paged(k_new, v_new, *p, pc, B, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- decode
lg_status_t lg_sparse_decode_splits(int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax, int32_t num_splits,
                                    int32_t* splits) {
  if (splits == nullptr || B <= 0 || H <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0 || num_splits < 0)
    return LG_ERR_INVALID_ARG;
  if (H % Hkv != 0) return LG_ERR_INVALID_ARG;
  int ns, rps;
  decode_split_rule(B, H, Hkv, D, Lmax, num_splits, &ns, &rps);
  *splits = ns;
  return LG_OK;
}

lg_status_t lg_sparse_decode_workspace(int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax, int32_t num_splits,
                                       size_t* bytes) {
  int32_t ns = 0;
  lg_status_t st = lg_sparse_decode_splits(B, H, Hkv, D, Lmax, num_splits, &ns);
  if (st != LG_OK) return st;
  if (bytes == nullptr) return LG_ERR_INVALID_ARG;
  *bytes = lg::decode_scratch_bytes(B, H, Hkv, D, ns);
  return LG_OK;
}

}  // extern "C"

namespace lg {

// Bytes of split partials and tickets for ns pieces (0 for one piece): the
// workspace layout of every decode entry point.
size_t decode_scratch_bytes(int B, int H, int Hkv, int D, int ns) {
  if (ns <= 1) return 0;
  return round256((size_t)B * H * ns * D * 4) + round256((size_t)B * H * ns * 4) + round256((size_t)B * Hkv * 4);
}

lg_status_t decode_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_lens,
                        const int32_t* block_table, int32_t max_blocks, int64_t num_pages, void* o, int32_t o_dtype,
                        float* lse, int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax, int32_t num_splits,
                        float scale, void* workspace, size_t workspace_bytes, bool shrink_to_fit,
                        cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !cache_lens || !o) return LG_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0 || num_splits < 0) return LG_ERR_INVALID_ARG;
  if (H % Hkv != 0) return LG_ERR_INVALID_ARG;
  if (o_dtype != LG_BF16 && o_dtype != LG_F32) return LG_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return LG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return LG_ERR_UNSUPPORTED;
  const int G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return LG_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return LG_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(cache_lens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return LG_ERR_UNSUPPORTED;
  int ns, rps;
  decode_split_rule(B, H, Hkv, D, Lmax, num_splits, &ns, &rps);
  if (shrink_to_fit && num_splits == 0) {
    // Automatic count and a fixed scratch size: fewer, longer pieces until the partials fit.
    while (ns > 1 && decode_scratch_bytes(B, H, Hkv, D, ns) > workspace_bytes) --ns;
    rps = (Lmax + ns - 1) / ns;
    ns = (Lmax + rps - 1) / rps;
  }
  const size_t need = decode_scratch_bytes(B, H, Hkv, D, ns);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LG_ERR_WORKSPACE;
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LG_ERR_UNSUPPORTED;
  lg_status_t st;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  DecodeParams prm;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.lens = cache_lens;
  prm.block_table = block_table;
  prm.max_blocks = max_blocks;
  prm.num_pages = num_pages;
  prm.o = o;
  prm.o_f32 = o_dtype == LG_F32 ? 1 : 0;
  prm.lse = lse;
  prm.part_o = nullptr;
  prm.part_lse = nullptr;
  prm.tickets = nullptr;
  if (ns > 1) {
    char* w = static_cast<char*>(workspace);
    prm.part_o = reinterpret_cast<float*>(w);
    w += round256((size_t)B * H * ns * D * 4);
    prm.part_lse = reinterpret_cast<float*>(w);
    w += round256((size_t)B * H * ns * 4);
    prm.tickets = reinterpret_cast<unsigned int*>(w);
    // The tickets must start at zero whatever the workspace holds.
    st = cuda_status(cudaMemsetAsync(prm.tickets, 0, (size_t)B * Hkv * 4, stream));
    if (st != LG_OK) return st;
  }
  prm.B = B;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.Lmax = Lmax;
  prm.ns = ns;
  prm.rows_per_split = rps;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = err;
  return cuda_status(launch_decode(D, G, prm, stream));
}

}  // namespace lg

extern "C" {

lg_status_t lg_sparse_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_lens,
                             void* o, int32_t o_dtype, float* lse, int32_t B, int32_t H, int32_t Hkv, int32_t D,
                             int32_t Lmax, int32_t num_splits, float scale, void* workspace, size_t workspace_bytes,
                             lg_stream_t stream) {
  return lg::decode_call(q, k_cache, v_cache, cache_lens, nullptr, 0, 0, o, o_dtype, lse, B, H, Hkv, D, Lmax,
                         num_splits, scale, workspace, workspace_bytes, false, static_cast<cudaStream_t>(stream));
}

lg_status_t lg_sparse_decode_paged(const void* q, const void* k_pool, const void* v_pool, int64_t num_pages,
                                   const int32_t* block_table, int32_t max_blocks, const int32_t* cache_lens, void* o,
                                   int32_t o_dtype, float* lse, int32_t B, int32_t H, int32_t Hkv, int32_t D,
                                   int32_t num_splits, float scale, void* workspace, size_t workspace_bytes,
                                   lg_stream_t stream) {
  lg_status_t st = check_paged(k_pool, v_pool, num_pages, block_table, max_blocks, cache_lens, B, Hkv, D);
  if (st != LG_OK) return st;
  return lg::decode_call(q, k_pool, v_pool, cache_lens, block_table, max_blocks, num_pages, o, o_dtype, lse, B, H,
                         Hkv, D, 64 * max_blocks, num_splits, scale, workspace, workspace_bytes, false,
                         static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- numerics
lg_status_t lg_wait_selftest(int64_t limit_cycles, lg_stream_t stream) {
  if (limit_cycles <= 0 || limit_cycles > 4000000000LL) return LG_ERR_INVALID_ARG;
  lg_status_t st = LG_OK;
  unsigned int* err = error_word(&st);
  if (st != LG_OK) return st;
  return cuda_status(lg::launch_wait_selftest((long long)limit_cycles, err, static_cast<cudaStream_t>(stream)));
}

lg_status_t lg_exp2_device(const float* x, float* y, int64_t n, int32_t method, lg_stream_t stream) {
  if (x == nullptr || y == nullptr || n < 0) return LG_ERR_INVALID_ARG;
  if (method != 0) return LG_ERR_INVALID_ARG;
  if (n == 0) return LG_OK;
  if (n > (int64_t)1 << 40) return LG_ERR_UNSUPPORTED;
  return cuda_status(lg::launch_exp2(x, y, (long long)n, method, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- diagnostics
lg_status_t lg_device_status(int32_t device, uint32_t* flags) {
  if (flags == nullptr) return LG_ERR_INVALID_ARG;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return LG_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return LG_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_lg_error_word, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_lg_error_word, &zero, sizeof(zero));
  cudaSetDevice(prev);
  *flags = v;
  return cuda_status(e);
}

}  // extern "C"
