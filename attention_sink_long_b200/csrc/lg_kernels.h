// lg_kernels.h -- launch interfaces between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lg_attn.h"

namespace lg {

struct FwdParams {
  lg_pattern_t pat;
  float* lse;    // [B, H, S] (or [H, total] with cu_seqlens) or nullptr
  float* o_f32;  // [B, S, H, D] fp32 output, or nullptr for the bf16 TMA-stored output
  int S, H, Hkv;  // S: rows per sequence; with cu_seqlens the total row count
  int nqb;  // S / 64
  int nqt;  // CTAs along the sequence: ceil(S / 256), or ceil(max_len / 256) with cu_seqlens
  const int32_t* cu_seqlens;  // device [B + 1] sequence offsets (packed layout), or nullptr
  int max_len;                // with cu_seqlens: the longest sequence the grid covers
  float scale_log2;  // scale * log2(e)
  unsigned int* err;
};

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream);
// Head dim 128, bf16: the CTA-pair kernel (cta_group::2 MMAs over 512-row query spans).
cudaError_t launch_fwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream);
// Head dim 128, Q and K in fp8 e4m3 (tensor maps over bytes, one 128-byte panel per row).
cudaError_t launch_fwd_fp8qk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream);

struct BwdParams {
  lg_pattern_t pat;
  const float* lse;      // [B, H, S]
  const float* delta;    // [B, H, S] (workspace, written by the preprocess kernel)
  const float* lse2;     // [B, H, S] lse * log2(e) (workspace, written by the preprocess kernel)
  float* dq_acc;         // [B, H, S, D] fp32 (workspace)
  int S, H, Hkv, D;
  int nqb;  // S / 64
  int nkt;  // ceil(S / 128) KV tiles
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  int n_heavy;       // KV tiles scheduled first (for every head), ascending
  int heavy[128];    // their tile indices; see lg_bwd128_kernel's launch order
  int split_lo;      // 1: P and dS also enter dV / dK as bf16 residuals (GQA groups)
  int grad_f32;      // 1: dK / dV written as fp32 straight from the accumulators
  float* dk_f32;     // [B, S, Hkv, D] when grad_f32
  float* dv_f32;
  const int32_t* cu_seqlens = nullptr;  // device [B + 1] offsets of packed sequences (S = total rows), or nullptr
  int max_len = 0;                      // with cu_seqlens: the longest sequence (nkt covers it)
  // The single heavy tile of each head split into n_chunks query ranges of
  // chunk_steps 128-row steps, one CTA each (0: not split). Each chunk writes
  // its fp32 dV / dK partial to hk_part [B, Hkv, n_chunks, 2, 128, D]; the
  // last to finish (hk_ticket [B, Hkv], zero on entry) sums them in chunk
  // order and writes the gradients.
  int n_chunks = 0;
  int chunk_steps = 0;
  float* hk_part = nullptr;
  unsigned int* hk_ticket = nullptr;
  unsigned int* err;
};

cudaError_t launch_bwd_pre(const void* o, int o_f32, const void* dout, float* delta, float* dq_acc, const float* lse,
                           float* lse2, int B, int S,
                           int H, int D, cudaStream_t stream);
cudaError_t launch_bwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const BwdParams& prm,
                       int B, cudaStream_t stream);
// Head dims 64 and 128, with or without query-head groups: 128-row KV tiles
// (two 64-row blocks) and 128-row query steps.
cudaError_t launch_bwd128(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                          const CUtensorMap& tdk, const CUtensorMap& tdv, const BwdParams& prm, int B,
                          cudaStream_t stream);
cudaError_t launch_bwd_dq(const float* dq_acc, void* dq, int dq_f32, float scale, int B, int S, int H, int D,
                          cudaStream_t stream);

// Prefill -> decode hand-off (compact.cu).
struct CompactParams {
  lg_pattern_t pat;
  int S;                // prompt length (multiple of 64)
  int Lmax;             // cache rows per batch row
  long long row_chunks; // 16-byte chunks per token row of all KV heads (Hkv * D / 8)
};
int compact_blocks(const lg_pattern_t& pat, int S);
cudaError_t launch_compact(const void* k, const void* v, void* kc, void* vc, int32_t* lens, const CompactParams& prm,
                           int B, cudaStream_t stream);

// Paged decode cache: pools [num_pages, 64, Hkv, D]; per sequence a block table
// of pages, the pattern block each used entry holds, the cache length and the
// position of the next token.
struct PagedCache {
  void* k_pool;
  void* v_pool;
  long long num_pages;
  int32_t* block_table;  // [B, max_blocks]
  int32_t* block_ids;    // [B, max_blocks]
  int max_blocks;
  int32_t* cache_lens;   // [B]
  int32_t* positions;    // [B]
  long long row_chunks;  // 16-byte chunks per token row of all KV heads
  unsigned int* err;
};
cudaError_t launch_compact_paged(const void* k, const void* v, const lg_pattern_t& pat, int S, const PagedCache& pc,
                                 int B, cudaStream_t stream);
cudaError_t launch_append_paged(const void* k_new, const void* v_new, const lg_pattern_t& pat, const PagedCache& pc,
                                int B, cudaStream_t stream);

struct DecodeParams {
  const void* q;        // [B, H, D] bf16
  const void* k_cache;  // [B, Lmax, Hkv, D] bf16
  const void* v_cache;
  const int32_t* lens;  // [B]
  const int32_t* block_table = nullptr;  // [B, max_blocks] page of each 64-row cache block, or nullptr (contiguous)
  int max_blocks = 0;
  long long num_pages = 0;  // pages in the pool (paged cache)
  void* o;              // [B, H, D] bf16, or fp32 when o_f32
  int o_f32 = 0;        // 1: o is written as fp32 (the unrounded result)
  float* lse;           // [B, H] or nullptr
  float* part_o;        // [B, H, ns, D] fp32 (ns > 1)
  float* part_lse;      // [B, H, ns] (log2 units)
  unsigned int* tickets;  // [B, Hkv]
  int B, H, Hkv, Lmax, ns, rows_per_split;
  float scale_log2;
  unsigned int* err;
};

cudaError_t launch_decode(int D, int G, const DecodeParams& prm, cudaStream_t stream);

// Every decode entry point (api.cu): validation, the split rule, the scratch
// layout (decode_scratch_bytes) and the launch. With shrink_to_fit and an
// automatic split count, the count is lowered until the partials fit
// workspace_bytes (the fixed scratch of lg_sparse_decode_noalloc).
size_t decode_scratch_bytes(int B, int H, int Hkv, int D, int ns);
lg_status_t decode_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_lens,
                        const int32_t* block_table, int32_t max_blocks, int64_t num_pages, void* o, int32_t o_dtype,
                        float* lse, int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax, int32_t num_splits,
                        float scale, void* workspace, size_t workspace_bytes, bool shrink_to_fit,
                        cudaStream_t stream);

cudaError_t launch_wait_selftest(long long limit, unsigned int* err, cudaStream_t stream);
cudaError_t launch_exp2(const float* x, float* y, long long n, int method, cudaStream_t stream);

cudaError_t launch_pattern_iterate(const lg_pattern_t& p, int seqlen, int tile_blocks, int mode, int32_t* out,
                                   int cap, cudaStream_t stream);

}  // namespace lg
