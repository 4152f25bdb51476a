/*
 * lg_attn.h -- C ABI of the LongGen sparse-attention hot path for NVIDIA B200 (sm_100a).
 *
 * Method: "A Little Goes a Long Way: Efficient Long Context Training and
 * Inference with Partial Contexts" (LongGen, arXiv 2410.01485).
 *   - Abstract, insight 1: sparse layers keep the initial tokens (attention
 *     sink), the recent tokens (window attention) and strided token blocks
 *     (blockwise sparse attention), chosen for GPU-friendly memory access.
 *   - Abstract, insight 2: the middle 1/3 of the layers keep full attention
 *     (the all-blocks causal special case of the same kernels).
 *   - atlas.scime.ai summary, "Approach": static, block-wise access; training
 *     with a FlashAttention-2-based kernel (exact attention); serving over the
 *     reduced KV cache of the sparse layers.
 *   - Abstract / summary, "Key results": 1.67x prefill and 1.41x decode speedup
 *     and KV cache 69.2 GB -> 26.5 GB at 128K (the decode entry point below is
 *     the step those figures time).
 *
 * Conventions for every entry point:
 *   - Every function returns lg_status_t (LG_OK == 0). Argument errors are
 *     detected on the host before anything is launched; nothing is written.
 *   - The caller owns every buffer. The library never allocates or frees
 *     device memory and never synchronises the stream it is given (the one
 *     exception, lg_device_status, says so). Pointers marked "device" must be
 *     device memory of the current device, 16-byte aligned.
 *   - Tensors are contiguous, row-major, with the layouts given per call:
 *       q, o, dout, dq   [B, S, H, D]    bf16 (o, dq may be fp32, see lg_dtype_t)
 *       k, v, dk, dv     [B, S, Hkv, D]  bf16 (dk, dv may be fp32)
 *       lse              [B, H, S]       fp32, natural log
 *     Query head h reads KV head h / (H / Hkv).
 *   - Launch errors map to LG_ERR_CUDA. Asynchronous device faults surface at
 *     the caller's next synchronisation. Every device-side wait in the kernels
 *     is bounded; a wait that runs out sets a flag readable with
 *     lg_device_status and the kernel returns early (its outputs are then
 *     undefined).
 *   - Supported: D in {64, 128}; block_size == 64; S % 64 == 0; H % Hkv == 0;
 *     1 <= local_blocks; sink_blocks >= 0; stride >= 0. Anything else returns
 *     LG_ERR_UNSUPPORTED or LG_ERR_INVALID_ARG.
 */
#ifndef LG_ATTN_H_
#define LG_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef void* lg_stream_t;

typedef enum {
  LG_OK = 0,
  LG_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad pattern field */
  LG_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes / alignment */
  LG_ERR_WORKSPACE = 3,    /* workspace missing or smaller than the query says */
  LG_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed */
  LG_ERR_INTERNAL = 5,
  LG_ERR_CAPACITY = 6      /* an output buffer given with a capacity is too small */
} lg_status_t;

/*
 * Static block pattern (atlas.scime.ai summary, "Approach": static, block-wise
 * access; Abstract, insight 1: sink, window, strided blocks).
 * Query block i = q / block_size attends to KV block j = k / block_size iff
 *   j <= i  and  ( j < sink_blocks  or  i - j < local_blocks
 *                  or (stride > 0 and j % stride == 0) ),
 * with token-level causality (k <= q) inside the diagonal block.
 * local_blocks counts the diagonal block; stride == 0 disables the strided
 * term. Full causal attention is {64, 0, INT32_MAX, 0}.
 */
typedef struct {
  int32_t block_size;
  int32_t sink_blocks;
  int32_t local_blocks;
  int32_t stride;
} lg_pattern_t;

/* Human-readable name of a status code (static storage; never NULL). */
const char* lg_strerror(lg_status_t status);

/* ABI version of this library, (major << 16) | minor. */
int32_t lg_version(void);

/*
 * Element type of the forward output O (and of O as an input of the
 * backward) and of the gradient outputs. LG_BF16 rounds to nearest even and
 * is the training format; LG_F32 keeps the fp32 accumulators as they are --
 * the backward's Delta = rowsum(dO * O) is then exact to fp32, and parity can
 * be checked apart from the output rounding.
 */
typedef enum { LG_BF16 = 0, LG_F32 = 1 } lg_dtype_t;

/* ------------------------------------------------------------------------ */
/* Pattern expansion (host, pure integer)                                    */
/* ------------------------------------------------------------------------ */

/*
 * CSR of KV blocks per query block for a sequence of seqlen tokens
 * (seqlen % block_size == 0, nqb = seqlen / block_size): row_ptr[nqb + 1] and
 * col[nnz], each row sorted ascending without duplicates. Host pointers.
 * Capacity idiom: with col == NULL only *nnz is written (row_ptr may also be
 * NULL); otherwise cap is the length of col and LG_ERR_CAPACITY is returned
 * (with *nnz set) when cap < nnz.
 */
lg_status_t lg_pattern_expand(const lg_pattern_t* pattern, int32_t seqlen, int32_t* row_ptr,
                              int32_t* col, int64_t cap, int64_t* nnz);

/* The transpose (CSC): query blocks per KV block, col_ptr[nqb + 1], row[nnz]. Same idiom. */
lg_status_t lg_pattern_expand_t(const lg_pattern_t* pattern, int32_t seqlen, int32_t* col_ptr,
                                int32_t* row, int64_t cap, int64_t* nnz);

/* Number of unmasked (query, key) token pairs of one head: the unit of useful work. */
lg_status_t lg_pattern_pairs(const lg_pattern_t* pattern, int32_t seqlen, int64_t* pairs);

/*
 * Runs, on the device, the block iterators the attention kernels use, and
 * records what they visit, so tests can compare them bit for bit with the
 * CSR / CSC lists (static, block-wise access: atlas.scime.ai summary,
 * "Approach"). One record per tile u at out[u * (cap + 1)]: the entry count
 * n, then the entries (entries beyond cap are not written; the count still
 * is). A block entry is (block << 8) | membership, bit t of the membership
 * saying whether the entry is in the list of the tile's t-th block. Modes:
 *   0  forward union: tiles of tile_blocks (1, 2, 4, 8) query blocks; the
 *      KV blocks of the union of their lists, ascending (n < 0 flags an
 *      iterator whose closed-form count disagrees with its walk);
 *   1  backward union: tiles of tile_blocks (1, 2) KV blocks; the query
 *      blocks of the union of their transposed lists, ascending;
 *   2  the forward kernels' chunked walk of a query span of tile_blocks
 *      (4 or 8) blocks: two entries per chunk of two consecutive listed KV
 *      blocks, the second -1 when the chunk holds one block;
 *   3  the backward kernels' KV tiles (tile_blocks == 2): tile u of the
 *      pairing of KV blocks (sink / strided blocks with each other, then the
 *      window blocks in order) records its blocks kx, ky (-1 for none), the
 *      first and last query block it walks, then one entry per query block
 *      in that range, bit 0 / bit 1 for kx / ky.
 * Device pointer out holds (number of tiles) * (cap + 1) int32 (mode 3:
 * ceil(nqb / 2) tiles). Errors: LG_ERR_INVALID_ARG (bad pattern or mode,
 * NULL out, seqlen not a positive multiple of block_size, cap < 0),
 * LG_ERR_UNSUPPORTED (block_size != 64, tile_blocks not listed for the
 * mode, 2^23 or more blocks), LG_ERR_CUDA (launch).
 */
lg_status_t lg_pattern_iterate_device(const lg_pattern_t* pattern, int32_t seqlen, int32_t tile_blocks,
                                      int32_t mode, int32_t* out, int32_t cap, lg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Prefill forward                                                          */
/* ------------------------------------------------------------------------ */

/* Workspace bytes for lg_sparse_attn_fwd (currently 0: the block lists are generated in-kernel). */
lg_status_t lg_sparse_attn_fwd_workspace(const lg_pattern_t* pattern, int32_t B, int32_t S, int32_t H,
                                         int32_t Hkv, int32_t D, size_t* bytes);

/*
 * O = softmax_mask(scale * Q K^T) V for every (b, h), and LSE per query row.
 * Abstract, insights 1-2; atlas.scime.ai summary, "Approach" (exact,
 * FlashAttention-style attention under the static mask above).
 * Device pointers: q [B,S,H,D] bf16, k/v [B,S,Hkv,D] bf16, o [B,S,H,D]
 * (written) of element type o_dtype (LG_BF16 or LG_F32), lse [B,H,S] fp32
 * (written; may be NULL when not needed). KV blocks outside the pattern are
 * never read.
 */
lg_status_t lg_sparse_attn_fwd(const lg_pattern_t* pattern, const void* q, const void* k, const void* v,
                               void* o, int32_t o_dtype, float* lse, int32_t B, int32_t S, int32_t H, int32_t Hkv,
                               int32_t D, float scale, void* workspace, size_t workspace_bytes, lg_stream_t stream);

/*
 * The forward above (head dim 128) computed by pairs of CTAs that share
 * 256-row tcgen05 MMAs (cta_group::2; no TMA multicast): each pair owns a
 * 512-row query span of one head, each CTA loads half of every K/V chunk,
 * and P goes through shared memory so the next chunk's S = Q K^T runs while
 * the softmax of this one is still exponentiating. Same arithmetic and
 * results as lg_sparse_attn_fwd (bit-equal on the dense pattern; within one
 * bf16 ulp of O and 2e-6 of LSE where the wider span changes which
 * partially-masked chunks a row meets). A throughput variant: on the
 * workloads measured it runs at 0.9-1.0x of lg_sparse_attn_fwd's speed.
 * Arguments, layouts and errors as lg_sparse_attn_fwd (no workspace);
 * LG_ERR_UNSUPPORTED for D != 128.
 */
lg_status_t lg_sparse_attn_fwd_pair(const lg_pattern_t* pattern, const void* q, const void* k, const void* v,
                                    void* o, int32_t o_dtype, float* lse, int32_t B, int32_t S, int32_t H,
                                    int32_t Hkv, int32_t D, float scale, lg_stream_t stream);

/*
 * The forward above with Q and K in fp8 e4m3 (one byte each, head dim 128):
 * S = (q8 k8^T) * q_descale * k_descale, computed on the fp8 tensor-core path
 * at twice the bf16 rate; the softmax, P V (bf16) and the outputs are those of
 * lg_sparse_attn_fwd. A throughput experiment: the pages make no fp8 claim,
 * and the result is exact attention over the dequantised Q and K (the
 * quantisation error is the caller's). Device pointers: q8 [B,S,H,128],
 * k8 [B,S,Hkv,128] e4m3 bytes; v bf16; o, lse as lg_sparse_attn_fwd.
 * Errors: those of lg_sparse_attn_fwd; LG_ERR_INVALID_ARG for a descale that
 * is not positive and finite; LG_ERR_UNSUPPORTED for D != 128.
 */
lg_status_t lg_sparse_attn_fwd_fp8qk(const lg_pattern_t* pattern, const void* q8, const void* k8, const void* v,
                                     float q_descale, float k_descale, void* o, int32_t o_dtype, float* lse, int32_t B,
                                     int32_t S, int32_t H, int32_t Hkv, int32_t D, float scale, lg_stream_t stream);

/*
 * The forward above for a batch of sequences of different lengths, packed
 * one after another (the prefill of several prompts; Abstract and summary,
 * "Key results": 1.67x prefill). Sequence b is rows [cu_seqlens[b],
 * cu_seqlens[b+1]) of the packed tensors and the pattern applies to positions
 * inside it (its first row is position 0); no sequence sees another's rows.
 * Device pointers: q [total,H,D] bf16, k/v [total,Hkv,D] bf16, o [total,H,D]
 * (written) of element type o_dtype, lse [H,total] fp32 (written; may be
 * NULL), cu_seqlens [B+1] int32 (read on the device): non-decreasing, starting
 * at >= 0, ending at <= total, every length a multiple of 64 and at most
 * max_seqlen (a multiple of 64 that sizes the grid). Rows of o outside every
 * sequence are not written. A cu_seqlens entry that breaks these rules is
 * found on the device: that sequence is skipped (its o rows unwritten) and
 * lg_device_status reports bit 4.
 */
lg_status_t lg_sparse_attn_fwd_varlen(const lg_pattern_t* pattern, const void* q, const void* k, const void* v,
                                      void* o, int32_t o_dtype, float* lse, const int32_t* cu_seqlens, int32_t B,
                                      int32_t total, int32_t max_seqlen, int32_t H, int32_t Hkv, int32_t D,
                                      float scale, lg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Training backward                                                        */
/* ------------------------------------------------------------------------ */

/*
 * Workspace bytes for lg_sparse_attn_bwd: fp32 dQ accumulator [B,H,S,D] plus
 * Delta and LSE * log2(e) [B,H,S]; and, when each head has a single KV tile
 * that far more queries see than the rest (the sink tile of a sink + window
 * pattern), fp32 dV / dK partials of that tile's walk split into chunks
 * [B,Hkv,chunks,2,128,D] and B*Hkv counters.
 */
lg_status_t lg_sparse_attn_bwd_workspace(const lg_pattern_t* pattern, int32_t B, int32_t S, int32_t H,
                                         int32_t Hkv, int32_t D, size_t* bytes);

/*
 * Gradients of the forward above given dO (atlas.scime.ai summary, "Approach":
 * the training kernel; "Key results": 1.55x training speedup at 128K):
 *   P = exp(scale Q K^T - LSE) on the mask, Delta = rowsum(dO * O),
 *   dV = P^T dO, dS = P * (dO V^T - Delta), dQ = scale dS K, dK = scale dS^T Q.
 * Device pointers: q, k, v, dout bf16; o as written by the forward, of
 * element type o_dtype; lse as written by the forward; dq [B,S,H,D], dk/dv
 * [B,S,Hkv,D] (written; dk/dv sum over the query heads of a KV group) of
 * element type grad_dtype. P and dS enter the tensor-core products as bf16;
 * with query-head groups (H > Hkv) they also enter dV / dK as a bf16 hi + lo
 * pair (exact to fp32 accumulation), since those sums grow with the group.
 * A single heavy KV tile per head (the sink tile) is walked by several CTAs,
 * each over a range of query rows; its dV / dK are the sum of their fp32
 * partials taken in a fixed order, so results do not vary from run to run.
 * workspace (device, 256-byte aligned) of at least the queried size; its
 * contents on entry do not matter.
 */
lg_status_t lg_sparse_attn_bwd(const lg_pattern_t* pattern, const void* q, const void* k, const void* v,
                               const void* o, int32_t o_dtype, const void* dout, const float* lse, void* dq,
                               void* dk, void* dv, int32_t grad_dtype, int32_t B, int32_t S, int32_t H, int32_t Hkv,
                               int32_t D, float scale, void* workspace, size_t workspace_bytes, lg_stream_t stream);

/*
 * The backward above for packed sequences of different lengths, the
 * counterpart of lg_sparse_attn_fwd_varlen (training on a batch of documents
 * of mixed lengths; summary, "Key results": 1.55x training). Tensors and the
 * offsets as in lg_sparse_attn_fwd_varlen: q, o, dout, dq [total,H,D];
 * k, v, dk, dv [total,Hkv,D]; lse [H,total] as that forward wrote it;
 * cu_seqlens [B+1] int32 on the device. In addition every offset must be a
 * multiple of 4 (16-byte aligned LSE rows) and total a multiple of 4
 * (LG_ERR_UNSUPPORTED otherwise, on the host for total). Gradients of a
 * sequence depend only on its own rows. dq rows outside every sequence are
 * written as zero; dk / dv rows outside every sequence are not written. A
 * cu_seqlens entry that breaks the rules is found on the device: that
 * sequence is skipped and lg_device_status reports bit 4. Workspace:
 * lg_sparse_attn_bwd_workspace(pattern, 1, total, H, Hkv, D) bytes.
 */
lg_status_t lg_sparse_attn_bwd_varlen(const lg_pattern_t* pattern, const void* q, const void* k, const void* v,
                                      const void* o, int32_t o_dtype, const void* dout, const float* lse, void* dq,
                                      void* dk, void* dv, int32_t grad_dtype, const int32_t* cu_seqlens, int32_t B,
                                      int32_t total, int32_t max_seqlen, int32_t H, int32_t Hkv, int32_t D,
                                      float scale, void* workspace, size_t workspace_bytes, lg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Prefill -> decode hand-off: the reduced KV cache                         */
/* ------------------------------------------------------------------------ */

/*
 * Rows of the reduced cache lg_kv_compact writes for a prompt of S tokens
 * (S a multiple of block_size = 64): 64 x the number of whole blocks kb < S/64
 * with kb < sink_blocks, or S/64 - kb < local_blocks, or (stride > 0 and
 * kb % stride == 0). Written to *rows. Host only; errors: LG_ERR_INVALID_ARG
 * (bad pattern, S <= 0, rows NULL), LG_ERR_UNSUPPORTED (block_size != 64,
 * S % 64 != 0).
 */
lg_status_t lg_kv_compact_rows(const lg_pattern_t* pattern, int32_t S, int32_t* rows);

/*
 * Prefill -> decode hand-off for a sparse layer (Abstract: the static patterns
 * allow a "GPU-friendly KV cache reduction"; summary, "Key results": 69.2 ->
 * 26.5 GB of KV cache at 128K). After the prefill of S tokens, the next token
 * (position S) may attend exactly the whole earlier blocks counted by
 * lg_kv_compact_rows; this call copies those 64-row blocks of k and v, in
 * ascending block order, to rows [0, rows) of k_cache / v_cache and writes
 * cache_lens[b] = rows for every batch row. Decoding token S over rows
 * [0, rows) plus its own K/V row (appended by the caller at row `rows`)
 * equals prefill attention row S. Values are copied bit for bit.
 * Device pointers, 16-byte aligned: k, v [B,S,Hkv,D] bf16 (read);
 * k_cache, v_cache [B,Lmax,Hkv,D] bf16 (rows [0, rows) written, the rest
 * untouched; must not overlap k / v); cache_lens [B] int32 (written).
 * Errors: LG_ERR_INVALID_ARG (NULL pointer, non-positive sizes, bad pattern),
 * LG_ERR_UNSUPPORTED (block_size != 64, S % 64 != 0, D not 64 or 128,
 * misaligned pointer), LG_ERR_CAPACITY (Lmax < rows), LG_ERR_CUDA (launch).
 */
lg_status_t lg_kv_compact(const lg_pattern_t* pattern, const void* k, const void* v, int32_t B, int32_t S,
                          int32_t Hkv, int32_t D, void* k_cache, void* v_cache, int32_t Lmax, int32_t* cache_lens,
                          lg_stream_t stream);

/*
 * Paged decode cache (PagedAttention-style block tables, the layout the
 * pages' vLLM decoding runs on). One page holds one 64-token pattern block
 * of every KV head: k_pool, v_pool are [num_pages, 64, Hkv, D] bf16. Per
 * sequence b, all device int32:
 *   block_table[b, 0..max_blocks)  page indices owned by the sequence. The
 *       caller assigns them (distinct across sequences; -1 = none). Entries
 *       [0, n) with n = ceil(cache_lens[b] / 64) hold the cache in ascending
 *       block order, only entry n-1 may be partial; entries [n, max_blocks)
 *       are spare pages the sequence takes as it grows. The calls below
 *       permute the entries they manage.
 *   block_ids[b, 0..max_blocks)    pattern block index held by each entry
 *       in [0, n) (written by the calls below).
 *   cache_lens[b]                  rows in the cache.
 *   positions[b]                   position of the next token (tokens seen).
 *
 * lg_kv_compact_paged: the hand-off of lg_kv_compact into pages. Block i of
 * the reduced cache goes to page block_table[b][i]; then block_ids[b][i] is
 * that block, cache_lens[b] = lg_kv_compact_rows(S), positions[b] = S.
 * Errors: those of lg_kv_compact; LG_ERR_CAPACITY when the reduced cache has
 * more blocks than max_blocks. A page index outside [0, num_pages) is
 * reported through lg_device_status (bit 6) and that block is not copied.
 *
 * lg_kv_append_paged: appends one token per sequence (k_new, v_new
 * [B, Hkv, D] bf16, the token at positions[b]) and advances positions[b].
 * When the token opens a new block qn (position % 64 == 0), the entries whose
 * block is no longer in qn's list (the block that just left the local
 * window) are dropped, keeping the others in order, and block qn takes the
 * first dropped page, else the next spare one: the window's pages are reused
 * as a ring, so a sink+window layer needs sink_blocks + local_blocks pages
 * for any length. After the append, the cache of b holds exactly the rows
 * prefill attention row positions[b]-1 may attend, and lg_sparse_decode_paged
 * over it gives that row. A state that breaks the rules above (cache_lens and
 * positions disagreeing modulo 64, cache_lens > positions, no page left, a
 * page outside the pool) is reported (bit 6) and the sequence left as it was.
 * Start a sequence with lg_kv_compact_paged, or with cache_lens = positions
 * = 0.
 */
lg_status_t lg_kv_compact_paged(const lg_pattern_t* pattern, const void* k, const void* v, int32_t B, int32_t S,
                                int32_t Hkv, int32_t D, void* k_pool, void* v_pool, int64_t num_pages,
                                int32_t* block_table, int32_t* block_ids, int32_t max_blocks, int32_t* cache_lens,
                                int32_t* positions, lg_stream_t stream);
lg_status_t lg_kv_append_paged(const lg_pattern_t* pattern, const void* k_new, const void* v_new, int32_t B,
                               int32_t Hkv, int32_t D, void* k_pool, void* v_pool, int64_t num_pages,
                               int32_t* block_table, int32_t* block_ids, int32_t max_blocks, int32_t* cache_lens,
                               int32_t* positions, lg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Decode over the reduced KV cache                                         */
/* ------------------------------------------------------------------------ */

/*
 * The number of KV splits lg_sparse_decode uses when num_splits == 0 (auto),
 * written to *splits. Always >= 1. One query head per KV head: pieces of 512
 * cache rows (1024 at D = 64), halved while B * Hkv * splits < 1184. Query-
 * head groups: pieces of 1024 rows when B * Hkv > 128, else about 256 / (B *
 * Hkv) pieces (about 256 CTAs). Never more than ceil(Lmax / 64) pieces.
 */
lg_status_t lg_sparse_decode_splits(int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax,
                                    int32_t num_splits, int32_t* splits);

/* Workspace bytes for lg_sparse_decode (per-split partial o and lse, plus one ticket per (b, kv head)). */
lg_status_t lg_sparse_decode_workspace(int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax,
                                       int32_t num_splits, size_t* bytes);

/*
 * Single-token attention of each sequence's query over its cached rows:
 *   o[b,h] = sum_{r < cache_lens[b]} softmax_r(scale q[b,h] . K[b,r]) V[b,r],
 *   lse[b,h] = log sum_r exp(scale q[b,h] . K[b,r]).
 * The cache of a sparse layer holds only what its pattern can still reach
 * (sink + window, + strided blocks), a full layer's holds every token
 * (Abstract: KV cache reduction; summary, "Key results": 69.2 -> 26.5 GB and
 * 1.41x decode). Row order does not matter (softmax is permutation
 * invariant), so a ring-buffered window is fine.
 * Device pointers: q [B,H,D] bf16; k_cache, v_cache [B,Lmax,Hkv,D] bf16;
 * cache_lens [B] int32 with 1 <= cache_lens[b] <= Lmax (values are read on
 * the device and clamped to [0, Lmax]; a zero length yields o = 0,
 * lse = -inf); o [B,H,D] (written) of element type o_dtype: LG_BF16 (round
 * to nearest even) or LG_F32 (the merged fp32 result before that rounding);
 * lse [B,H] fp32 (written, may be NULL).
 * The KV range of each (b, kv head) is cut into num_splits pieces (0 = auto,
 * see lg_sparse_decode_splits); partial results are merged by
 * log-sum-exp in the same launch by the last CTA to finish each (b, kv head).
 * workspace (device, 256-byte aligned) of at least the queried size; its
 * ticket region is cleared on the stream by every call.
 */
lg_status_t lg_sparse_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_lens,
                             void* o, int32_t o_dtype, float* lse, int32_t B, int32_t H, int32_t Hkv, int32_t D,
                             int32_t Lmax, int32_t num_splits, float scale, void* workspace, size_t workspace_bytes,
                             lg_stream_t stream);

/*
 * lg_sparse_decode over a paged cache (see lg_kv_compact_paged): cache row r
 * of sequence b is row r % 64 of page block_table[b][r / 64]. Arguments as
 * lg_sparse_decode, with Lmax = 64 * max_blocks for the split rule and the
 * workspace size (lg_sparse_decode_workspace with that Lmax). cache_lens[b] is
 * clamped to [0, 64 * max_blocks]; a page index outside [0, num_pages) is
 * reported (bit 6) and its rows left out. Errors: those of lg_sparse_decode,
 * plus LG_ERR_INVALID_ARG for num_pages or max_blocks <= 0 and
 * LG_ERR_UNSUPPORTED for max_blocks > 2^24.
 */
lg_status_t lg_sparse_decode_paged(const void* q, const void* k_pool, const void* v_pool, int64_t num_pages,
                                   const int32_t* block_table, int32_t max_blocks, const int32_t* cache_lens, void* o,
                                   int32_t o_dtype, float* lse, int32_t B, int32_t H, int32_t Hkv, int32_t D,
                                   int32_t num_splits, float scale, void* workspace, size_t workspace_bytes,
                                   lg_stream_t stream);

/*
 * Size of the fixed device scratch array behind lg_sparse_decode_noalloc:
 * 16 MiB on every device that loads the library, held until process exit.
 */
#define LG_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/*
 * lg_sparse_decode without a workspace, for callers that cannot allocate
 * device memory. The paper has no counterpart: this is a deployment
 * convenience. Typical such callers are a plugin inside a host framework that
 * owns all device memory through its own pool and forbids side allocations, a
 * latency-critical decode loop where cudaMalloc / cudaFree would synchronise
 * the device and stall every other stream, and a thin C / FFI caller with no
 * device allocator of its own. Arguments and results are those of
 * lg_sparse_decode minus the workspace; the caller still passes all inputs
 * and outputs (o of element type o_dtype, as lg_sparse_decode). Nothing is
 * allocated or freed.
 * The split partials and tickets live in one file-scope device array of
 * LG_DECODE_NOALLOC_SCRATCH_BYTES. The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current)
 * and caches it with the device's current context; a call that finds a new
 * context there (after cudaDeviceReset) looks it up again. Make the first
 * call on a device before any stream capture. The current device must be the
 * one the stream and q belong to (LG_ERR_INVALID_ARG otherwise: the array of
 * one device is not the scratch of another). With num_splits == 0 the
 * automatic split count is lowered until the partials fit the array; an
 * explicit num_splits whose partials need more than the array holds
 * (B * H * num_splits * (D + 1) * 4 bytes, roughly) returns LG_ERR_WORKSPACE
 * and launches nothing. Every call shares the array: the tickets are cleared
 * on the given stream at each call, and calls that overlap on the GPU (other
 * streams, other host threads) race on it, so serialise them.
 */
lg_status_t lg_sparse_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* cache_lens, void* o, int32_t o_dtype, float* lse, int32_t B,
                                     int32_t H, int32_t Hkv, int32_t D, int32_t Lmax, int32_t num_splits,
                                     float scale, lg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Numerics                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * y[k] = 2^x[k] for k < n, evaluated on the device exactly as the softmax
 * kernels evaluate their exponentials: the special-function unit's
 * ex2.approx (method 0; any other method is LG_ERR_INVALID_ARG). Device
 * pointers x, y of n fp32. For tests of the softmax arithmetic; not on the
 * attention path itself.
 */
lg_status_t lg_exp2_device(const float* x, float* y, int64_t n, int32_t method, lg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                              */
/* ------------------------------------------------------------------------ */

/*
 * Self-test of the bounded-wait failure path every kernel uses (no passage of
 * the pages; this is the library's own failure detection): launches one
 * thread that waits on a barrier nothing arrives on, gives up after
 * limit_cycles SM cycles (1 .. 4e9) and sets bit 5 of the device error word
 * (read it with lg_device_status). The device stays usable afterwards.
 * Errors: LG_ERR_INVALID_ARG (limit out of range), LG_ERR_CUDA.
 */
lg_status_t lg_wait_selftest(int64_t limit_cycles, lg_stream_t stream);

/*
 * Reads and clears the device-side error flags of the given device (bit 0:
 * a forward wait ran out, bit 1: a backward wait ran out, bit 2: decode,
 * bit 3: a kernel found its shared-memory layout would not fit the block's
 * allocation and did no work, bit 4: a variable-length call skipped a
 * sequence whose offsets broke the rules, bit 5: lg_wait_selftest's wait ran
 * out, as it should, bit 6: a paged-cache call met a page index outside the
 * pool, an inconsistent sequence state or a full block table, and skipped
 * that work). SYNCHRONISES that device. *flags == 0 means
 * every kernel since the last call ran to completion.
 */
lg_status_t lg_device_status(int32_t device, uint32_t* flags);

#ifdef __cplusplus
}
#endif

#endif /* LG_ATTN_H_ */
