// compact.cu -- prefill -> decode hand-off: the reduced KV cache of a sparse layer.
//
// "A Little Goes a Long Way" (LongGen), Abstract: the sparse layers' static
// block patterns make a "GPU-friendly KV cache reduction" possible -- a layer
// only ever needs the KV blocks its pattern can still reach. After the
// prefill of a prompt of S tokens, the next token (position S, the start of
// block S/64) may attend every earlier whole block that is a sink block, a
// strided block or inside its window. This kernel gathers exactly those
// blocks of K and V, in ascending order, into rows [0, n) of the decode cache
// and sets the cache length. Decoding token S over that cache plus its own
// row is then prefill attention row S.
//
// In the [B, S, Hkv, D] layout a 64-token block of all heads is one
// contiguous range (64 * Hkv * D bf16), so the gather is a list of contiguous
// block copies: one CTA per (output block, batch row), 16-byte streaming loads
// (no L1 allocation: every byte is read once) and stores, four in flight per
// thread. HBM-bound: 2 x 2 x 64 * Hkv * D * 2 bytes per kept block (K and V,
// read and written).
#include "lg_common.cuh"
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_stream_v4(uint4* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__global__ void __launch_bounds__(512) lg_compact_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                         uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                         int32_t* __restrict__ lens, const CompactParams prm) {
  const int b = blockIdx.y;
  const int qb = prm.S / 64;
  const KvIter it(prm.pat, qb, qb - 1);  // blocks below the query's own block
  const int n = it.count();
  if (blockIdx.x == 0 && threadIdx.x == 0) lens[b] = 64 * n;
  if ((int)blockIdx.x >= n) return;
  const int kb = it.nth((int)blockIdx.x);
  const long long chunks = 64 * prm.row_chunks;  // 16-byte chunks in one 64-row block of all heads
  const long long src = ((long long)b * prm.S + 64LL * kb) * prm.row_chunks;
  const long long dst = ((long long)b * prm.Lmax + 64LL * blockIdx.x) * prm.row_chunks;
  const uint4* ks = k + src;
  const uint4* vs = v + src;
  uint4* kd = kc + dst;
  uint4* vd = vc + dst;
  constexpr int U = 4;
  long long c = threadIdx.x;
  for (; c + (U - 1) * 512 < chunks; c += U * 512) {
    uint4 rk[U], rv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      rk[u] = ld_stream_v4(ks + c + u * 512);
      rv[u] = ld_stream_v4(vs + c + u * 512);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      st_stream_v4(kd + c + u * 512, rk[u]);
      st_stream_v4(vd + c + u * 512, rv[u]);
    }
  }
  for (; c < chunks; c += 512) {
    st_stream_v4(kd + c, ld_stream_v4(ks + c));
    st_stream_v4(vd + c, ld_stream_v4(vs + c));
  }
}

// The same gather into a paged cache: output block i of sequence b goes to
// page block_table[b][i] (pages [64, Hkv, D]); the kernel also records the
// block index of each entry, the cache length and the position of the next
// token. A page index outside the pool is reported and its copy skipped.
__global__ void __launch_bounds__(512) lg_compact_paged_kernel(const uint4* __restrict__ k,
                                                               const uint4* __restrict__ v, const lg_pattern_t pat,
                                                               const int S, const PagedCache pc) {
  const int b = blockIdx.y;
  const int qb = S / 64;
  const KvIter it(pat, qb, qb - 1);
  const int n = it.count();
  int32_t* table = pc.block_table + (size_t)b * pc.max_blocks;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    pc.cache_lens[b] = 64 * n;
    pc.positions[b] = S;
  }
  if ((int)blockIdx.x >= n) return;
  const int kb = it.nth((int)blockIdx.x);
  const int page = table[blockIdx.x];
  if (threadIdx.x == 0) pc.block_ids[(size_t)b * pc.max_blocks + blockIdx.x] = kb;
  if (page < 0 || (long long)page >= pc.num_pages) {
    if (threadIdx.x == 0) atomicOr(pc.err, kErrPaged);
    return;
  }
  const long long chunks = 64 * pc.row_chunks;
  const uint4* ks = k + ((long long)b * S + 64LL * kb) * pc.row_chunks;
  const uint4* vs = v + ((long long)b * S + 64LL * kb) * pc.row_chunks;
  uint4* kd = static_cast<uint4*>(pc.k_pool) + (long long)page * chunks;
  uint4* vd = static_cast<uint4*>(pc.v_pool) + (long long)page * chunks;
  constexpr int U = 4;
  long long c = threadIdx.x;
  for (; c + (U - 1) * 512 < chunks; c += U * 512) {
    uint4 rk[U], rv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      rk[u] = ld_stream_v4(ks + c + u * 512);
      rv[u] = ld_stream_v4(vs + c + u * 512);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      st_stream_v4(kd + c + u * 512, rk[u]);
      st_stream_v4(vd + c + u * 512, rv[u]);
    }
  }
  for (; c < chunks; c += 512) {
    st_stream_v4(kd + c, ld_stream_v4(ks + c));
    st_stream_v4(vd + c, ld_stream_v4(vs + c));
  }
}

// Append one decoded token per sequence. The cache of sequence b is entries
// [0, n) of its block table (n = ceil(cache_len / 64)), ascending by pattern
// block, only the last one partial. When the token opens a new block qn
// (position % 64 == 0), the entries whose block is no longer in qn's list --
// the block that just left the local window -- are dropped (kept entries stay
// in order) and the new block takes the first freed page, or the next spare
// page of the table when none was freed: the window's pages form a ring, and
// a layer keeps only what its static pattern can still reach. The token's K
// and V rows are then written to the block's page. An inconsistent state
// (length and position disagreeing, no page left, a page outside the pool)
// is reported and the sequence left unchanged.
__global__ void __launch_bounds__(256) lg_append_paged_kernel(const uint4* __restrict__ k_new,
                                                              const uint4* __restrict__ v_new, const lg_pattern_t pat,
                                                              const PagedCache pc) {
  __shared__ int sm_page, sm_row;
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    int32_t* table = pc.block_table + (size_t)b * pc.max_blocks;
    int32_t* ids = pc.block_ids + (size_t)b * pc.max_blocks;
    const int pos = pc.positions[b];
    const int len = pc.cache_lens[b];
    const int n = (len + 63) / 64;
    bool ok = pos >= 0 && pos < 0x7fffffff && len >= 0 && len <= pos && n <= pc.max_blocks && (len & 63) == (pos & 63);
    int page = -1, row = 0, new_len = len;
    if (ok && (pos & 63) == 0) {
      const int qn = pos >> 6;
      int w = 0;
      for (int x = 0; x < n; ++x) {
        if (!in_list(pat, qn, ids[x])) continue;
        if (w != x) {  // stable partition: kept entries move down in order, freed pages up
          const int tp = table[w], ti = ids[w];
          table[w] = table[x];
          ids[w] = ids[x];
          table[x] = tp;
          ids[x] = ti;
        }
        ++w;
      }
      if (w < pc.max_blocks) {
        page = table[w];
        ids[w] = qn;
        new_len = 64 * w + 1;
      } else {
        ok = false;
      }
    } else if (ok) {
      page = table[n - 1];
      row = pos & 63;
      new_len = len + 1;
    }
    if (ok && (page < 0 || (long long)page >= pc.num_pages)) ok = false;
    if (ok) {
      pc.cache_lens[b] = new_len;
      pc.positions[b] = pos + 1;
    } else {
      atomicOr(pc.err, kErrPaged);
      page = -1;
    }
    sm_page = page;
    sm_row = row;
  }
  __syncthreads();
  const int page = sm_page;
  if (page < 0) return;
  const long long dst = ((long long)page * 64 + sm_row) * pc.row_chunks;
  const long long src = (long long)b * pc.row_chunks;
  uint4* kd = static_cast<uint4*>(pc.k_pool) + dst;
  uint4* vd = static_cast<uint4*>(pc.v_pool) + dst;
  for (long long c = threadIdx.x; c < pc.row_chunks; c += 256) {
    kd[c] = k_new[src + c];
    vd[c] = v_new[src + c];
  }
}

int compact_blocks(const lg_pattern_t& pat, int S) {
  const int qb = S / 64;
  return KvIter(pat, qb, qb - 1).count();
}

cudaError_t launch_compact(const void* k, const void* v, void* kc, void* vc, int32_t* lens, const CompactParams& prm,
                           int B, cudaStream_t stream) {
  const int n = compact_blocks(prm.pat, prm.S);
  dim3 grid(n > 0 ? n : 1, B);
  lg_compact_kernel<<<grid, 512, 0, stream>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v),
                                              static_cast<uint4*>(kc), static_cast<uint4*>(vc), lens, prm);
  return cudaGetLastError();
}

cudaError_t launch_compact_paged(const void* k, const void* v, const lg_pattern_t& pat, int S, const PagedCache& pc,
                                 int B, cudaStream_t stream) {
  const int n = compact_blocks(pat, S);
  dim3 grid(n > 0 ? n : 1, B);
  lg_compact_paged_kernel<<<grid, 512, 0, stream>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), pat, S,
                                                    pc);
  return cudaGetLastError();
}

cudaError_t launch_append_paged(const void* k_new, const void* v_new, const lg_pattern_t& pat, const PagedCache& pc,
                                int B, cudaStream_t stream) {
  lg_append_paged_kernel<<<B, 256, 0, stream>>>(static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                                                pat, pc);
  return cudaGetLastError();
}

}  // namespace lg
