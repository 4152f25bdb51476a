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

}  // namespace lg
