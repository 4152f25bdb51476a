// decode.cu -- single-token decode over the (reduced) KV cache, split-KV with an
// in-launch log-sum-exp merge.
//
// "A Little Goes a Long Way" (LongGen), Abstract (GPU-friendly KV cache
// reduction) and the atlas.scime.ai summary, "Key results" (KV cache 69.2 GB ->
// 26.5 GB, 1.41x decoding): a sparse layer's cache holds only the rows its
// static pattern can still reach, a full layer's holds all of them; decode is
// one query row attending to every cached row, so it is a pure HBM stream.
//
// Two kernels, both with grid (splits, Hkv, B) and 128 threads, and both
// serving all G = H/Hkv query heads of a KV head from one CTA so K/V bytes are
// read once per KV head:
//   lg_decode_kernel (G = 1): D/8 threads share one cache row (16 B each, one
//     non-allocating vector load for K and one for V); a warp covers 32*8/D
//     rows per step and U steps are unrolled so each thread has 2*U loads in
//     flight.
//   lg_decode_mma_kernel (G >= 2): cache blocks staged in shared memory and
//     computed with warp tensor-core MMAs, the heads on the M side (below).
// Each CTA reduces its rows to a partial (o, lse); with more than one split
// the last CTA of each (b, kv head) -- found through an atomic ticket, with no
// waiting -- merges the partials.
//
// Paged caches (PAGED = true): cache row r of sequence b lives in page
// block_table[b][r / 64] at page row r % 64, every page [64, Hkv, D]; a page
// index outside the pool is reported (kErrPaged) and its rows are skipped.
#include "lg_common.cuh"
#include "lg_kernels.h"

// Grouped-query kernel: cache rows per staged block and stages in flight
// (measured: 64 rows and two stages beat 128-row blocks and three or four
// stages, which leave fewer CTAs per SM).
#ifndef LG_DECODE_MMA_BR
#define LG_DECODE_MMA_BR 64
#endif
#ifndef LG_DECODE_MMA_STAGES
#define LG_DECODE_MMA_STAGES 2
#endif

namespace lg {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16);
  f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16);
  f[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Merge (m2, l2, a2) into (m, l, a): both are softmax partials in log2 units.
template <int E>
__device__ __forceinline__ void merge_state(float& m, float& l, float (&a)[E], float m2, float l2, const float (&a2)[E]) {
  const float mn = fmaxf(m, m2);
  const float mu = (mn == -INFINITY) ? 0.f : mn;
  const float c1 = ex2_approx(m - mu);
  const float c2 = ex2_approx(m2 - mu);
  l = l * c1 + l2 * c2;
#pragma unroll
  for (int e = 0; e < E; ++e) a[e] = a[e] * c1 + a2[e] * c2;
  m = mn;
}

// Eight consecutive output elements a[e] * inv at element offset idx of o:
// bf16 (round to nearest even, one 16-byte store) or, in the fp32 output
// mode, the fp32 values themselves (two 16-byte stores).
template <int D>
__device__ __forceinline__ void store_o8(const DecodeParams& prm, size_t idx, const float (&a)[8], float inv) {
  if (prm.o_f32) {
    float4* d = reinterpret_cast<float4*>(static_cast<float*>(prm.o) + idx);
    d[0] = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
    d[1] = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
  } else {
    uint4 out;
    out.x = pack_bf16x2(a[0] * inv, a[1] * inv);
    out.y = pack_bf16x2(a[2] * inv, a[3] * inv);
    out.z = pack_bf16x2(a[4] * inv, a[5] * inv);
    out.w = pack_bf16x2(a[6] * inv, a[7] * inv);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.o) + idx) = out;
  }
}

// The end of every decode kernel: merge the NW warp states (m, l in log2 units,
// unnormalised o) of each query head in shared memory, then write o / lse
// (one split) or the split's partial, and let the last CTA of each (b, kv
// head) merge the partials (found through an atomic ticket, no waiting).
template <int D, int G, int NW>
__device__ __forceinline__ void decode_finish(const DecodeParams& prm, const float (&sm_m)[NW][G],
                                              const float (&sm_l)[NW][G], const float (&sm_acc)[NW][G][D],
                                              int* sm_last_p, int split, int kvh, int b) {
  constexpr int TPR = D / 8;
  int& sm_last = *sm_last_p;
  const int H = prm.H;
  const int h0 = kvh * G;
  // Combine the warps: thread t < G*TPR owns (head g, chunk c).
  const int ns = prm.ns;
  const int t = threadIdx.x;
  const bool owner = t < G * TPR;
  const int g = owner ? t / TPR : 0;
  const int c = t % TPR;
  const int h = h0 + g;
  float M = -INFINITY, Lsum = 0.f, A[8];
  if (owner) {
#pragma unroll
    for (int e = 0; e < 8; ++e) A[e] = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      float a2[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a2[e] = sm_acc[w][g][8 * c + e];
      merge_state<8>(M, Lsum, A, sm_m[w][g], sm_l[w][g], a2);
    }
  }
  if (ns == 1) {
    if (owner) {
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      store_o8<D>(prm, ((size_t)b * H + h) * D + 8 * c, A, inv);
      if (c == 0 && prm.lse != nullptr)
        prm.lse[(size_t)b * H + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
    }
    return;
  }

  // Split partial (normalised o, lse in log2 units).
  const size_t pidx = ((size_t)b * H + h) * ns + split;
  if (owner) {
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    float4* po = reinterpret_cast<float4*>(prm.part_o + pidx * D + 8 * c);
    po[0] = make_float4(A[0] * inv, A[1] * inv, A[2] * inv, A[3] * inv);
    po[1] = make_float4(A[4] * inv, A[5] * inv, A[6] * inv, A[7] * inv);
    if (c == 0) prm.part_lse[pidx] = Lsum > 0.f ? M + __log2f(Lsum) : -INFINITY;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int ticket = atomicAdd(&prm.tickets[(size_t)b * prm.Hkv + kvh], 1u);
    sm_last = (ticket == (unsigned int)(ns - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!sm_last) return;
  __threadfence();
  if (owner) {
    const size_t p0 = ((size_t)b * H + h) * ns;
    float Mx = -INFINITY;
    for (int s2 = 0; s2 < ns; ++s2) Mx = fmaxf(Mx, __ldcg(prm.part_lse + p0 + s2));
    const float mu = (Mx == -INFINITY) ? 0.f : Mx;
    float Ls = 0.f, Af[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) Af[e] = 0.f;
    for (int s2 = 0; s2 < ns; ++s2) {
      const float w = ex2_approx(__ldcg(prm.part_lse + p0 + s2) - mu);
      if (w == 0.f) continue;
      Ls += w;
      const float4* po = reinterpret_cast<const float4*>(prm.part_o + (p0 + s2) * D + 8 * c);
      const float4 x0 = __ldcg(po), x1 = __ldcg(po + 1);
      Af[0] = fmaf(w, x0.x, Af[0]);
      Af[1] = fmaf(w, x0.y, Af[1]);
      Af[2] = fmaf(w, x0.z, Af[2]);
      Af[3] = fmaf(w, x0.w, Af[3]);
      Af[4] = fmaf(w, x1.x, Af[4]);
      Af[5] = fmaf(w, x1.y, Af[5]);
      Af[6] = fmaf(w, x1.z, Af[6]);
      Af[7] = fmaf(w, x1.w, Af[7]);
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    store_o8<D>(prm, ((size_t)b * H + h) * D + 8 * c, Af, inv);
    if (c == 0 && prm.lse != nullptr)
      prm.lse[(size_t)b * H + h] = Ls > 0.f ? (Mx + __log2f(Ls)) * 0.69314718055994531f : -INFINITY;
  }
  if (threadIdx.x == 0) prm.tickets[(size_t)b * prm.Hkv + kvh] = 0u;
}

template <int D, int G, int U, bool PAGED>
__global__ void __launch_bounds__(128) lg_decode_kernel(const DecodeParams prm) {
  constexpr int TPR = D / 8;     // threads per cache row
  constexpr int RPW = 32 / TPR;  // rows per warp per step
  constexpr int NW = 4;
  constexpr int RSTEP = NW * RPW;
  __shared__ float sm_m[NW][G];
  __shared__ float sm_l[NW][G];
  __shared__ float sm_acc[NW][G][D];
  __shared__ int sm_last;

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int chunk = lane % TPR;
  const int slot = warp * RPW + lane / TPR;
  const int H = prm.H;
  const int h0 = kvh * G;

  int len = prm.lens[b];
  len = len < 0 ? 0 : (len > prm.Lmax ? prm.Lmax : len);
  const int r0 = split * prm.rows_per_split;
  const int r1 = min(len, r0 + prm.rows_per_split);

  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(prm.q);
  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 u = *reinterpret_cast<const uint4*>(q + ((size_t)b * H + h0 + g) * D + 8 * chunk);
    bf16x8_to_f32(u, qf[g]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] *= prm.scale_log2;
  }
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }

  const size_t row_stride = (size_t)prm.Hkv * D;  // elements between consecutive cache rows
  // Contiguous cache: rows of sequence b from row b * Lmax. Paged: from the pool's base.
  const size_t seq0 = PAGED ? 0 : (size_t)b * prm.Lmax * prm.Hkv * D;
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(prm.k_cache) + seq0 + (size_t)kvh * D + 8 * chunk;
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(prm.v_cache) + seq0 + (size_t)kvh * D + 8 * chunk;
  const int32_t* table = PAGED ? prm.block_table + (size_t)b * prm.max_blocks : nullptr;

  for (int base = r0; base < r1; base += RSTEP * U) {  // warp-uniform trip count
    uint4 kr[U], vr[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + slot + u * RSTEP;
      live[u] = row < r1;
      size_t off = (size_t)row * row_stride;
      if (PAGED && live[u]) {
        const int pg = __ldg(table + (row >> 6));
        if (pg < 0 || (long long)pg >= prm.num_pages) {
          if (prm.err != nullptr) atomicOr(prm.err, kErrPaged);
          live[u] = false;
        }
        off = ((size_t)pg * 64 + (row & 63)) * row_stride;
      }
      if (live[u]) {
        kr[u] = ld_stream_v4(kb + off);
        vr[u] = ld_stream_v4(vb + off);
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s[U];
      float smax = -INFINITY;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float kf[8];
        bf16x8_to_f32(kr[u], kf);
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) d = fmaf(qf[g][e], kf[e], d);
#pragma unroll
        for (int off = TPR / 2; off >= 1; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        s[u] = live[u] ? d : -INFINITY;
        smax = fmaxf(smax, s[u]);
      }
      const float mn = fmaxf(m[g], smax);
      const float mu = (mn == -INFINITY) ? 0.f : mn;
      const float alpha = ex2_approx(m[g] - mu);
      l[g] *= alpha;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float p = ex2_approx(s[u] - mu);
        float vf[8];
        bf16x8_to_f32(vr[u], vf);
        l[g] += p;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(p, vf[e], acc[g][e]);
      }
      m[g] = mn;
    }
  }

  // Combine the RPW row slots of this warp (lanes with the same chunk).
#pragma unroll
  for (int off = TPR; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m[g], off);
      const float l2 = __shfl_xor_sync(0xffffffffu, l[g], off);
      float a2[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a2[e] = __shfl_xor_sync(0xffffffffu, acc[g][e], off);
      merge_state<8>(m[g], l[g], acc[g], m2, l2, a2);
    }
  }
  if (lane < TPR) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (chunk == 0) {
        sm_m[warp][g] = m[g];
        sm_l[warp][g] = l[g];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_acc[warp][g][8 * chunk + e] = acc[g][e];
    }
  }
  __syncthreads();

  decode_finish<D, G, NW>(prm, sm_m, sm_l, sm_acc, &sm_last, split, kvh, b);
}

// ---------------------------------------------------------------------------
// Query-head groups (G = H / Hkv >= 2): the G query rows of a KV head make the
// decode a thin GEMM per block of cache rows, S = Q K^T and O += P V, so it
// runs on warp-level tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32
// accumulate) with the G heads on the M side (padded to 16). The scalar
// kernel above spends 4 shuffles and 16 redundant exponentials per (row,
// head) and falls to 0.2-0.5 of HBM bandwidth at G = 4-8.
// The CTA stages 64-row blocks of K and V in shared memory with cp.async
// (two stages, 16-byte chunks XOR-swizzled by row, zero-filled past the
// cache), so a whole block is in flight while the previous one is computed;
// warp w computes rows [16 w, 16 w + 16) of each block:
//   S (16 heads x 8 rows per MMA), K fragments by ldmatrix;
//   P: the S accumulators of two 8-row tiles are, element for element, the A
//     fragment of P for the next MMA;
//   O (16 heads x 8 d per MMA) += P V, V fragments by ldmatrix.trans.
// Each warp keeps an online softmax per head; the warps and the splits merge
// as in the scalar kernel, the warps' partial O passing through the (by then
// idle) K/V stages, so the CTA's shared memory is the stages alone (64 KB at
// D = 128: three CTAs per SM for every group size).
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(saddr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(saddr)
               : "memory");
}
// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D>
struct DecodeMmaLayout {
  static constexpr int NW = 4;                // warps; warp w owns rows [WR w, +WR) of a block
  static constexpr int BR = LG_DECODE_MMA_BR; // cache rows per block
  static constexpr int WR = BR / NW;          // rows per warp and block (a multiple of 16)
  static constexpr int ROWB = D * 2;          // bytes of one K or V row (one KV head)
  static constexpr int TILE = BR * ROWB;      // one K or V block
  static constexpr int NST = LG_DECODE_MMA_STAGES;  // K / V stages
  static constexpr int SMEM = NST * 2 * TILE;       // dynamic
};

template <int D, int G, bool PAGED>
__global__ void __launch_bounds__(128) lg_decode_mma_kernel(const DecodeParams prm) {
  using L = DecodeMmaLayout<D>;
  constexpr int NW = L::NW;
  constexpr int BR = L::BR;
  constexpr int KS = D / 16;  // k-steps of S
  constexpr int DT = D / 8;   // 8-column d tiles of O (one 16-byte chunk each)
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  static_assert(G >= 2 && G <= 8, "query heads per KV head");
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ float sm_m[NW][G];
  __shared__ float sm_l[NW][G];
  __shared__ int sm_last;
  static_assert(NW * G * D * 4 <= L::SMEM, "the warps' partial O fits the K/V stages");

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2;  // fragment row group: query heads gq, gq + 8
  const int tq = lane & 3;
  const int H = prm.H;
  const int h0 = kvh * G;

  int len = prm.lens[b];
  len = len < 0 ? 0 : (len > prm.Lmax ? prm.Lmax : len);
  const int r0 = split * prm.rows_per_split;
  const int r1 = min(len, r0 + prm.rows_per_split);

  // Q as A fragments (heads >= G are zero rows).
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(prm.q);
  uint32_t qa[KS][4];
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    const int d0 = 16 * kk + 2 * tq;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(q + ((size_t)b * H + h0 + gq) * D + d0);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(q + ((size_t)b * H + h0 + gq + 8) * D + d0);
    qa[kk][0] = gq < G ? q0[0] : 0u;
    qa[kk][1] = gq + 8 < G ? q1[0] : 0u;
    qa[kk][2] = gq < G ? q0[4] : 0u;  // d0 + 8
    qa[kk][3] = gq + 8 < G ? q1[4] : 0u;
  }

  const size_t row_stride = (size_t)prm.Hkv * D;
  const size_t seq0 = PAGED ? 0 : (size_t)b * prm.Lmax * prm.Hkv * D;
  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(prm.k_cache) + seq0 + (size_t)kvh * D;
  const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(prm.v_cache) + seq0 + (size_t)kvh * D;
  const int32_t* table = PAGED ? prm.block_table + (size_t)b * prm.max_blocks : nullptr;
  // Element offset of cache row r (-1: outside the cache or its page is not in the pool).
  auto row_off = [&](int r) -> long long {
    if (r >= r1) return -1;
    if (PAGED) {
      const int pg = __ldg(table + (r >> 6));
      if (pg < 0 || (long long)pg >= prm.num_pages) {
        if (prm.err != nullptr) atomicOr(prm.err, kErrPaged);
        return -1;
      }
      return (long long)(((size_t)pg * 64 + (r & 63)) * row_stride);
    }
    return (long long)((size_t)r * row_stride);
  };
  const uint32_t s0 = smem_u32(dsm);
  // Chunk c of row r of a block sits at r * ROWB + (c ^ (r & 7)) * 16.
  auto swz = [](int r, int c) -> uint32_t { return (uint32_t)(r * L::ROWB + ((c ^ (r & 7)) * 16)); };
  auto stage = [&](int blk, int st) {
    const uint32_t sk = s0 + (uint32_t)(st * 2 * L::TILE), sv = sk + (uint32_t)L::TILE;
#pragma unroll 4
    for (int c = threadIdx.x; c < BR * CPR; c += 128) {
      const int r = c / CPR, ch = c % CPR;
      const long long off = row_off(blk + r);
      const size_t src = (size_t)(off < 0 ? 0 : off) + 8 * ch;
      cp_async16(sk + swz(r, ch), kbase + src, off < 0 ? 0u : 16u);
      cp_async16(sv + swz(r, ch), vbase + src, off < 0 ? 0u : 16u);
    }
  };

  const float sl2 = prm.scale_log2;
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads gq, gq + 8 (l: this lane's columns)
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix and row this lane addresses

  constexpr int NST = L::NST;
  const int nblk = r1 > r0 ? (r1 - r0 + BR - 1) / BR : 0;
  // NST - 1 blocks in flight ahead of the one being computed; one commit group per block slot.
#pragma unroll
  for (int i = 0; i < NST - 1; ++i) {
    if (i < nblk) stage(r0 + BR * i, i);
    cp_async_commit();
  }
  for (int bi = 0; bi < nblk; ++bi) {
    const int blk = r0 + BR * bi;
    const int nx = bi + NST - 1;
    if (nx < nblk) stage(r0 + BR * nx, nx % NST);
    cp_async_commit();
    cp_async_wait<NST - 1>();  // block bi's group is complete (later ones may be pending)
    __syncthreads();           // every thread's copies of this block landed
    const uint32_t sk = s0 + (uint32_t)((bi % NST) * 2 * L::TILE), sv = sk + (uint32_t)L::TILE;
    constexpr int NJ = L::WR / 8;  // 8-row tiles per warp and block
    const int wr = L::WR * warp;   // this warp's first row in the block

    // ---- S = Q K^T: NJ tiles of 8 rows; ldmatrix matrices {rows n0..+7} x {d chunk 2kk, 2kk+1}
    float sc[NJ][4];
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j][e] = 0.f;
#pragma unroll
    for (int jp = 0; jp < NJ / 2; ++jp) {
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        // matrices: 0 = tile 2jp, chunk 2kk; 1 = tile 2jp, chunk 2kk+1; 2, 3 = tile 2jp+1
        const int row = wr + 8 * (2 * jp + (mi >> 1)) + rr;
        uint32_t b00, b01, b10, b11;
        ldsm_x4(sk + swz(row, 2 * kk + (mi & 1)), b00, b01, b10, b11);
        mma_16816_bf16(sc[2 * jp], qa[kk], b00, b01);
        mma_16816_bf16(sc[2 * jp + 1], qa[kk], b10, b11);
      }
    }

    // ---- online softmax per head (log2 units); rows past the cache are -inf
    float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = blk + wr + 8 * j + 2 * tq + (e & 1);
        const bool ok = r < r1 && (!PAGED || row_off(r) >= 0);
        sc[j][e] = ok ? sc[j][e] * sl2 : -INFINITY;
      }
      bm0 = fmaxf(bm0, fmaxf(sc[j][0], sc[j][1]));
      bm1 = fmaxf(bm1, fmaxf(sc[j][2], sc[j][3]));
    }
    bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 1));
    bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 2));
    bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 1));
    bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 2));
    const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2_approx(m0 - mu0), al1 = ex2_approx(m1 - mu1);
    m0 = mn0;
    m1 = mn1;
    l0 *= al0;
    l1 *= al1;
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      o[i][0] *= al0;
      o[i][1] *= al0;
      o[i][2] *= al1;
      o[i][3] *= al1;
    }
    uint32_t pa[NJ / 2][4];  // P as A fragments, one per 16-row k-step
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float p0 = ex2_approx(sc[j][0] - mu0), p1 = ex2_approx(sc[j][1] - mu0);
      const float p2 = ex2_approx(sc[j][2] - mu1), p3 = ex2_approx(sc[j][3] - mu1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      pa[j >> 1][2 * (j & 1) + 0] = pack_bf16x2(p0, p1);
      pa[j >> 1][2 * (j & 1) + 1] = pack_bf16x2(p2, p3);
    }

    // ---- O += P V; ldmatrix.trans matrices {rows r16 half} x {d tile}
#pragma unroll
    for (int r16 = 0; r16 < NJ / 2; ++r16) {
      const int row = wr + 16 * r16 + 8 * (mi & 1) + rr;
#pragma unroll
      for (int dp = 0; dp < DT / 2; ++dp) {
        uint32_t b00, b01, b10, b11;
        ldsm_x4_trans(sv + swz(row, 2 * dp + (mi >> 1)), b00, b01, b10, b11);
        mma_16816_bf16(o[2 * dp], pa[r16], b00, b01);
        mma_16816_bf16(o[2 * dp + 1], pa[r16], b10, b11);
      }
    }
    __syncthreads();  // the stage may be refilled once every warp has read it
  }

  // Every copy has landed and every warp is past its last read of the
  // stages (the loop ends on a barrier): they now hold the warps' partial O.
  cp_async_wait<0>();
  __syncthreads();
  float(&sm_acc)[NW][G][D] = *reinterpret_cast<float(*)[NW][G][D]>(dsm);
  // Row sums over the four lanes of a fragment row group.
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (gq < G) {
    if (tq == 0) {
      sm_m[warp][gq] = m0;
      sm_l[warp][gq] = l0;
    }
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      sm_acc[warp][gq][8 * i + 2 * tq] = o[i][0];
      sm_acc[warp][gq][8 * i + 2 * tq + 1] = o[i][1];
    }
  }
  if (gq + 8 < G) {
    if (tq == 0) {
      sm_m[warp][gq + 8] = m1;
      sm_l[warp][gq + 8] = l1;
    }
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      sm_acc[warp][gq + 8][8 * i + 2 * tq] = o[i][2];
      sm_acc[warp][gq + 8][8 * i + 2 * tq + 1] = o[i][3];
    }
  }
  __syncthreads();
  decode_finish<D, G, NW>(prm, sm_m, sm_l, sm_acc, &sm_last, split, kvh, b);
}

template <int D, int G>
static cudaError_t launch_decode_dg(const DecodeParams& prm, cudaStream_t stream) {
  constexpr int U = (G <= 2) ? 4 : 2;
  dim3 grid(prm.ns, prm.Hkv, prm.B);
  if constexpr (G >= 2) {  // query-head groups: the tensor-core kernel
    constexpr int SM = DecodeMmaLayout<D>::SMEM;
    cudaError_t e;
    if (prm.block_table != nullptr) {
      e = cudaFuncSetAttribute(lg_decode_mma_kernel<D, G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM);
      if (e != cudaSuccess) return e;
      lg_decode_mma_kernel<D, G, true><<<grid, 128, SM, stream>>>(prm);
    } else {
      e = cudaFuncSetAttribute(lg_decode_mma_kernel<D, G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM);
      if (e != cudaSuccess) return e;
      lg_decode_mma_kernel<D, G, false><<<grid, 128, SM, stream>>>(prm);
    }
    return cudaGetLastError();
  } else {
    if (prm.block_table != nullptr)
      lg_decode_kernel<D, G, U, true><<<grid, 128, 0, stream>>>(prm);
    else
      lg_decode_kernel<D, G, U, false><<<grid, 128, 0, stream>>>(prm);
    return cudaGetLastError();
  }
}

template <int D>
static cudaError_t launch_decode_d(int G, const DecodeParams& prm, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_decode_dg<D, 1>(prm, stream);
    case 2: return launch_decode_dg<D, 2>(prm, stream);
    case 4: return launch_decode_dg<D, 4>(prm, stream);
    case 8: return launch_decode_dg<D, 8>(prm, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode(int D, int G, const DecodeParams& prm, cudaStream_t stream) {
  if (D == 64) return launch_decode_d<64>(G, prm, stream);
  return launch_decode_d<128>(G, prm, stream);
}

}  // namespace lg
