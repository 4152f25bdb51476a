// decode.cu -- single-token decode over the (reduced) KV cache, split-KV with an
// in-launch log-sum-exp merge.
//
// "A Little Goes a Long Way" (LongGen), Abstract (GPU-friendly KV cache
// reduction) and the atlas.scime.ai summary, "Key results" (KV cache 69.2 GB ->
// 26.5 GB, 1.41x decoding): a sparse layer's cache holds only the rows its
// static pattern can still reach, a full layer's holds all of them; decode is
// one query row attending to every cached row, so it is a pure HBM stream.
//
// Grid (splits, Hkv, B), 128 threads. D/8 threads share one cache row (16 B
// each, one non-allocating vector load for K and one for V); a warp covers
// 32*8/D rows per step and U steps are unrolled so each thread has 2*U loads
// in flight. All G = H/Hkv query heads of a KV head are served by the same
// CTA, so K/V bytes are read once per KV head. Each CTA reduces its rows to a
// partial (o, lse); with more than one split the last CTA of each (b, kv head)
// -- found through an atomic ticket, with no waiting -- merges the partials.
//
// Paged caches (PAGED = true): cache row r of sequence b lives in page
// block_table[b][r / 64] at page row r % 64, every page [64, Hkv, D]; a page
// index outside the pool is reported (kErrPaged) and its rows are skipped.
#include "lg_common.cuh"
#include "lg_kernels.h"

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
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(prm.o);
  if (ns == 1) {
    if (owner) {
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      uint4 out;
      out.x = pack_bf16x2(A[0] * inv, A[1] * inv);
      out.y = pack_bf16x2(A[2] * inv, A[3] * inv);
      out.z = pack_bf16x2(A[4] * inv, A[5] * inv);
      out.w = pack_bf16x2(A[6] * inv, A[7] * inv);
      *reinterpret_cast<uint4*>(o + ((size_t)b * H + h) * D + 8 * c) = out;
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
    uint4 out;
    out.x = pack_bf16x2(Af[0] * inv, Af[1] * inv);
    out.y = pack_bf16x2(Af[2] * inv, Af[3] * inv);
    out.z = pack_bf16x2(Af[4] * inv, Af[5] * inv);
    out.w = pack_bf16x2(Af[6] * inv, Af[7] * inv);
    *reinterpret_cast<uint4*>(o + ((size_t)b * H + h) * D + 8 * c) = out;
    if (c == 0 && prm.lse != nullptr)
      prm.lse[(size_t)b * H + h] = Ls > 0.f ? (Mx + __log2f(Ls)) * 0.69314718055994531f : -INFINITY;
  }
  if (threadIdx.x == 0) prm.tickets[(size_t)b * prm.Hkv + kvh] = 0u;
}

template <int D, int G>
static cudaError_t launch_decode_dg(const DecodeParams& prm, cudaStream_t stream) {
  constexpr int U = (G <= 2) ? 4 : 2;
  dim3 grid(prm.ns, prm.Hkv, prm.B);
  if (prm.block_table != nullptr)
    lg_decode_kernel<D, G, U, true><<<grid, 128, 0, stream>>>(prm);
  else
    lg_decode_kernel<D, G, U, false><<<grid, 128, 0, stream>>>(prm);
  return cudaGetLastError();
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
