// fwd_sm100.cu -- LongGen sparse causal attention, prefill forward, for sm_100a.
//
// "A Little Goes a Long Way" (LongGen): Abstract insights 1-2 (sink / window /
// strided-block sparse layers, full-attention middle layers) and the
// atlas.scime.ai summary, "Approach" (static block-wise access, exact
// FlashAttention-2-style attention). For each (b, h, 128-row query tile) the
// CTA walks the union of the KV-block lists of the tile's two 64-row query
// blocks, computes S = Q K^T and O += P V on the tcgen05 tensor cores with the
// accumulators in TMEM, and keeps an online softmax per row.
//
// CTA = 6 warps:
//   warps 0-3  softmax + epilogue; thread r owns query row r of the tile, which
//              is TMEM lane r (a warp may only touch its own 32-lane quarter);
//   warp 4     TMA producer (Q once, then K/V blocks through a 3-stage ring);
//   warp 5     TMEM allocation and the single MMA-issuing thread.
// TMEM columns: O [0, D), S double buffer [D, D + 128).
// Shared memory (128B-swizzled, as TMA writes it): Q [128 x D], K/V stages
// [64 x D], P double buffer [128 x 64] bf16.
// The MMA thread issues QK(n+1) before PV(n) so the tensor core works on the
// next block while the softmax warps finish the current one. O is rescaled
// lazily, only when a row's running max grows by more than 2^8.
#include "lg_common.cuh"
#include "lg_pattern.cuh"
#include "lg_kernels.h"

namespace lg {

template <int D>
struct FwdLayout {
  static constexpr int DP = D / 64;  // 64-element (128-byte) panels per row
  static constexpr int NS = 3;       // K/V ring depth
  static constexpr int Q_BYTES = 128 * D * 2;
  static constexpr int KV_BYTES = 64 * D * 2;
  static constexpr int P_BYTES = 128 * 64 * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int NBAR = 1 + 4 * NS + 8;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1024 bytes
  static constexpr uint32_t TMEM_COLS = 256;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    lg_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams prm) {
  using L = FwdLayout<D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + NS;
  uint64_t* v_full = bars + 1 + 2 * NS;
  uint64_t* v_empty = bars + 1 + 3 * NS;
  uint64_t* s_full = bars + 1 + 4 * NS;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* pv_done = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = prm.nqt - 1 - (int)blockIdx.x;  // heaviest (latest) tiles first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int kvh = h / (prm.H / prm.Hkv);
  const int i_lo = 2 * tile;
  const int i_hi = imin(2 * tile + 1, prm.nqb - 1);
  const KvIter it(prm.pat, i_lo, i_hi);
  const int N = it.count();
  unsigned int* err = prm.err;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 128);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, L::Q_BYTES);
      for (int p = 0; p < L::DP; ++p)
        tma_load_4d(smem + L::OFF_Q + p * 16384, &tmQ, q_full, 64 * p, h, 128 * tile, b);
      int n = 0;
      bool ok = true;
      for (int j = it.first(); j >= 0 && ok; j = it.next(j), ++n) {
        const int st = n % NS;
        const uint32_t use = (uint32_t)(n / NS);
        if (use > 0 && !mbar_wait(&k_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[st], L::KV_BYTES);
        for (int p = 0; p < L::DP; ++p)
          tma_load_4d(smem + L::OFF_K + st * L::KV_BYTES + p * 8192, &tmK, &k_full[st], 64 * p, kvh, 64 * j, b);
        if (use > 0 && !mbar_wait(&v_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[st], L::KV_BYTES);
        for (int p = 0; p < L::DP; ++p)
          tma_load_4d(smem + L::OFF_V + st * L::KV_BYTES + p * 8192, &tmV, &v_full[st], 64 * p, kvh, 64 * j, b);
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA's shared memory goes away.
        for (int s = 0; s < NS && s < n; ++s) {
          const int last = n - 1 - ((n - 1 - s) % NS);
          const uint32_t u = (uint32_t)(last / NS);
          const long long t0 = clock64();
          while (!(mbar_try_wait(&k_full[s], u & 1) && mbar_try_wait(&v_full[s], u & 1)) &&
                 clock64() - t0 < 20000000LL) {
          }
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, kErrFwdWait);
      tc_fence_after();
      auto issue_qk = [&](int n) -> bool {
        const int st = n % NS;
        const uint32_t use = (uint32_t)(n / NS);
        const int sb = n & 1;
        const uint32_t su = (uint32_t)(n >> 1);
        if (!mbar_wait(&k_full[st], use & 1, abort_flag, err, kErrFwdWait)) return false;
        if (n >= 2 && !mbar_wait(&s_empty[sb], (su - 1) & 1, abort_flag, err, kErrFwdWait)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(D + 64 * sb);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a = sbase + L::OFF_Q + (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t bb = sbase + L::OFF_K + st * L::KV_BYTES + (kk >> 2) * 8192 + (kk & 3) * 32;
          tc_mma_ss(d_tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        tc_commit(&k_empty[st]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int n = 0; n < N && ok; ++n) {
        if (n + 1 < N && !issue_qk(n + 1)) break;
        const int st = n % NS;
        const uint32_t use = (uint32_t)(n / NS);
        const int sb = n & 1;
        const uint32_t su = (uint32_t)(n >> 1);
        if (!mbar_wait(&p_full[sb], su & 1, abort_flag, err, kErrFwdWait)) break;
        if (!mbar_wait(&v_full[st], use & 1, abort_flag, err, kErrFwdWait)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t a = sbase + L::OFF_P + sb * L::P_BYTES + kk * 32;
          const uint32_t bb = sbase + L::OFF_V + st * L::KV_BYTES + kk * 2048;
          tc_mma_ss(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), idesc_pv,
                    (n > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[sb]);
        tc_commit(&v_empty[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = threadIdx.x;  // tile row == TMEM lane
    const int half = r >> 6;
    const int rr = r & 63;
    const int i = 2 * tile + half;
    const bool row_live = i < prm.nqb;
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = prm.scale_log2;
    float m = -INFINITY;  // running max in log2 units of the scaled scores
    float l = 0.f;
    int n = 0;
    for (int j = it.first(); j >= 0; j = it.next(j), ++n) {
      const int sb = n & 1;
      const uint32_t su = (uint32_t)(n >> 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], su & 1, abort_flag, err, kErrFwdWait))) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld64(t_lane + (uint32_t)(D + 64 * sb), sr);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);

      float x[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(sr[c]);
      const bool vis = row_live && in_list(prm.pat, i, j);
      if (!vis) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = -INFINITY;
      } else if (j == i) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c > rr) x[c] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < 64; ++c) mx = fmaxf(mx, x[c]);
      const float m_blk = mx * sl2;
      const bool need = m_blk > m + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m - m_blk);
        m = m_blk;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      uint32_t pk[32];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2_approx(fmaf(x[c], sl2, -m_use));
        const float p1 = ex2_approx(fmaf(x[c + 1], sl2, -m_use));
        rs += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + rs;

      // P buffer sb is free once PV(n-2) has completed.
      if (n >= 2 &&
          !__all_sync(0xffffffffu, mbar_wait(&pv_done[sb], (su - 1) & 1, abort_flag, err, kErrFwdWait)))
        break;
      const uint32_t prow = sbase + L::OFF_P + sb * L::P_BYTES;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(prow + sw128_offset(r, c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_async_smem();

      // Lazy rescale of O (warp-uniform because tcgen05.ld/st are warp-collective).
      if (__any_sync(0xffffffffu, need && n > 0)) {
        const int pb = (n - 1) & 1;
        const uint32_t pu = (uint32_t)((n - 1) >> 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[pb], pu & 1, abort_flag, err, kErrFwdWait))) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(t_lane + (uint32_t)(32 * ch), o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_lane + (uint32_t)(32 * ch), o);
        }
      }
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }

    // ------------------------------------------------------------ epilogue
    bool ok = (n == N) && !*abort_flag;
    if (ok) {
      const int lb = (N - 1) & 1;
      const uint32_t lu = (uint32_t)((N - 1) >> 1);
      ok = mbar_wait(&pv_done[lb], lu & 1, abort_flag, err, kErrFwdWait);
    }
    ok = __all_sync(0xffffffffu, ok);
    const int srow = 128 * tile + r;
    if (ok && prm.o_f32 != nullptr) {
      // fp32 output: each thread stores its row straight from TMEM.
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      float* dst = prm.o_f32 + (((size_t)b * prm.S + srow) * prm.H + h) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(t_lane + (uint32_t)(32 * ch), o);
        if (row_live && srow < prm.S) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * ch);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
        }
      }
    } else if (ok) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(t_lane + (uint32_t)(32 * ch), o);
        const uint32_t panel = sbase + L::OFF_Q + (uint32_t)((32 * ch) >> 6) * 16384;
        const int c0 = ((32 * ch) & 63) >> 3;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float* f = reinterpret_cast<const float*>(&o[8 * q4]);
          st_shared_v4(panel + sw128_offset(r, c0 + q4), pack_bf16x2(f[0] * inv_l, f[1] * inv_l),
                       pack_bf16x2(f[2] * inv_l, f[3] * inv_l), pack_bf16x2(f[4] * inv_l, f[5] * inv_l),
                       pack_bf16x2(f[6] * inv_l, f[7] * inv_l));
        }
      }
    }
    if (ok && prm.lse != nullptr && row_live && srow < prm.S) {
      const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      prm.lse[((size_t)b * prm.H + h) * prm.S + srow] = lse;
    }
    fence_async_smem();
    named_bar_sync(1, 128);
    if (r == 0 && !*abort_flag && prm.o_f32 == nullptr) {
      for (int p = 0; p < L::DP; ++p) tma_store_4d(&tmO, smem + L::OFF_Q + p * 16384, 64 * p, h, 128 * tile, b);
      bulk_commit();
      bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                            const FwdParams& prm, int B, cudaStream_t stream) {
  using L = FwdLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(lg_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(prm.nqt, prm.H, B);
  lg_fwd_kernel<D><<<grid, 192, L::ALLOC, stream>>>(tq, tk, tv, to, prm);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream) {
  if (D == 64) return launch_fwd_impl<64>(tq, tk, tv, to, prm, B, stream);
  return launch_fwd_impl<128>(tq, tk, tv, to, prm, B, stream);
}

}  // namespace lg
