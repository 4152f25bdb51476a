// fwd_sm100.cu -- LongGen sparse causal attention, prefill forward, for sm_100a.
//
// "A Little Goes a Long Way" (LongGen): Abstract insights 1-2 (sink / window /
// strided-block sparse layers, full-attention middle layers) and the
// atlas.scime.ai summary, "Approach" (static block-wise access, exact
// FlashAttention-2-style attention). For each (b, h, 256-row query span) the
// CTA walks the union of the KV-block lists of the span's four 64-row query
// blocks, computes S = Q K^T and O += P V on the tcgen05 tensor cores with the
// accumulators in TMEM, and keeps an online softmax per row.
//
// CTA = 10 warps, two 128-row query tiles that share every K/V block:
//   warps 0-3 / 4-7  softmax + epilogue of tile 0 / tile 1; thread r of a group
//                    owns row r of its tile, which is TMEM lane r (a warp may
//                    only touch its own 32-lane quarter);
//   warp 8           TMA producer (both Q tiles once, then K/V blocks through a
//                    ring of stages);
//   warp 9           TMEM allocation and the single MMA-issuing thread.
// TMEM columns: O of tile t at [t*D, (t+1)*D); S of tile t, buffer sb at
// 2D + 128t + 64sb (64 columns each).
// Shared memory (128B-swizzled, as TMA writes it): Q tiles [128 x D], K/V
// stages [64 x D], P double buffer per tile [128 x 64] bf16.
// Per KV block the MMA thread issues, per tile, QK(n+1) before PV(n) so the
// tensor core works on the next block while that tile's softmax finishes the
// current one; the two tiles interleave. O is rescaled lazily, only when a
// row's running max grows by more than 2^8.
#include "lg_common.cuh"
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

template <int D>
struct FwdLayout {
  static constexpr int DP = D / 64;               // 64-element (128-byte) panels per row
  static constexpr int NT = 2;                    // 128-row query tiles per CTA
  static constexpr int NS = (D == 128) ? 3 : 4;   // K/V ring depth
  static constexpr int Q_BYTES = 128 * D * 2;     // one query tile
  static constexpr int KV_BYTES = 64 * D * 2;     // one K or V block
  static constexpr int P_BYTES = 128 * 64 * 2;
  static constexpr int OFF_Q = 0;                 // NT tiles
  static constexpr int OFF_K = OFF_Q + NT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;  // NT tiles x 2 buffers
  static constexpr int OFF_BAR = OFF_P + NT * 2 * P_BYTES;
  static constexpr int NBAR = 1 + 4 * NS + NT * 8;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1024 bytes
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 2 * D;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    lg_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams prm) {
  using L = FwdLayout<D>;
  constexpr int NS = L::NS;
  constexpr int NT = L::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + NS;
  uint64_t* v_full = bars + 1 + 2 * NS;
  uint64_t* v_empty = bars + 1 + 3 * NS;
  uint64_t* tile_bars = bars + 1 + 4 * NS;  // per tile: s_full[2], s_empty[2], p_full[2], pv_done[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int span = prm.nqt - 1 - (int)blockIdx.x;  // heaviest (latest) spans first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int kvh = h / (prm.H / prm.Hkv);
  const int i_lo = 4 * span;
  const int i_hi = imin(4 * span + 3, prm.nqb - 1);
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
    for (int t = 0; t < NT; ++t) {
      uint64_t* tb = tile_bars + 8 * t;
      for (int s = 0; s < 2; ++s) {
        mbar_init(&tb[0 + s], 1);    // s_full
        mbar_init(&tb[2 + s], 128);  // s_empty
        mbar_init(&tb[4 + s], 128);  // p_full
        mbar_init(&tb[6 + s], 1);    // pv_done
      }
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, NT * L::Q_BYTES);
      for (int t = 0; t < NT; ++t)
        for (int p = 0; p < L::DP; ++p)
          tma_load_4d(smem + L::OFF_Q + t * L::Q_BYTES + p * 16384, &tmQ, q_full, 64 * p, h, 256 * span + 128 * t,
                      b);
      int n = 0;
      for (int j = it.first(); j >= 0; j = it.next(j), ++n) {
        const int st = n % NS;
        const uint32_t use = (uint32_t)(n / NS);
        if (use > 0 && !mbar_wait(&k_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) break;
        mbar_arrive_expect_tx(&k_full[st], L::KV_BYTES);
        for (int p = 0; p < L::DP; ++p)
          tma_load_4d(smem + L::OFF_K + st * L::KV_BYTES + p * 8192, &tmK, &k_full[st], 64 * p, kvh, 64 * j, b);
        if (use > 0 && !mbar_wait(&v_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) break;
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
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, kErrFwdWait);
      tc_fence_after();
      // S_t(n) = Q_t K(n)^T into the tile's S buffer n % 2.
      auto issue_qk = [&](int n, int t) -> bool {
        const int st = n % NS;
        const int sb = n & 1;
        const uint32_t su = (uint32_t)(n >> 1);
        uint64_t* tb = tile_bars + 8 * t;
        if (!mbar_wait(&k_full[st], (uint32_t)(n / NS) & 1, abort_flag, err, kErrFwdWait)) return false;
        if (n >= 2 && !mbar_wait(&tb[2 + sb], (su - 1) & 1, abort_flag, err, kErrFwdWait)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + L::T_S + (uint32_t)(128 * t + 64 * sb);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a = sbase + L::OFF_Q + t * L::Q_BYTES + (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t bb = sbase + L::OFF_K + st * L::KV_BYTES + (kk >> 2) * 8192 + (kk & 3) * 32;
          tc_mma_ss(d_tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(&tb[0 + sb]);
        return true;
      };
      // O_t += P_t(n) V(n).
      auto issue_pv = [&](int n, int t) -> bool {
        const int st = n % NS;
        const int sb = n & 1;
        uint64_t* tb = tile_bars + 8 * t;
        if (!mbar_wait(&tb[4 + sb], (uint32_t)(n >> 1) & 1, abort_flag, err, kErrFwdWait)) return false;
        if (!mbar_wait(&v_full[st], (uint32_t)(n / NS) & 1, abort_flag, err, kErrFwdWait)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t a = sbase + L::OFF_P + (2 * t + sb) * L::P_BYTES + kk * 32;
          const uint32_t bb = sbase + L::OFF_V + st * L::KV_BYTES + kk * 2048;
          tc_mma_ss(tmem + (uint32_t)(t * D), sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), idesc_pv,
                    (n > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&tb[6 + sb]);
        return true;
      };
      for (int t = 0; t < NT && ok; ++t) ok = issue_qk(0, t);
      if (ok && N > 0) tc_commit(&k_empty[0]);
      for (int n = 0; n < N && ok; ++n) {
        for (int t = 0; t < NT && ok; ++t) {
          if (n + 1 < N) ok = issue_qk(n + 1, t);
          if (ok) ok = issue_pv(n, t);
        }
        if (!ok) break;
        if (n + 1 < N) tc_commit(&k_empty[(n + 1) % NS]);
        tc_commit(&v_empty[n % NS]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int t = warp >> 2;                 // query tile of this warp group
    const int r = threadIdx.x & 127;         // tile row == TMEM lane
    const int i = 4 * span + 2 * t + (r >> 6);
    const int rr = r & 63;
    const bool row_live = i < prm.nqb;
    uint64_t* tb = tile_bars + 8 * t;
    const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t t_o = t_lane + (uint32_t)(t * D);
    const uint32_t t_s = t_lane + L::T_S + (uint32_t)(128 * t);
    const float sl2 = prm.scale_log2;
    float m = -INFINITY;  // running max in log2 units of the scaled scores
    float l = 0.f;
    int n = 0;
    for (int j = it.first(); j >= 0; j = it.next(j), ++n) {
      const int sb = n & 1;
      const uint32_t su = (uint32_t)(n >> 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&tb[0 + sb], su & 1, abort_flag, err, kErrFwdWait))) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld64(t_s + (uint32_t)(64 * sb), sr);
      tc_fence_before();
      mbar_arrive(&tb[2 + sb]);

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
      // Row max as a tree (short dependency chains keep the pipes busy).
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(x[e], x[e + 8]);
#pragma unroll
      for (int c = 16; c < 64; c += 8)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], x[c + e]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_blk = mx * sl2;
      const bool need = m_blk > m + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m - m_blk);
        m = m_blk;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      uint32_t pk[32];
      float rs8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) rs8[e] = 0.f;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2_approx(fmaf(x[c], sl2, -m_use));
        const float p1 = ex2_approx(fmaf(x[c + 1], sl2, -m_use));
        rs8[(c >> 1) & 7] += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      l = l * alpha + rs;

      // P buffer sb is free once PV(n-2) of this tile has completed.
      if (n >= 2 &&
          !__all_sync(0xffffffffu, mbar_wait(&tb[6 + sb], (su - 1) & 1, abort_flag, err, kErrFwdWait)))
        break;
      const uint32_t prow = sbase + L::OFF_P + (2 * t + sb) * L::P_BYTES;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(prow + sw128_offset(r, c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_async_smem();

      // Lazy rescale of O (warp-uniform because tcgen05.ld/st are warp-collective).
      if (__any_sync(0xffffffffu, need && n > 0)) {
        const int pb = (n - 1) & 1;
        const uint32_t pu = (uint32_t)((n - 1) >> 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&tb[6 + pb], pu & 1, abort_flag, err, kErrFwdWait))) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(t_o + (uint32_t)(32 * ch), o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_o + (uint32_t)(32 * ch), o);
        }
      }
      tc_fence_before();
      mbar_arrive(&tb[4 + sb]);
    }

    // ------------------------------------------------------------ epilogue
    bool ok = (n == N) && !*abort_flag;
    if (ok) {
      const int lb = (N - 1) & 1;
      const uint32_t lu = (uint32_t)((N - 1) >> 1);
      ok = mbar_wait(&tb[6 + lb], lu & 1, abort_flag, err, kErrFwdWait);
    }
    ok = __all_sync(0xffffffffu, ok);
    const int row0 = 256 * span + 128 * t;  // first sequence row of this tile
    const int srow = row0 + r;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    if (ok && prm.o_f32 != nullptr) {
      // fp32 output: each thread stores its row straight from TMEM.
      tc_fence_after();
      float* dst = prm.o_f32 + (((size_t)b * prm.S + srow) * prm.H + h) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(t_o + (uint32_t)(32 * ch), o);
        if (row_live && srow < prm.S) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * ch);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
        }
      }
    } else if (ok) {
      // bf16 output: stage the tile in its (no longer needed) Q buffer, then one TMA store.
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(t_o + (uint32_t)(32 * ch), o);
        const uint32_t panel = sbase + L::OFF_Q + t * L::Q_BYTES + (uint32_t)((32 * ch) >> 6) * 16384;
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
    named_bar_sync(1 + t, 128);
    if (r == 0 && !*abort_flag && prm.o_f32 == nullptr && row0 < prm.S) {
      for (int p = 0; p < L::DP; ++p)
        tma_store_4d(&tmO, smem + L::OFF_Q + t * L::Q_BYTES + p * 16384, 64 * p, h, row0, b);
      bulk_commit();
      bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                            const FwdParams& prm, int B, cudaStream_t stream) {
  using L = FwdLayout<D>;
  static_assert(L::ALLOC <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(lg_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(prm.nqt, prm.H, B);
  lg_fwd_kernel<D><<<grid, 320, L::ALLOC, stream>>>(tq, tk, tv, to, prm);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream) {
  if (D == 64) return launch_fwd_impl<64>(tq, tk, tv, to, prm, B, stream);
  return launch_fwd_impl<128>(tq, tk, tv, to, prm, B, stream);
}

}  // namespace lg
