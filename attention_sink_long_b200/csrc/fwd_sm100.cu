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
// KV blocks are consumed in chunks of two consecutive listed blocks (KvChunks;
// adjacent or not, each 64-row half loaded by its own TMA copy), so the MMAs
// run with N = 128 (S) and K = 128 (PV) on every pattern term.
//
// CTA = 10 warps, two 128-row query tiles that share every K/V chunk:
//   warps 0-3 / 4-7  softmax + epilogue of tile 0 / tile 1; thread r of a group
//                    owns row r of its tile, which is TMEM lane r (a warp may
//                    only touch its own 32-lane quarter);
//   warp 8           TMA producer (both Q tiles once, then K/V chunks through a
//                    two-stage ring);
//   warp 9           TMEM allocation and the single MMA-issuing thread.
// TMEM columns: O of tile t at [t*D, (t+1)*D); S of tile t at 2D + 128t
// (128 columns). The softmax writes P back over the first 64 columns of its S
// (bf16, two per column) and the PV product reads it from there (A operand in
// TMEM), so P never touches shared memory.
// The MMA thread ping-pongs the tiles: PV_0(c), S_0(c+1), PV_1(c), S_1(c+1) --
// the tensor core runs one tile's GEMMs while the other tile's softmax works.
// Issue order also protects the P/S aliasing: S_t(c+1) is issued after
// PV_t(c), and tcgen05 MMAs of one thread execute in order. When a tile's
// softmax sees S_t(c) complete, PV_t(c-1) is complete too (same commit), so O
// can be rescaled right away. O is rescaled lazily, only when a row's running
// max grows by more than 2^8.
#include "lg_common.cuh"
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

// F8: Q and K in fp8 e4m3 (S = Q K^T on the fp8 tensor-core path, K = 32 per
// MMA; head dim 128 only, one 128-byte panel per row); V, P and O as in bf16.
template <int D, bool F8 = false>
struct FwdLayout {
  static constexpr int DP = D / 64;              // 64-element (128-byte) bf16 panels per row
  static constexpr int NT = 2;                   // 128-row query tiles per CTA
  static constexpr int NS = 2;                   // K/V chunk stages
  static constexpr int QK_ELEM = F8 ? 1 : 2;     // bytes per Q / K element
  static constexpr int Q_BYTES = 128 * D * QK_ELEM;   // one query tile
  static constexpr int K_BYTES = 128 * D * QK_ELEM;   // one K chunk (up to 128 rows)
  static constexpr int KVC_BYTES = 128 * D * 2;       // one V chunk
  static constexpr int OFF_Q = 0;                // NT tiles
  static constexpr int OFF_K = OFF_Q + NT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * KVC_BYTES;
  // The bf16 O tile of query tile t is staged at OFF_Q + t * O_STAGE for its
  // TMA store: the Q tiles (and with F8 the K stages) are free by then.
  static constexpr int O_STAGE = 128 * D * 2;
  static_assert(NT * O_STAGE <= OFF_V, "O staging must fit in the Q / K area");
  static constexpr int NBAR = 1 + 3 * NS + NT * 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1024 bytes
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 2 * D;
  static constexpr int THREADS = 320;
};

template <int D, bool F8>
__global__ void __launch_bounds__(FwdLayout<D, F8>::THREADS, 1)
    lg_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams prm) {
  using L = FwdLayout<D, F8>;
  static_assert(!F8 || D == 128, "fp8 Q/K: head dim 128");
  constexpr int NS = L::NS;
  constexpr int NT = L::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + NS;
  uint64_t* kv_empty = bars + 1 + 2 * NS;
  uint64_t* tile_bars = bars + 1 + 3 * NS;  // per tile: s_full, p_full, pv_done, p_half
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Spans vary fastest in launch order, from the last (heaviest under a causal
  // mask) to the first; CTAs running together share one head's K/V in L2.
  const int span = prm.nqt - 1 - (int)blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int kvh = h / (prm.H / prm.Hkv);
  // Sequence b occupies rows [base, base + len) at tensor-map batch coordinate
  // bc: the (B, S) layout, or the packed variable-length layout (one batch of
  // all rows) whose offsets come from cu_seqlens and are checked here; a bad
  // list is reported and its sequence skipped, never read out of bounds.
  int len = prm.S, base = 0, bc = b;
  long long lin0 = (long long)b * prm.S;  // linear row of the sequence's first row
  if (prm.cu_seqlens != nullptr) {
    const int s0 = prm.cu_seqlens[b], s1 = prm.cu_seqlens[b + 1];
    if (s0 < 0 || s1 < s0 || ((s1 - s0) & 63) != 0 || s1 > prm.S || s1 - s0 > prm.max_len) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) atomicOr(prm.err, kErrVarlen);
      return;
    }
    len = s1 - s0;
    base = s0;
    bc = 0;
    lin0 = s0;
  }
  const int nqb = len / 64;
  if (span >= (len + 255) / 256) return;  // this span lies past a shorter sequence's end (uniform exit)
  const KvChunks chunks(prm.pat, 4 * span, imin(4 * span + 3, nqb - 1));
  unsigned int* err = prm.err;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < NT; ++t) {
      mbar_init(&tile_bars[4 * t + 0], 1);    // s_full
      mbar_init(&tile_bars[4 * t + 1], 128);  // p_full: all of P written (and the row state updated)
      mbar_init(&tile_bars[4 * t + 2], 1);    // pv_done
      mbar_init(&tile_bars[4 * t + 3], 128);  // p_half: O rescaled and P of the first 64 columns written
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
        for (int p = 0; p < (F8 ? 1 : L::DP); ++p)  // fp8: one 128-byte panel holds a whole row
          tma_load_4d(smem + L::OFF_Q + t * L::Q_BYTES + p * 16384, &tmQ, q_full, 64 * p, h,
                      base + 256 * span + 128 * t, bc);
      int c = 0;
      int nb = 1;
      for (int j = chunks.first(); j >= 0; ++c) {
        int j2 = -1;
        const int jn = chunks.span(j, &nb, &j2);
        const int st = c % NS;
        const uint32_t use = (uint32_t)(c / NS);
        if (use > 0 && !mbar_wait(&kv_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) break;
        mbar_arrive_expect_tx(&k_full[st], nb * 64 * D * L::QK_ELEM);
        for (int hb = 0; hb < nb; ++hb)
          for (int p = 0; p < (F8 ? 1 : L::DP); ++p)
            tma_load_4d(smem + L::OFF_K + st * L::K_BYTES + p * 16384 + hb * 8192, &tmK, &k_full[st], 64 * p, kvh,
                        base + 64 * (hb == 0 ? j : j2), bc);
        mbar_arrive_expect_tx(&v_full[st], nb * 64 * D * 2);
        for (int hb = 0; hb < nb; ++hb)
          for (int p = 0; p < L::DP; ++p)
            tma_load_4d(smem + L::OFF_V + st * L::KVC_BYTES + p * 16384 + hb * 8192, &tmV, &v_full[st], 64 * p, kvh,
                        base + 64 * (hb == 0 ? j : j2), bc);
        j = jn;
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA's shared memory goes away.
        for (int s = 0; s < NS && s < c; ++s) {
          const int last = c - 1 - ((c - 1 - s) % NS);
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
    // The whole warp walks the schedule (uniform control flow); one elected
    // lane issues each MMA and commit.
    {
      const uint32_t leader = elect_one();
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      // Operand descriptors are formed once; per MMA only the start-address
      // field moves (it counts 16-byte units in bits [0, 14), and shared
      // addresses stay below 2^18, so a plain add never carries out of it).
      // Keeping the issue path to a few integer adds per MMA matters: one
      // thread feeds the tensor core, which finishes an M128 N128 K16 MMA in
      // 64 cycles.
      const uint64_t dQ0 = sdesc_sw128(sbase + L::OFF_Q, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(sbase + L::OFF_K, 16, 1024);
      const uint64_t dV0 = sdesc_sw128(sbase + L::OFF_V, 16384, 1024);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, kErrFwdWait);
      tc_fence_after();
      // S_t(c) = Q_t K(c)^T, N = 64 * nb, into the tile's S columns.
      auto issue_s = [&](int c, int nb, int t) -> bool {
        const int st = c % NS;
        if (t == 0 && !mbar_wait(&k_full[st], (uint32_t)(c / NS) & 1, abort_flag, err, kErrFwdWait)) return false;
        tc_fence_after();
        const uint64_t a0 = dQ0 + (uint32_t)((t * L::Q_BYTES) >> 4);
        const uint64_t b0 = dK0 + (uint32_t)((st * L::K_BYTES) >> 4);
        const uint32_t d = tmem + L::T_S + 128 * t;
        if (F8) {
          // e4m3 x e4m3, fp32 accumulate: K = 32 per MMA, 32 bytes per k-step in the row's panel
          const uint32_t idesc = nb == 2 ? idesc_e4m3(128, 128) : idesc_e4m3(128, 64);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            tc_mma_f8_ss_if(leader, d, a0 + (uint32_t)(kk * 2), b0 + (uint32_t)(kk * 2), idesc, kk > 0 ? 1u : 0u);
        } else {
          const uint32_t idesc = nb == 2 ? idesc_bf16(128, 128, false, false) : idesc_bf16(128, 64, false, false);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            tc_mma_ss_if(leader, d, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit_if(leader, &tile_bars[4 * t + 0]);
        return true;
      };
      // O_t += P_t(c) V(c), K = 64 * nb, P from TMEM. The first 64 KV rows go
      // as soon as the softmax has written their P (p_half), the second 64
      // once the whole chunk is done (p_full), so half of PV overlaps the
      // softmax's second half.
      auto issue_pv = [&](int c, int nb, int t) -> bool {
        const int st = c % NS;
        if (!mbar_wait(&tile_bars[4 * t + 3], (uint32_t)c & 1, abort_flag, err, kErrFwdWait)) return false;
        if (t == 0 && !mbar_wait(&v_full[st], (uint32_t)(c / NS) & 1, abort_flag, err, kErrFwdWait)) return false;
        tc_fence_after();
        const uint64_t b0 = dV0 + (uint32_t)((st * L::KVC_BYTES) >> 4);
        const uint32_t d = tmem + (uint32_t)(t * D);
        const uint32_t a = tmem + L::T_S + 128 * t;
        const uint32_t acc0 = c > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts_if(leader, d, a + 8 * kk, b0 + (uint32_t)(kk * 2048 >> 4), idesc_pv, kk > 0 ? 1u : acc0);
        if (!mbar_wait(&tile_bars[4 * t + 1], (uint32_t)c & 1, abort_flag, err, kErrFwdWait)) return false;
        tc_fence_after();
        if (nb == 2) {
#pragma unroll
          for (int kk = 4; kk < 8; ++kk)
            tc_mma_ts_if(leader, d, a + 8 * kk, b0 + (uint32_t)(kk * 2048 >> 4), idesc_pv, 1u);
        }
        tc_commit_if(leader, &tile_bars[4 * t + 2]);
        return true;
      };
      int nb = 1;
      int j = chunks.first();
      int jx = -1;
      int jn = j >= 0 ? chunks.span(j, &nb, &jx) : -1;
      for (int t = 0; t < NT && ok && j >= 0; ++t) ok = issue_s(0, nb, t);
      for (int c = 0; j >= 0 && ok; ++c) {
        int nb_next = 1;
        const int jnn = jn >= 0 ? chunks.span(jn, &nb_next, &jx) : -1;
        for (int t = 0; t < NT && ok; ++t) {
          ok = issue_pv(c, nb, t);
          if (ok && jn >= 0) ok = issue_s(c + 1, nb_next, t);
        }
        if (!ok) break;
        tc_commit_if(leader, &kv_empty[c % NS]);
        j = jn;
        jn = jnn;
        nb = nb_next;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int t = warp >> 2;          // query tile of this warp group
    const int r = threadIdx.x & 127;  // tile row == TMEM lane
    const int i = 4 * span + 2 * t + (r >> 6);
    const int rr = r & 63;
    const bool row_live = i < nqb;
    uint64_t* s_full = &tile_bars[4 * t + 0];
    uint64_t* p_full = &tile_bars[4 * t + 1];
    uint64_t* pv_done = &tile_bars[4 * t + 2];
    uint64_t* p_half = &tile_bars[4 * t + 3];
    const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t t_o = t_lane + (uint32_t)(t * D);
    const uint32_t t_s = t_lane + L::T_S + (uint32_t)(128 * t);
    const float sl2 = prm.scale_log2;
    float m = -INFINITY;  // running max in log2 units of the scaled scores
    float l = 0.f;
    int c = 0;
    int nb = 1;
    for (int j = chunks.first(); j >= 0; ++c) {
      int j2 = -1;
      const int jn = chunks.span(j, &nb, &j2);
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, (uint32_t)c & 1, abort_flag, err, kErrFwdWait))) break;
      tc_fence_after();
      // One TMEM read of the whole chunk (128 columns, one wait), masked per
      // 64-column half (blocks outside this row's list, causality inside the
      // diagonal block); the row max, the exponentials and the packed P then
      // all come from registers.
      bool vis[2], diag[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int kb = hb == 0 ? j : j2;
        vis[hb] = hb < nb && row_live && in_list(prm.pat, i, kb);
        diag[hb] = (kb == i);
      }
      uint32_t xs[128];
      tmem_ld128(t_s, xs);
      // vis and diag are warp-uniform (a warp's rows share a query block). The
      // register values stay as loaded: masking is applied to the max and to
      // P, never written back.
      float mxh[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
        if (vis[hb] && !diag[hb]) {
#pragma unroll
          for (int e = 0; e < 64; e += 16)
#pragma unroll
            for (int q = 0; q < 8; ++q)
              m8[q] = max3f(m8[q], __uint_as_float(xs[64 * hb + e + q]), __uint_as_float(xs[64 * hb + e + 8 + q]));
        } else if (vis[hb]) {
#pragma unroll
          for (int e = 0; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], e > rr ? -INFINITY : __uint_as_float(xs[64 * hb + e]));
        }
        mxh[hb] = fmaxf(max3f(m8[0], m8[1], m8[2]), fmaxf(max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      const float mx = fmaxf(mxh[0], mxh[1]);
      const float m_blk = mx * sl2;
      const bool need = m_blk > m + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m - m_blk);
        m = m_blk;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      // Lazy rescale of O (warp-uniform: tcgen05.ld/st are warp-collective),
      // before any P of this chunk is handed to the tensor core. PV_t(c-1)
      // completed before S_t(c) did, so O is stable here.
      if (__any_sync(0xffffffffu, need && c > 0)) {
#pragma unroll 1
        for (int ch = 0; ch < D / 16; ++ch) {  // 16 columns at a time: the chunk's S is live
          uint32_t o[16];
          tmem_ld16(t_o + (uint32_t)(16 * ch), o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(t_o + (uint32_t)(16 * ch), o);
        }
      }
      // P = 2^(x * scale * log2 e - m), packed to bf16 and written back over the
      // first half of this tile's S columns (already read). All exponentials
      // run on the special-function unit (measured: moving a share of them to
      // an FMA-pipe polynomial made this kernel slower -- the softmax is bound
      // by instruction issue and latency, not by the special-function unit);
      // scaling and row sums run on paired fp32 instructions.
      const float2 sc2 = make_float2(sl2, sl2);
      const float2 nm2 = make_float2(-m_use, -m_use);
      float2 rs4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) rs4[e] = make_float2(0.f, 0.f);
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        if (hb < nb) {
          uint32_t pk[32];
          if (vis[hb] && !diag[hb]) {
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              const float2 a = fma2(make_float2(__uint_as_float(xs[64 * hb + e]), __uint_as_float(xs[64 * hb + e + 1])),
                                    sc2, nm2);
              const float2 pp = make_float2(ex2_approx(a.x), ex2_approx(a.y));
              rs4[(e >> 1) & 3] = add2(rs4[(e >> 1) & 3], pp);
              pk[e >> 1] = pack_bf16x2(pp.x, pp.y);
            }
          } else if (vis[hb]) {  // the diagonal block: P = 0 above the diagonal
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              const float2 a = fma2(make_float2(__uint_as_float(xs[64 * hb + e]), __uint_as_float(xs[64 * hb + e + 1])),
                                    sc2, nm2);
              const float2 pp = make_float2(e > rr ? 0.f : ex2_approx(a.x), e + 1 > rr ? 0.f : ex2_approx(a.y));
              rs4[(e >> 1) & 3] = add2(rs4[(e >> 1) & 3], pp);
              pk[e >> 1] = pack_bf16x2(pp.x, pp.y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = 0u;
          }
          tmem_st32(t_s + 32 * hb, pk);
        }
        if (hb == 0) {
          tc_fence_before();
          mbar_arrive(p_half);
        }
      }
      const float2 rs2 = add2(add2(rs4[0], rs4[1]), add2(rs4[2], rs4[3]));
      l = l * alpha + (rs2.x + rs2.y);

      tc_fence_before();
      mbar_arrive(p_full);
      j = jn;
    }
    const int NC = c;

    // ------------------------------------------------------------ epilogue
    bool ok = !*abort_flag && NC > 0;
    if (ok) ok = mbar_wait(pv_done, (uint32_t)(NC - 1) & 1, abort_flag, err, kErrFwdWait);
    ok = __all_sync(0xffffffffu, ok);
    const int row0 = 256 * span + 128 * t;  // first sequence row of this tile
    const int srow = row0 + r;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    if (ok && prm.o_f32 != nullptr) {
      // fp32 output: each thread stores its row straight from TMEM.
      tc_fence_after();
      float* dst = prm.o_f32 + ((size_t)(lin0 + srow) * prm.H + h) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(t_o + (uint32_t)(32 * ch), o);
        if (row_live && srow < len) {
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
        const uint32_t panel = sbase + L::OFF_Q + t * L::O_STAGE + (uint32_t)((32 * ch) >> 6) * 16384;
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
    if (ok && prm.lse != nullptr && row_live && srow < len) {
      const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t li = prm.cu_seqlens != nullptr ? (size_t)h * prm.S + (size_t)(base + srow)
                                                  : ((size_t)b * prm.H + h) * prm.S + srow;
      prm.lse[li] = lse;
    }
    fence_async_smem();
    named_bar_sync(1 + t, 128);
    if (r == 0 && !*abort_flag && prm.o_f32 == nullptr && row0 < len) {
      // One 64-row box per block inside the sequence: a box never reaches into
      // the next sequence of a packed batch.
      for (int hb = 0; hb < 2 && row0 + 64 * hb < len; ++hb)
        for (int p = 0; p < L::DP; ++p)
          tma_store_4d(&tmO, smem + L::OFF_Q + t * L::O_STAGE + p * 16384 + hb * 8192, 64 * p, h,
                       base + row0 + 64 * hb, bc);
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

template <int D, bool F8>
cudaError_t launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                            const FwdParams& prm, int B, cudaStream_t stream) {
  using L = FwdLayout<D, F8>;
  static_assert(L::ALLOC <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(lg_fwd_kernel<D, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(prm.nqt, prm.H, B);
  lg_fwd_kernel<D, F8><<<grid, L::THREADS, L::ALLOC, stream>>>(tq, tk, tv, to, prm);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream) {
  if (D == 64) return launch_fwd_impl<64, false>(tq, tk, tv, to, prm, B, stream);
  return launch_fwd_impl<128, false>(tq, tk, tv, to, prm, B, stream);
}

cudaError_t launch_fwd_fp8qk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const FwdParams& prm, int B, cudaStream_t stream) {
  return launch_fwd_impl<128, true>(tq, tk, tv, to, prm, B, stream);
}

}  // namespace lg
