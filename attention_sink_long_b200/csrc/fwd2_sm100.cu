// fwd2_sm100.cu -- LongGen sparse causal attention, prefill forward for head
// dim 128 (bf16), on a pair of CTAs that share 256-row tcgen05 MMAs.
//
// "A Little Goes a Long Way" (LongGen): Abstract insights 1-2 (sink / window /
// strided-block sparse layers, full-attention middle layers) and the
// atlas.scime.ai summary, "Approach" (static block-wise access, exact
// FlashAttention-2-style attention). The arithmetic per row is that of the
// single-CTA forward (fwd_sm100.cu): S = Q K^T per listed KV chunk, an online
// softmax with a lazy O rescale, O += P V, O / l and LSE = m + ln l.
//
// A cluster of two CTAs owns a 512-row query span (eight 64-row query blocks)
// of one head: CTA r holds rows 256 r .. 256 r + 255 as two 128-row tiles.
// Query tile t of the pair is CTA 0's tile t stacked on CTA 1's tile t, and
// every MMA is a cta_group::2 instruction with M = 256 issued by one thread of
// CTA 0: each CTA supplies its own 128 rows of A and receives its 128 rows of
// the accumulator in its own TMEM, and each supplies half of B:
//   S_t  = Q_t K^T   N = 128 KV rows: CTA 0 holds the chunk's first 64-row KV
//                    block (all 128 columns), CTA 1 the second;
//   O_t += P_t V     N = 128 columns of V: each CTA holds all 128 KV rows of
//                    the chunk, CTA r columns 64 r .. 64 r + 63.
// So each CTA loads half of every K/V chunk (32 KB instead of 64 KB) and the
// tensor core reads half of B from each CTA's shared memory.
//
// P goes to shared memory (bf16, the MMA's K-major 128-byte-swizzled layout)
// instead of over S in TMEM: the softmax releases S_t as soon as it has read
// it into registers, so S_t(c+1) runs on the tensor core while the softmax of
// chunk c computes its exponentials -- the MMA of the next chunk no longer
// waits behind P V of this one. The freed shared memory of the halved K/V
// chunks holds P.
//
// CTA = 10 warps (both CTAs alike):
//   warps 0-3 / 4-7  softmax + epilogue of tile 0 / tile 1 (thread r = tile
//                    row r = TMEM lane r);
//   warp 8           TMA producer: this CTA's two Q tiles, then its halves of
//                    the K/V chunks through three-stage K and V rings; every
//                    load counts on CTA 0's barrier (no multicast);
//   warp 9           TMEM allocation for the pair; in CTA 0 the MMA issuer.
// TMEM (both CTAs, same offsets): O_t at 128 t, S_t at 256 + 128 t.
// MMA order per chunk c: S_0(c+1), P_1(c-1) V, S_1(c+1), P_0(c) V (each S
// once the tile's softmax has read the previous S, each P V once its P is
// written). The two softmax warps of a lane quarter share an SM
// sub-partition; they take turns on its special-function unit through a
// token barrier, so one exponentiates while the other reads S, takes its row
// max and stores P (measured: in lockstep, both spent ~2300 of each ~4300
// cycles per chunk on exponentials at half rate).
// Barrier traffic between the CTAs: MMA completions arrive on both CTAs'
// barriers (tcgen05.commit multicast); the softmax warps of both CTAs arrive
// on CTA 0's "S read" and "P written" barriers (remote arrive). Each CTA's P
// rows are read by its own SM's share of the pair MMA, so a CTA-scope proxy
// fence and release order them before the arrive, and every wait acquires at
// CTA scope -- the pattern of CUTLASS's two-SM pipelines. (Cluster-scope
// release on every arrive and acquire on every poll stalled the softmax warps
// on memory barriers.)
#include "lg_common.cuh"
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

struct Fwd2Layout {
  static constexpr int D = 128;
  static constexpr int NT = 2;                   // 128-row query tiles per CTA
  static constexpr int NS = 3;                   // K and V stages
  static constexpr int Q_BYTES = 128 * 128 * 2;  // a query tile: two 64-column panels of 128 rows
  static constexpr int K_BYTES = 64 * 128 * 2;   // this CTA's K block of a chunk: two panels of 64 rows
  static constexpr int V_BYTES = 128 * 64 * 2;   // this CTA's V columns of a chunk: one panel of 128 rows
  static constexpr int P_BYTES = 128 * 128 * 2;  // P of a tile: two 64-column panels of 128 rows
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_P = OFF_V + NS * V_BYTES;
  static constexpr int OFF_BAR = OFF_P + NT * P_BYTES;  // 229376
  // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], per tile s_full, s_free, p_full, pv_done,
  // then the exponential-phase tokens tok[tile][lane quarter]
  static constexpr int NBAR = 1 + 4 * NS + 4 * NT + NT * 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = 232448;  // the per-block maximum
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 256;
  static constexpr int THREADS = 320;
  static_assert(NT * Q_BYTES >= NT * 128 * D * 2, "O staging must fit in the Q tiles");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Fwd2Layout::THREADS, 1)
    lg_fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const FwdParams prm) {
  using L = Fwd2Layout;
  constexpr int NS = L::NS;
  constexpr int NT = L::NT;
  constexpr int D = L::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Both CTAs run the same kernel image, so this check (and every early exit
  // below) takes the same branch in both: neither waits on a peer that left.
  if ((size_t)(smem - smem_raw) + (size_t)L::BYTES > (size_t)L::ALLOC) {
    if (threadIdx.x == 0) atomicOr(prm.err, kErrSmemFit);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the pair's MMAs

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + NS;
  uint64_t* v_full = bars + 1 + 2 * NS;
  uint64_t* v_empty = bars + 1 + 3 * NS;
  uint64_t* tile_bars = bars + 1 + 4 * NS;  // per tile: s_full, s_free, p_full, pv_done
  uint64_t* tok = tile_bars + 4 * NT;       // [tile][lane quarter]: that warp finished a chunk's exponentials
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair spans run from the last (heaviest under a causal mask) to the first.
  const int pspan = prm.nqt - 1 - (int)(blockIdx.x >> 1);
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int kvh = h / (prm.H / prm.Hkv);
  // Fixed-length batches: sequence b is batch coordinate b of the tensor maps.
  const int len = prm.S, base = 0, bc = b;
  const long long lin0 = (long long)b * prm.S;
  const int nqb = len / 64;
  if (pspan >= (len + 511) / 512) return;  // the span lies past a shorter sequence's end
  const int qb0 = 8 * pspan;               // first query block of the pair's span
  const KvChunks chunks(prm.pat, qb0, imin(qb0 + 7, nqb - 1));
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
      mbar_init(&tile_bars[4 * t + 0], 1);  // s_full: S_t in TMEM (commit, both CTAs)
      mbar_init(&tile_bars[4 * t + 1], 8);  // s_free: the 8 softmax warps of the tile read S_t (CTA 0)
      mbar_init(&tile_bars[4 * t + 2], 8);  // p_full: the 8 softmax warps wrote P_t (CTA 0)
      mbar_init(&tile_bars[4 * t + 3], 1);  // pv_done: P_t V completed (commit, both CTAs)
    }
    for (int e = 0; e < NT * 4; ++e) mbar_init(&tok[e], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA traffic
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // A lone block of an odd list: the odd CTA's K / V rows come from block nqb,
  // past the sequence (the tensor map fills them with zeros), and the softmax
  // gives them P = 0.
  const int pad_blk = nqb;

  if (warp == 8) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint32_t q_full_cl = mapa_shared(smem_u32(q_full), 0);
      if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * NT * L::Q_BYTES);
      for (int t = 0; t < NT; ++t)
        for (int p = 0; p < 2; ++p)
          tma_load_4d_pair(smem + L::OFF_Q + t * L::Q_BYTES + p * 16384, &tmQ, q_full_cl, 64 * p, h,
                           base + 512 * pspan + 256 * (int)rank + 128 * t, bc);
      int c = 0;
      int nb = 1;
      for (int j = chunks.first(); j >= 0; ++c) {
        int j2 = -1;
        const int jn = chunks.span(j, &nb, &j2);
        const int st = c % NS;
        const uint32_t use = (uint32_t)(c / NS);
        const int second = nb == 2 ? j2 : pad_blk;
        if (use > 0 && !mbar_wait(&k_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) break;
        if (rank == 0) mbar_arrive_expect_tx(&k_full[st], 2 * L::K_BYTES);
        const uint32_t kf_cl = mapa_shared(smem_u32(&k_full[st]), 0);
        for (int p = 0; p < 2; ++p)
          tma_load_4d_pair(smem + L::OFF_K + st * L::K_BYTES + p * 8192, &tmK, kf_cl, 64 * p, kvh,
                           base + 64 * (rank == 0 ? j : second), bc);
        if (use > 0 && !mbar_wait(&v_empty[st], (use - 1) & 1, abort_flag, err, kErrFwdWait)) break;
        if (rank == 0) mbar_arrive_expect_tx(&v_full[st], 2 * L::V_BYTES);
        const uint32_t vf_cl = mapa_shared(smem_u32(&v_full[st]), 0);
        for (int hb = 0; hb < 2; ++hb)
          tma_load_4d_pair(smem + L::OFF_V + st * L::V_BYTES + hb * 8192, &tmV, vf_cl, 64 * (int)rank, kvh,
                           base + 64 * (hb == 0 ? j : second), bc);
        j = jn;
      }
      if (*abort_flag) {
        // The copies count on CTA 0's barriers, which this CTA cannot poll:
        // give any copy still in flight time to land before shared memory goes.
        const long long t0 = clock64();
        while (clock64() - t0 < 20000000LL) {
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer (CTA 0 only)
    if (rank == 0) {
      const uint32_t leader = elect_one();
      constexpr uint32_t idesc_s = idesc_bf16(256, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(256, 128, false, true);
      // Descriptors are formed once; per MMA only the start-address field moves.
      const uint64_t dQ0 = sdesc_sw128(sbase + L::OFF_Q, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(sbase + L::OFF_K, 16, 1024);
      const uint64_t dV0 = sdesc_sw128(sbase + L::OFF_V, 16384, 1024);
      const uint64_t dP0 = sdesc_sw128(sbase + L::OFF_P, 16, 1024);
      // K-major 16-column step kk inside 64-column panels of `panel` bytes.
      auto kofs = [](int kk, int panel) -> uint32_t { return (uint32_t)(((kk >> 2) * panel + (kk & 3) * 32) >> 4); };
      auto issue_s = [&](int c, int t) {
        const uint64_t a0 = dQ0 + (uint32_t)((t * L::Q_BYTES) >> 4);
        const uint64_t b0 = dK0 + (uint32_t)(((c % NS) * L::K_BYTES) >> 4);
        const uint32_t d = tmem + L::T_S + 128 * t;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma2_ss_if(leader, d, a0 + kofs(kk, 16384), b0 + kofs(kk, 8192), idesc_s, kk > 0 ? 1u : 0u);
        tc_commit_pair_if(leader, &tile_bars[4 * t + 0], 3);
      };
      auto issue_pv = [&](int c, int t) {
        const uint64_t a0 = dP0 + (uint32_t)((t * L::P_BYTES) >> 4);
        const uint64_t b0 = dV0 + (uint32_t)(((c % NS) * L::V_BYTES) >> 4);
        const uint32_t d = tmem + (uint32_t)(128 * t);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma2_ss_if(leader, d, a0 + kofs(kk, 16384), b0 + (uint32_t)((kk * 2048) >> 4), idesc_pv,
                        (c > 0 || kk > 0) ? 1u : 0u);
        tc_commit_pair_if(leader, &tile_bars[4 * t + 3], 3);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, err, kErrFwdWait);
      int j = chunks.first();
      int nb = 1, jx = -1;
      int jn = j >= 0 ? chunks.span(j, &nb, &jx) : -1;
      if (ok && j >= 0) {
        ok = mbar_wait(&k_full[0], 0, abort_flag, err, kErrFwdWait);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          issue_s(0, 1);
          tc_commit_pair_if(leader, &k_empty[0], 3);
        }
      }
      // The tiles run half a chunk apart: per chunk c the issue order is
      // S_0(c+1), P_1(c-1) V, S_1(c+1), P_0(c) V -- the order in which the
      // tiles' softmax warps release S and hand over P once tile 1 trails
      // tile 0 by half a period, so one tile's exponentials overlap the other
      // tile's TMEM read and row max instead of competing for the
      // special-function unit.
      int c = 0;
      for (; j >= 0 && ok; ++c) {
        const uint32_t par = (uint32_t)c & 1;
        const int c1 = c + 1;
        if (jn >= 0) {
          ok = mbar_wait(&k_full[c1 % NS], (uint32_t)(c1 / NS) & 1, abort_flag, err, kErrFwdWait) &&
               mbar_wait(&tile_bars[4 * 0 + 1], par, abort_flag, err, kErrFwdWait);
          if (!ok) break;
          tc_fence_after();
          issue_s(c1, 0);
        }
        if (c > 0) {
          ok = mbar_wait(&tile_bars[4 * 1 + 2], par ^ 1u, abort_flag, err, kErrFwdWait);
          if (!ok) break;
          tc_fence_after();
          issue_pv(c - 1, 1);
          tc_commit_pair_if(leader, &v_empty[(c - 1) % NS], 3);
        }
        if (jn >= 0) {
          ok = mbar_wait(&tile_bars[4 * 1 + 1], par, abort_flag, err, kErrFwdWait);
          if (!ok) break;
          tc_fence_after();
          issue_s(c1, 1);
          tc_commit_pair_if(leader, &k_empty[c1 % NS], 3);
        }
        ok = mbar_wait(&v_full[c % NS], (uint32_t)(c / NS) & 1, abort_flag, err, kErrFwdWait) &&
             mbar_wait(&tile_bars[4 * 0 + 2], par, abort_flag, err, kErrFwdWait);
        if (!ok) break;
        tc_fence_after();
        issue_pv(c, 0);
        j = jn;
        int nbn = 1;
        jn = jn >= 0 ? chunks.span(jn, &nbn, &jx) : -1;
      }
      if (ok && c > 0) {  // P_1 V of the last chunk
        ok = mbar_wait(&tile_bars[4 * 1 + 2], (uint32_t)(c - 1) & 1, abort_flag, err, kErrFwdWait);
        if (ok) {
          tc_fence_after();
          issue_pv(c - 1, 1);
          tc_commit_pair_if(leader, &v_empty[(c - 1) % NS], 3);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-7 (both CTAs)
    const int t = warp >> 2;          // query tile of this warp group
    const int r = threadIdx.x & 127;  // tile row == TMEM lane
    const int i = qb0 + 4 * (int)rank + 2 * t + (r >> 6);
    const int rr = r & 63;
    const bool row_live = i < nqb;
    uint64_t* s_full = &tile_bars[4 * t + 0];
    uint64_t* pv_done = &tile_bars[4 * t + 3];
    const uint32_t s_free_cl = mapa_shared(smem_u32(&tile_bars[4 * t + 1]), 0);
    const uint32_t p_full_cl = mapa_shared(smem_u32(&tile_bars[4 * t + 2]), 0);
    const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t t_o = t_lane + (uint32_t)(128 * t);
    const uint32_t t_s = t_lane + L::T_S + (uint32_t)(128 * t);
    const uint32_t p_row = sbase + L::OFF_P + (uint32_t)(t * L::P_BYTES);
    // Warps w and w + 4 (tile 0 and tile 1 of lane quarter w) share one SM
    // sub-partition and its special-function unit; they take turns on it: the
    // tile-0 warp exponentiates chunk c after the tile-1 warp finished chunk
    // c - 1, the tile-1 warp after the tile-0 warp finished chunk c.
    uint64_t* tok_mine = &tok[4 * t + (warp & 3)];
    uint64_t* tok_other = &tok[4 * (t ^ 1) + (warp & 3)];
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
      uint32_t xs[128];
      tmem_ld128(t_s, xs);
      // S_t(c) is in registers: let the pair compute S_t(c+1) into these columns.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(s_free_cl);
      bool vis[2], diag[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int kb = hb == 0 ? j : j2;
        vis[hb] = hb < nb && row_live && in_list(prm.pat, i, kb);
        diag[hb] = (kb == i);
      }
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
      const float m_blk = fmaxf(mxh[0], mxh[1]) * sl2;
      const bool need = m_blk > m + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m - m_blk);
        m = m_blk;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      // P = 2^(x * scale * log2 e - m), packed to bf16 in registers -- on this
      // warp's turn of the special-function unit.
      if ((t == 1 || c > 0) &&
          !__all_sync(0xffffffffu, mbar_wait(tok_other, (uint32_t)(t == 0 ? c - 1 : c) & 1, abort_flag, err,
                                             kErrFwdWait)))
        break;
      const float2 sc2 = make_float2(sl2, sl2);
      const float2 nm2 = make_float2(-m_use, -m_use);
      float2 rs4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) rs4[e] = make_float2(0.f, 0.f);
      uint32_t pk[64];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        if (vis[hb] && !diag[hb]) {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float2 a = fma2(make_float2(__uint_as_float(xs[64 * hb + e]), __uint_as_float(xs[64 * hb + e + 1])),
                                  sc2, nm2);
            const float2 pp = make_float2(ex2_approx(a.x), ex2_approx(a.y));
            rs4[(e >> 1) & 3] = add2(rs4[(e >> 1) & 3], pp);
            pk[32 * hb + (e >> 1)] = pack_bf16x2(pp.x, pp.y);
          }
        } else if (vis[hb]) {  // the diagonal block: P = 0 above the diagonal
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float2 a = fma2(make_float2(__uint_as_float(xs[64 * hb + e]), __uint_as_float(xs[64 * hb + e + 1])),
                                  sc2, nm2);
            const float2 pp = make_float2(e > rr ? 0.f : ex2_approx(a.x), e + 1 > rr ? 0.f : ex2_approx(a.y));
            rs4[(e >> 1) & 3] = add2(rs4[(e >> 1) & 3], pp);
            pk[32 * hb + (e >> 1)] = pack_bf16x2(pp.x, pp.y);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[32 * hb + e] = 0u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(tok_mine);
      const float2 rs2 = add2(add2(rs4[0], rs4[1]), add2(rs4[2], rs4[3]));
      l = l * alpha + (rs2.x + rs2.y);
      // P_t(c-1) V has completed: its P buffer may be overwritten and O_t is stable.
      if (c > 0 && !__all_sync(0xffffffffu, mbar_wait(pv_done, (uint32_t)(c - 1) & 1, abort_flag, err,
                                                         kErrFwdWait)))
        break;
      tc_fence_after();
      // Lazy rescale of O (warp-uniform: tcgen05.ld/st are warp-collective).
      if (__any_sync(0xffffffffu, need && c > 0)) {
#pragma unroll 1
        for (int ch = 0; ch < D / 16; ++ch) {
          uint32_t o[16];
          tmem_ld16(t_o + (uint32_t)(16 * ch), o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(t_o + (uint32_t)(16 * ch), o);
        }
      }
      // P_t row r into the tile's two 64-column panels (128-byte swizzle).
#pragma unroll
      for (int hb = 0; hb < 2; ++hb)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(p_row + (uint32_t)(hb * 16384) + sw128_offset((uint32_t)r, (uint32_t)ch),
                       pk[32 * hb + 4 * ch], pk[32 * hb + 4 * ch + 1], pk[32 * hb + 4 * ch + 2],
                       pk[32 * hb + 4 * ch + 3]);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_full_cl);
      j = jn;
    }
    const int NC = c;

    // ------------------------------------------------------------ epilogue
    bool ok = !*abort_flag && NC > 0;
    if (ok) ok = mbar_wait(pv_done, (uint32_t)(NC - 1) & 1, abort_flag, err, kErrFwdWait);
    ok = __all_sync(0xffffffffu, ok);
    const int row0 = 512 * pspan + 256 * (int)rank + 128 * t;  // first sequence row of this tile
    const int srow = row0 + r;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    if (ok && prm.o_f32 != nullptr) {
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
      // bf16 output: stage the tile in its Q buffer (every S MMA of the tile has
      // completed), then 64-row TMA stores.
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
    if (ok && prm.lse != nullptr && row_live && srow < len) {
      const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t li = ((size_t)b * prm.H + h) * prm.S + srow;
      prm.lse[li] = lse;
    }
    fence_async_smem();
    named_bar_sync(1 + t, 128);
    if (r == 0 && ok && prm.o_f32 == nullptr && row0 < len) {
      for (int hb = 0; hb < 2 && row0 + 64 * hb < len; ++hb)
        for (int p = 0; p < 2; ++p)
          tma_store_4d(&tmO, smem + L::OFF_Q + t * L::Q_BYTES + p * 16384 + hb * 8192, 64 * p, h,
                       base + row0 + 64 * hb, bc);
      bulk_commit();
      bulk_wait_all();
    }
  }

  // Both CTAs leave together: every remote arrive has landed and every pair
  // MMA (which reads both CTAs' shared memory) has completed before either
  // CTA's shared memory and TMEM go away.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, L::TMEM_COLS);
  }
}

cudaError_t launch_fwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                        const FwdParams& prm_in, int B, cudaStream_t stream) {
  using L = Fwd2Layout;
  static_assert(L::BYTES + 1023 <= L::ALLOC, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(lg_fwd2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  FwdParams prm = prm_in;
  prm.nqt = (prm.S + 511) / 512;  // 512-row pair spans
  dim3 grid(2 * prm.nqt, prm.H, B);
  lg_fwd2_kernel<<<grid, L::THREADS, L::ALLOC, stream>>>(tq, tk, tv, to, prm);
  return cudaGetLastError();
}

}  // namespace lg
