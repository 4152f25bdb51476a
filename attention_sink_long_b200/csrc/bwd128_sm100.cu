// bwd128_sm100.cu -- LongGen sparse causal attention, training backward with
// 128-row KV tiles and 128-row query steps, for head dims 64 and 128, on sm_100a.
//
// "A Little Goes a Long Way" (LongGen), Abstract insights 1-2 and the
// atlas.scime.ai summary, "Approach": the sparse layers are trained, so the
// attention backward runs over the same static block pattern as the forward.
// Gradients follow from O = softmax(Q K^T * scale) V (FlashAttention-2 style
// recomputation from the saved row log-sum-exp):
//   P = exp(S * scale - lse),  dV = P^T dO,  dP = dO V^T,
//   dS = P o (dP - Delta) with Delta = rowsum(dO o O),
//   dK = scale * dS^T Q,  dQ = scale * dS K.
//
// One CTA owns a 128-row KV tile of one KV head -- two 64-row KV blocks paired
// by BlockPairing (blocks every later query sees pair with each other, then
// the window-only blocks pair in order), so both halves of the tile see nearly
// the same query blocks -- and walks those query blocks two at a time: a
// 128-row query step (with query-head groups, the steps of every query head
// of the group in turn, dK and dV accumulating over all of them). The one KV
// tile per head that far more queries see (the sink tile) is instead walked by
// several CTAs, each over a range of query steps, whose fp32 dK / dV partials
// the last of them sums (see the launch order below).
// At head dim 128 every GEMM of a step is then an M = 128, N = 128 tcgen05
// MMA -- the shape the tensor core runs at full rate (an N = 64 instruction
// takes about as long as an N = 128 one):
//   S^T  = K Q^T       SS, both K-major               -> TMEM region R_s
//   dP^T = V dO^T      SS, both K-major               -> TMEM region R_d
//   dV  += P^T dO      TS: P^T (bf16) from TMEM, dO MN-major
//   dK  += dS^T Q      SS: dS^T (bf16) from shared memory, Q MN-major
//   dQ^T = K^T dS^T    SS, both MN-major              -> R_d, drained with
//                      coalesced fp32 reductions into the dQ accumulator.
// TMEM columns: dV [0,D), dK [D,2D), R_s [2D,2D+128), R_d [2D+128,2D+256).
// At head dim 64 S^T and dP^T keep M = N = 128 (K = 64), dV and dK run with
// N = 64, and dQ^T keeps M = 128: its A operand's second 64-row half reads
// whatever lies one panel further on and lands in TMEM lanes 64-127, which
// nothing reads (an M = 64 instruction would take as long).
// The P/dS warps read S^T and write P^T (bf16, two per column) over the first
// half of the columns they read, so no warp overwrites columns another warp
// still reads. R_d holds dP^T until the warps have read it, then dQ^T.
// With query-head groups dV and dK sum over the group's heads and grow with
// it, so P and dS also enter them as bf16 residuals (x - bf16(x)): P^T's into
// the second half of each warp's S^T columns, dS^T's into the first half of
// each warp's dP^T columns (both already read), each an extra TS MMA.
//
// MMA order (one thread; tcgen05 MMAs of one thread execute in order):
//   S^T(0), dP^T(0), dV(0), S^T(1), then per step n:
//   [dS(n) ready]  dQ^T(n), dK(n)    (dQ^T first: the drain, on the step's
//                  critical chain, starts a GEMM earlier -- +2 % -- while Q(n)'s
//                  stage refills a GEMM later; with query-head groups dK's
//                  residual half, which reads R_d, must come before dQ^T and its
//                  shared-memory half follows: +3 % at four query heads per KV head)
//   [dQ^T(n) drained]  dP^T(n+1)
//   [P(n+1) ready]  dV(n+1)          (dO(n+1)'s stage refills after it)
//   [Q(n+2) loaded]  S^T(n+2)        (after dV(n+1), which reads P^T(n+1))
// so the P/dS warps find S^T of the next step computed while they finish dS,
// and the tensor pipe has the next GEMMs queued while each wait resolves.
//
// Warps: 0-7 P / dS + epilogue (two per TMEM lane quarter: KV rows
// 32 (w % 4) .. +31, query columns [64 (w / 4), +64) of the step), 8 TMA
// producer, 9 TMEM owner + MMA issuer, 10-13 dQ drain (one per lane quarter).
// Shared memory: K, V, two Q / dO stages (128 x D bf16 each) and dS^T
// (128 x 128 bf16) -- 224 KB at head dim 128, 128 KB at 64 -- plus barriers
// and the LSE / Delta stages after them.
#include "lg_common.cuh"
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

template <int D_>
struct Bwd128Layout {
  static constexpr int D = D_;
  static constexpr int DP = D / 64;             // 64-column (128-byte) panels per row
  static constexpr int QS = 2;                  // Q / dO / LSE / Delta stages
  static constexpr int TILE = 128 * D * 2;      // a 128 x D bf16 tile (K, V, Q, dO)
  static constexpr int PANEL = 128 * 128;       // one 64-column panel of 128 rows (bytes)
  static constexpr int DS_TILE = 128 * 128 * 2; // dS^T: 128 KV rows x 128 query columns, two panels
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;          // QS stages
  static constexpr int OFF_DO = OFF_Q + QS * TILE;    // QS stages
  static constexpr int OFF_DS = OFF_DO + QS * TILE;   // dS^T, rows = KV, columns = query
  static constexpr int TILES = OFF_DS + DS_TILE;      // 229376 at head dim 128
  static constexpr int NBAR = 1 + 4 * QS + 8;
  static constexpr int OFF_BAR = TILES;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_LSE = (OFF_MISC + 16 + 15) / 16 * 16;  // QS x 128 fp32
  static constexpr int OFF_DEL = OFF_LSE + QS * 512;   // QS x 128 fp32
  static constexpr int BYTES = OFF_DEL + QS * 512;
  // Head dim 128 needs nearly the whole per-block maximum; the smaller layout
  // asks for its size plus the 1024-byte alignment slack.
  static constexpr int ALLOC = D == 128 ? 232448 : BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DV = 0, T_DK = D, T_RS = 2 * D, T_RD = 2 * D + 128;
  static_assert(OFF_LSE % 16 == 0, "bulk copies need 16-byte aligned destinations");
  static_assert(BYTES <= ALLOC && ALLOC <= 232448, "shared memory budget");
  static_assert(T_RD + 128 <= TMEM_COLS, "TMEM budget");
};

template <int D, bool GQA>
__global__ void __launch_bounds__(448, 1)
    lg_bwd128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                     const BwdParams prm) {
  using L = Bwd128Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // The tiles need a 1024-byte aligned base (128-byte swizzle); at head dim
  // 128 the layout uses nearly the whole per-block allocation, so it only fits
  // when the dynamic shared memory starts close enough to such a boundary. Checked
  // uniformly before anything else; a misfit is reported, never run.
  if ((size_t)(smem - smem_raw) + (size_t)L::BYTES > (size_t)L::ALLOC) {
    if (threadIdx.x == 0) atomicOr(prm.err, kErrSmemFit);
    return;
  }
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars;
  // Q (+ LSE) and dO (+ Delta) stage separately: dO is done with after
  // dV, Q only after dK, so each refill starts as soon as its own tile frees.
  uint64_t* qq_full = bars + 1;               // [QS] Q and LSE of a step landed
  uint64_t* qq_empty = bars + 1 + L::QS;      // [QS] ... may be refilled
  uint64_t* qo_full = bars + 1 + 2 * L::QS;   // [QS] dO and Delta of a step landed
  uint64_t* qo_empty = bars + 1 + 3 * L::QS;  // [QS] ... may be refilled
  uint64_t* s_full = bars + 1 + 4 * L::QS;    // S^T of the next step in R_s
  uint64_t* dp_full = s_full + 1;          // dP^T in R_d
  uint64_t* p_full = s_full + 2;           // every P/dS warp wrote its P^T
  uint64_t* ds_full = s_full + 3;          // dS^T in shared memory, dP^T read
  uint64_t* dq_full = s_full + 4;          // dQ^T in R_d
  uint64_t* dq_free = s_full + 5;          // dQ^T read out of R_d
  uint64_t* dss_free = s_full + 6;         // dQ^T and dK done with the dS^T tile
  uint64_t* acc_done = s_full + 7;         // every MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);  // this chunk sums the partials
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_del = reinterpret_cast<const float*>(smem + L::OFF_DEL);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  // Sequence b occupies rows [base, base + len) at tensor-map batch coordinate
  // bc: the (B, S) layout, or the packed variable-length layout whose offsets
  // come from cu_seqlens and are checked here (a bad list is reported and its
  // sequence skipped). Per head, LSE, Delta and dQ-accumulator rows of the
  // sequence start at hrow0 + h * S; its dK / dV rows at lin0.
  int len = prm.S, base = 0, bc = b;
  if (prm.cu_seqlens != nullptr) {
    const int s0 = prm.cu_seqlens[b], s1 = prm.cu_seqlens[b + 1];
    // (s0 % 4 == 0 keeps the 64-row LSE / Delta copies 16-byte aligned.)
    if (s0 < 0 || (s0 & 3) != 0 || s1 < s0 || ((s1 - s0) & 63) != 0 || s1 > prm.S || s1 - s0 > prm.max_len) {
      if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(prm.err, kErrVarlen);
      return;
    }
    len = s1 - s0;
    base = s0;
    bc = 0;
  }
  const int nqb = len / 64;
  // Launch order: first the heavy KV tiles (those a sink or strided block makes
  // visible to many more queries, listed by the host), then the other tiles
  // head by head in ascending order. A heavy tile walks the query blocks from
  // its own block to the end of the sequence, streaming the head's Q, dO and
  // fp32 dQ accumulator (len x 1 KB). From 64K rows on that no longer fits
  // beside other heads in the 126 MB L2, so when a head has several heavy
  // tiles they run together, head by head, and all walk the query blocks
  // downwards from the end: they then read and reduce into the same blocks at
  // about the same time, and L2 serves one sweep to all of them (measured on
  // the 128K block-sparse {64,1,16,32} backward: 22.0 ms against 24.3-26.5;
  // at 32K, where each tile's own order hits L2 anyway, the change was within
  // +-4 %). Otherwise the heavy tiles run interleaved across heads, ascending.
  // When each head has a single heavy tile (the sink tile of a sink + window
  // pattern) in a fixed-length batch, its walk is split instead into
  // n_chunks ranges of query steps, one CTA each, placed evenly among the
  // head's other tiles in launch order: each chunk then sweeps the query rows
  // that the tiles running beside it read and reduce into, so Q, dO and the
  // dQ accumulator come from L2 once rather than in a second sweep of their own.
  int u, h;
  int chunk = -1;     // this CTA's chunk of the split heavy tile, or -1
  bool down = false;  // walk the query steps from the last to the first
  if (prm.n_chunks > 0) {
    const int nch = prm.n_chunks;
    const int R = prm.nkt - 1 + nch;  // slots per head: the other tiles and the chunks
    h = blockIdx.x / R;
    const int sl = blockIdx.x % R;
    // Chunk c takes slot floor(c R / nch); cnt = chunk slots at or before sl.
    const int cnt = ((sl + 1) * nch + R - 1) / R;
    if (cnt > 0 && ((cnt - 1) * R) / nch == sl) {
      chunk = cnt - 1;
      u = prm.heavy[0];
    } else {
      u = sl - cnt;
      u += (u >= prm.heavy[0]) ? 1 : 0;  // skip the heavy tile
    }
  } else {
    const int Lx = blockIdx.x;
    const int nh = prm.n_heavy;
    if (Lx < nh * prm.Hkv) {
      if (nh > 1 && len >= 65536) {
        u = prm.heavy[Lx % nh];
        h = Lx / nh;
        down = true;
      } else {
        u = prm.heavy[Lx / prm.Hkv];
        h = Lx % prm.Hkv;
      }
    } else {
      const int rest = prm.nkt - nh;
      const int L2 = Lx - nh * prm.Hkv;
      h = L2 / rest;
      u = L2 % rest;
      for (int k = 0; k < nh; ++k) u += (prm.heavy[k] <= u) ? 1 : 0;  // skip the heavy tiles
    }
  }
  const size_t hrow0 = prm.cu_seqlens != nullptr ? (size_t)base : (size_t)b * prm.H * prm.S;
  const long long lin0 = prm.cu_seqlens != nullptr ? (long long)base : (long long)b * prm.S;
  // The tile's two KV blocks (ky = -1: the tile holds one block; its rows
  // 64..127 load past the sequence end -- zeros, or the next packed sequence's
  // rows -- stay masked and are never stored).
  const BlockPairing bp(prm.pat, nqb);
  if (u >= bp.tiles()) return;  // past a shorter sequence's last tile (uniform exit)
  int kx, ky;
  bp.pair(u, &kx, &ky);
  const int kload[2] = {kx, ky >= 0 ? ky : nqb};
  // Query blocks [q_first, last] see the tile (the union of both blocks' lists).
  const int q_first = ky >= 0 ? imin(kx, ky) : kx;
  const int last = ky >= 0 ? imax(bp.reach(kx), bp.reach(ky)) : bp.reach(kx);
  const int N = (last - q_first + 2) / 2;  // 128-row query steps (the last one may hold one block)
  // The query steps this CTA walks: [t0, t0 + NQ) (all N, or one chunk).
  const int t0 = chunk >= 0 ? chunk * prm.chunk_steps : 0;
  const int NQ = chunk >= 0 ? imin(prm.chunk_steps, N - t0) : N;
  if (NQ <= 0) return;  // (a chunk past the tile's last step: none with a fixed-length batch)
  // With query-head groups the CTA walks every query head of its KV head:
  // step m is query step t0 + m % NQ of query head h * G + m / NQ, and dK / dV
  // accumulate over the whole group.
  const int G = GQA ? prm.H / prm.Hkv : 1;
  const int NT = G * NQ;
  // First query block of step m (of its query head), in the tile's walk order.
  auto step_block = [&](int m) -> int {
    const int t = t0 + (GQA ? m % NQ : m);
    return q_first + 2 * (down ? N - 1 - t : t);
  };
  auto step_head = [&](int m) -> int { return GQA ? h * G + m / NQ : h; };
  unsigned int* err = prm.err;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < L::QS; ++s) {
      mbar_init(&qq_full[s], 1);
      mbar_init(&qq_empty[s], 1 + 256);
      mbar_init(&qo_full[s], 1);
      mbar_init(&qo_empty[s], 1 + 256);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, D);  // the drain threads of the D real dQ^T rows
    mbar_init(dss_free, 1);
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
      for (int hb = 0; hb < 2; ++hb)
        for (int p = 0; p < L::DP; ++p) {
          tma_load_4d(smem + L::OFF_K + p * L::PANEL + hb * 8192, &tmK, kv_full, 64 * p, h, base + 64 * kload[hb], bc);
          tma_load_4d(smem + L::OFF_V + p * L::PANEL + hb * 8192, &tmV, kv_full, 64 * p, h, base + 64 * kload[hb], bc);
        }
      int issued_o = 0, issued_q = 0;  // steps whose dO / Q copies were issued
      for (int m = 0; m < NT; ++m) {
        const int st = m & 1;
        const uint32_t use = (uint32_t)(m >> 1);
        const int hq = step_head(m);  // query head
        const int i0 = step_block(m);
        // Both 64-row halves always load (rows past the sequence arrive as
        // zeros), so a stage never holds stale operands; LSE / Delta only
        // exist for blocks inside the sequence.
        const int nl = (i0 + 1 < nqb) ? 2 : 1;
        if (use > 0 && !mbar_wait(&qo_empty[st], (use - 1) & 1, abort_flag, err, kErrBwdWait)) break;
        mbar_arrive_expect_tx(&qo_full[st], L::TILE + nl * 256);
        issued_o = m + 1;
        for (int hb = 0; hb < 2; ++hb)
          for (int p = 0; p < L::DP; ++p)
            tma_load_4d(smem + L::OFF_DO + st * L::TILE + p * L::PANEL + hb * 8192, &tmdO, &qo_full[st], 64 * p, hq,
                        base + 64 * (i0 + hb), bc);
        for (int hb = 0; hb < nl; ++hb) {
          const size_t row = hrow0 + (size_t)hq * prm.S + 64 * (size_t)(i0 + hb);
          bulk_load(smem + L::OFF_DEL + st * 512 + hb * 256, prm.delta + row, 256, &qo_full[st]);
        }
        if (use > 0 && !mbar_wait(&qq_empty[st], (use - 1) & 1, abort_flag, err, kErrBwdWait)) break;
        mbar_arrive_expect_tx(&qq_full[st], L::TILE + nl * 256);
        issued_q = m + 1;
        for (int hb = 0; hb < 2; ++hb)
          for (int p = 0; p < L::DP; ++p)
            tma_load_4d(smem + L::OFF_Q + st * L::TILE + p * L::PANEL + hb * 8192, &tmQ, &qq_full[st], 64 * p, hq,
                        base + 64 * (i0 + hb), bc);
        for (int hb = 0; hb < nl; ++hb) {
          const size_t row = hrow0 + (size_t)hq * prm.S + 64 * (size_t)(i0 + hb);
          bulk_load(smem + L::OFF_LSE + st * 512 + hb * 256, prm.lse2 + row, 256, &qq_full[st]);
        }
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA's shared memory goes away.
        const long long t0 = clock64();
        while (!mbar_try_wait(kv_full, 0) && clock64() - t0 < 20000000LL) {
        }
        for (int s = 0; s < 2 * L::QS; ++s) {
          const int issued = s < L::QS ? issued_o : issued_q;
          const int stg = s % L::QS;
          if (stg >= issued) continue;
          const int lastn = issued - 1 - ((issued - 1 - stg) & 1);
          uint64_t* bar = s < L::QS ? &qo_full[stg] : &qq_full[stg];
          const long long t1 = clock64();
          while (!mbar_try_wait(bar, (uint32_t)(lastn >> 1) & 1) && clock64() - t1 < 20000000LL) {
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
      constexpr uint32_t idesc_kk = idesc_bf16(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_kmn = idesc_bf16(128, D, false, true);     // dV (A in TMEM), dK
      constexpr uint32_t idesc_mnmn = idesc_bf16(128, 128, true, true);   // dQ^T
      // Descriptor bases (the start field moves by 16-byte units per k-step).
      // K-major operands advance 32 bytes per k-step inside a 64-column panel
      // and jump a panel every four; MN-major ones advance 16 rows (2048 bytes)
      // and reach their second 64-element half through the leading offset (at
      // head dim 64, K^T's second half is the unread upper half of dQ^T).
      const uint64_t dK_k = sdesc_sw128(sbase + L::OFF_K, 16, 1024);
      const uint64_t dV_k = sdesc_sw128(sbase + L::OFF_V, 16, 1024);
      const uint64_t dK_mn = sdesc_sw128(sbase + L::OFF_K, L::PANEL, 1024);
      const uint64_t dS_k = sdesc_sw128(sbase + L::OFF_DS, 16, 1024);
      const uint64_t dS_mn = sdesc_sw128(sbase + L::OFF_DS, L::PANEL, 1024);
      auto kofs = [](int kk) -> uint32_t { return (uint32_t)(((kk >> 2) * L::PANEL + (kk & 3) * 32) >> 4); };
      auto mofs = [](int kk) -> uint32_t { return (uint32_t)((kk * 2048) >> 4); };
      auto q_k = [&](int n) { return sdesc_sw128(sbase + L::OFF_Q + (n & 1) * L::TILE, 16, 1024); };
      auto o_k = [&](int n) { return sdesc_sw128(sbase + L::OFF_DO + (n & 1) * L::TILE, 16, 1024); };
      auto q_mn = [&](int n) {
        return sdesc_sw128(sbase + L::OFF_Q + (n & 1) * L::TILE, L::PANEL, 1024);
      };
      auto o_mn = [&](int n) {
        return sdesc_sw128(sbase + L::OFF_DO + (n & 1) * L::TILE, L::PANEL, 1024);
      };
      // S^T(n) = K Q(n)^T into R_s.
      auto issue_s = [&](int n) {
        const uint64_t q = q_k(n);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss_if(leader, tmem + L::T_RS, dK_k + kofs(kk), q + kofs(kk), idesc_kk, kk > 0 ? 1u : 0u);
      };
      // dP^T(n) = V dO(n)^T into R_d.
      auto issue_dp = [&](int n) {
        const uint64_t o = o_k(n);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss_if(leader, tmem + L::T_RD, dV_k + kofs(kk), o + kofs(kk), idesc_kk, kk > 0 ? 1u : 0u);
      };
      // dV += P^T(n) dO(n); P^T of query columns [64 hf, +64) sits in R_s
      // columns [64 hf, +32), two bf16 per column.
      auto issue_dv = [&](int n) {
        const uint64_t o = o_mn(n);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ts_if(leader, tmem + L::T_DV, tmem + L::T_RS + 64 * (kk >> 2) + 8 * (kk & 3), o + mofs(kk), idesc_kmn,
                    (n > 0 || kk > 0) ? 1u : 0u);
        if (GQA) {  // + the bf16 residual of P^T, 32 columns further on
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ts_if(leader, tmem + L::T_DV, tmem + L::T_RS + 32 + 64 * (kk >> 2) + 8 * (kk & 3), o + mofs(kk),
                         idesc_kmn, 1u);
        }
      };
      // dK += dS^T(n) Q(n).
      // (with query-head groups: dK's shared-memory half only; see issue_dk_lo)
      auto issue_dk = [&](int n) {
        const uint64_t q = q_mn(n);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ss_if(leader, tmem + L::T_DK, dS_k + kofs(kk), q + mofs(kk), idesc_kmn,
                       (GQA || n > 0 || kk > 0) ? 1u : 0u);
      };
      // dK += the bf16 residual of dS^T (query-head groups), left in R_d by the
      // dS phase; issued first, since dQ^T overwrites R_d next.
      auto issue_dk_lo = [&](int n) {
        const uint64_t q = q_mn(n);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ts_if(leader, tmem + L::T_DK, tmem + L::T_RD + 64 * (kk >> 2) + 8 * (kk & 3), q + mofs(kk),
                       idesc_kmn, (n > 0 || kk > 0) ? 1u : 0u);
      };
      // dQ^T(n) = K^T dS^T(n) into R_d (fresh each step).
      auto issue_dq = [&](int n) {
        (void)n;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ss_if(leader, tmem + L::T_RD, dK_mn + mofs(kk), dS_mn + mofs(kk), idesc_mnmn, kk > 0 ? 1u : 0u);
      };

      bool ok = mbar_wait(kv_full, 0, abort_flag, err, kErrBwdWait) &&
                mbar_wait(&qq_full[0], 0, abort_flag, err, kErrBwdWait);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        tc_commit_if(leader, s_full);
        ok = mbar_wait(&qo_full[0], 0, abort_flag, err, kErrBwdWait);
      }
      if (ok) {
        tc_fence_after();
        issue_dp(0);
        tc_commit_if(leader, dp_full);
        ok = mbar_wait(p_full, 0, abort_flag, err, kErrBwdWait);
      }
      if (ok) {
        tc_fence_after();
        issue_dv(0);
        tc_commit_if(leader, &qo_empty[0]);
        if (NT > 1) {
          ok = mbar_wait(&qq_full[1], 0, abort_flag, err, kErrBwdWait);
          if (ok) {
            tc_fence_after();
            issue_s(1);
            tc_commit_if(leader, s_full);
          }
        }
      }
      for (int n = 0; n < NT && ok; ++n) {  // n: global step
        const uint32_t par = (uint32_t)n & 1;
        if (!mbar_wait(ds_full, par, abort_flag, err, kErrBwdWait)) break;
        tc_fence_after();
        // dQ^T first: the drain that reads it is on the step's critical chain
        // (dQ^T(n) -> drain -> dP^T(n+1) -> dS(n+1)); dK, the last use of Q(n),
        // follows, so that stage's refill with Q(n+2) starts a GEMM later --
        // measured +2 % overall (interleaved A/B, 32K and 128K). With query-head
        // groups dK's residual half must precede dQ^T (both use R_d) and its
        // shared-memory half follows.
        if (GQA) {
          issue_dk_lo(n);
          issue_dq(n);
          tc_commit_if(leader, dq_full);
          issue_dk(n);
          tc_commit_if(leader, &qq_empty[n & 1]);
        } else {
          issue_dq(n);
          tc_commit_if(leader, dq_full);
          issue_dk(n);
          tc_commit_if(leader, &qq_empty[n & 1]);
        }
        tc_commit_if(leader, dss_free);
        if (n + 1 < NT) {
          // R_d takes dP^T(n+1) once the drain warps have read dQ^T(n).
          if (!mbar_wait(dq_free, par, abort_flag, err, kErrBwdWait)) break;
          if (!mbar_wait(&qo_full[(n + 1) & 1], (uint32_t)((n + 1) >> 1) & 1, abort_flag, err, kErrBwdWait)) break;
          tc_fence_after();
          issue_dp(n + 1);
          tc_commit_if(leader, dp_full);
          if (!mbar_wait(p_full, par ^ 1u, abort_flag, err, kErrBwdWait)) break;
          tc_fence_after();
          issue_dv(n + 1);
          tc_commit_if(leader, &qo_empty[(n + 1) & 1]);
          if (n + 2 < NT) {
            // S^T(n+2) overwrites P^T(n+1), which dV(n+1) -- issued just before --
            // reads first; its Q stage was refilled after dK(n) completed.
            if (!mbar_wait(&qq_full[n & 1], (uint32_t)((n + 2) >> 1) & 1, abort_flag, err, kErrBwdWait)) break;
            tc_fence_after();
            issue_s(n + 2);
            tc_commit_if(leader, s_full);
          }
        }
      }
      tc_commit_if(leader, acc_done);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P / dS warps
    // Warp w owns KV rows 32 (w % 4) .. +31 (its TMEM lane quarter) and query
    // columns [64 hf, +64) of each step, hf = w / 4 -- one 64 x 64 block pair,
    // so visibility and the diagonal mask are warp-uniform.
    const int hf = warp >> 2;
    const int c0 = 64 * hf;
    const int r = (warp & 3) * 32 + lane;  // KV row of the tile == TMEM lane
    const int kvb = (r >> 6) ? ky : kx;  // this thread's KV block (-1: none)
    const int rr = r & 63;
    const bool krow_live = kvb >= 0;
    const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = prm.scale_log2;
    int n = 0;
    for (; n < NT; ++n) {  // n: step of this CTA (query head step_head(n))
      const int st = n & 1;
      const uint32_t par = (uint32_t)n & 1;
      const int i = step_block(n) + hf;  // this warp's query block
      const bool vis = krow_live && i <= last && in_list(prm.pat, i, kvb);
      const bool diag = (i == kvb);
      if (!__all_sync(0xffffffffu, mbar_wait(&qq_full[st], (uint32_t)(n >> 1) & 1, abort_flag, err, kErrBwdWait)))
        break;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, par, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      // P^T = exp2(S^T * scale * log2 e - lse * log2 e), 32 columns at a time; the
      // bf16 pairs go back over the first 32 of this warp's 64 S^T columns
      // (already read), fp32 copies stay for dS.
      float pf[64];
      // LSE and Delta are the same for every thread of the warp: 16-byte
      // broadcast loads, four columns each.
      const float4* lse4 = reinterpret_cast<const float4*>(s_lse + st * 128 + c0);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t sr[32];
        tmem_ld32(t_lane + L::T_RS + c0 + 32 * ch, sr);
        if (vis) {
          // the stage holds LSE in log2 units (preprocess), so one paired FMA
          // gives the exponent of two columns
          const float2 sc2 = make_float2(sl2, sl2);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 l4 = lse4[8 * ch + g];
            const float2 a0 = fma2(make_float2(__uint_as_float(sr[4 * g]), __uint_as_float(sr[4 * g + 1])), sc2,
                                   make_float2(-l4.x, -l4.y));
            const float2 a1 = fma2(make_float2(__uint_as_float(sr[4 * g + 2]), __uint_as_float(sr[4 * g + 3])), sc2,
                                   make_float2(-l4.z, -l4.w));
            const float pv[4] = {ex2_approx(a0.x), ex2_approx(a0.y), ex2_approx(a1.x), ex2_approx(a1.y)};
#pragma unroll
            for (int e = 4 * g; e < 4 * g + 4; ++e) pf[32 * ch + e] = (diag && 32 * ch + e < rr) ? 0.f : pv[e - 4 * g];
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) pf[32 * ch + e] = 0.f;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pf[32 * ch + 2 * e], pf[32 * ch + 2 * e + 1]);
        tmem_st16(t_lane + L::T_RS + c0 + 16 * ch, pk);
      }
      if (GQA) {
        // The bf16 residual P - bf16(P) into columns [32, 64) of this warp's
        // S^T range (read above): dV takes P^T as a hi + lo pair, exact to the
        // fp32 accumulation, since its sum over the group grows with it.
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t pl[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = pf[32 * ch + 2 * e], b = pf[32 * ch + 2 * e + 1];
            const uint32_t hi = pack_bf16x2(a, b);
            pl[e] = pack_bf16x2(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
          }
          tmem_st16(t_lane + L::T_RS + c0 + 32 + 16 * ch, pl);
        }
      }
      tc_fence_before();
      mbar_arrive(p_full);
      mbar_arrive(&qq_empty[st]);  // done with this step's LSE
      if (!__all_sync(0xffffffffu, mbar_wait(&qo_full[st], (uint32_t)(n >> 1) & 1, abort_flag, err, kErrBwdWait)))
        break;
      if (!__all_sync(0xffffffffu, mbar_wait(dp_full, par, abort_flag, err, kErrBwdWait))) break;
      // The dS^T tile last fed dQ^T(n-1) and dK(n-1).
      if (n >= 1 && !__all_sync(0xffffffffu, mbar_wait(dss_free, par ^ 1u, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      // dS^T = P^T o (dP^T - Delta), bf16 into the swizzled dS^T tile (rows =
      // KV, query panel hf). Blocks this row does not see give exact zeros.
      const float4* del4 = reinterpret_cast<const float4*>(s_del + st * 128 + c0);
      const uint32_t drow = sbase + L::OFF_DS + hf * L::PANEL;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dpr[32];
        tmem_ld32(t_lane + L::T_RD + c0 + 32 * ch, dpr);
        uint32_t dlo[16];  // with query-head groups: dS - bf16(dS), packed, back into R_d
        // eight columns (one 16-byte chunk of the row) at a time
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[4];
          if (vis) {
            const float4 da = del4[8 * ch + 2 * c], db = del4[8 * ch + 2 * c + 1];
            const float dl[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int k = 32 * ch + 8 * c + 2 * e;
              const float2 d = mul2(make_float2(pf[k], pf[k + 1]),
                                    sub2(make_float2(__uint_as_float(dpr[8 * c + 2 * e]),
                                                     __uint_as_float(dpr[8 * c + 2 * e + 1])),
                                         make_float2(dl[2 * e], dl[2 * e + 1])));
              pk[e] = pack_bf16x2(d.x, d.y);
              if (GQA)
                dlo[4 * c + e] = pack_bf16x2(d.x - __uint_as_float(pk[e] << 16), d.y - __uint_as_float(pk[e] & 0xffff0000u));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              pk[e] = 0u;
              if (GQA) dlo[4 * c + e] = 0u;
            }
          }
          st_shared_v4(drow + sw128_offset(r, 4 * ch + c), pk[0], pk[1], pk[2], pk[3]);
        }
        // Columns [16 ch, +16) of this warp's R_d range were read by the load
        // above (ch = 0 read all 32 of them), and dK reads them as an MMA
        // operand before dQ^T overwrites R_d.
        if (GQA) tmem_st16(t_lane + L::T_RD + c0 + 16 * ch, dlo);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
      mbar_arrive(&qo_empty[st]);  // done with this step's Delta
    }

    // ------------------------------------------------------------ dK, dV epilogue
    // Warp (quarter, half) writes rows of its quarter, columns [D/2 half, +D/2).
    bool ok = (n == NT) && !*abort_flag;
    if (ok) ok = mbar_wait(acc_done, 0, abort_flag, err, kErrBwdWait);
    ok = __all_sync(0xffffffffu, ok);
    // A chunk of a split heavy tile hands its fp32 dV / dK partial to the
    // workspace; the chunk that finishes last sums all of them, in chunk order
    // (so the result does not depend on which one that is), and writes the
    // gradients below; the others stop here.
    const size_t per_chunk = (size_t)2 * 128 * L::D;
    const int nch_live = chunk >= 0 ? (N + prm.chunk_steps - 1) / prm.chunk_steps : 0;
    const float* part = nullptr;
    if (chunk >= 0) {
      float* mine = prm.hk_part + (((size_t)b * prm.Hkv + h) * prm.n_chunks + chunk) * per_chunk;
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int which = 0; which < 2; ++which)
#pragma unroll
          for (int q = 0; q < D / 64; ++q) {
            const int col = (D / 2) * hf + 32 * q;
            uint32_t o[32];
            tmem_ld32(t_lane + (which == 0 ? L::T_DV : L::T_DK) + col, o);
            float4* d4 = reinterpret_cast<float4*>(mine + ((size_t)which * 128 + r) * L::D + col);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                  __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
          }
      }
      __threadfence();
      named_bar_sync(1, 256);
      if (threadIdx.x == 0) {
        const unsigned int prev = ok ? atomicAdd(&prm.hk_ticket[b * prm.Hkv + h], 1u) : 0u;
        *last_flag = (ok && prev == (unsigned int)(nch_live - 1)) ? 1 : 0;
      }
      named_bar_sync(1, 256);
      ok = *last_flag != 0;
      if (ok) {
        __threadfence();
        part = prm.hk_part + ((size_t)b * prm.Hkv + h) * prm.n_chunks * per_chunk;
      }
    }
    // 32 columns of this thread's dV (which = 0) or dK row: from TMEM, or the
    // sum of the chunks' partials.
    auto acc_cols = [&](int which, int col, uint32_t (&o)[32]) {
      if (part == nullptr) {
        tmem_ld32(t_lane + (which == 0 ? L::T_DV : L::T_DK) + col, o);
        return;
      }
      float a[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) a[e] = 0.f;
      for (int c2 = 0; c2 < nch_live; ++c2) {
        const float4* src =
            reinterpret_cast<const float4*>(part + (size_t)c2 * per_chunk + ((size_t)which * 128 + r) * L::D + col);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 v = __ldcg(src + e);
          a[4 * e] += v.x;
          a[4 * e + 1] += v.y;
          a[4 * e + 2] += v.z;
          a[4 * e + 3] += v.w;
        }
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(a[e]);
    };
    if (ok && prm.grad_f32) {
      // fp32 gradients: each thread stores its part of a KV row straight from TMEM.
      tc_fence_after();
      const int krow = kvb >= 0 ? 64 * kvb + (r & 63) : 0;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const float mul = which == 0 ? 1.f : prm.scale;
        float* dst = (which == 0 ? prm.dv_f32 : prm.dk_f32) + (((size_t)lin0 + krow) * prm.Hkv + h) * L::D;
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {
          const int col = (D / 2) * hf + 32 * q;
          uint32_t o[32];
          acc_cols(which, col, o);
          if (kvb >= 0) {
            float4* d4 = reinterpret_cast<float4*>(dst + col);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(o[4 * e]) * mul, __uint_as_float(o[4 * e + 1]) * mul,
                                  __uint_as_float(o[4 * e + 2]) * mul, __uint_as_float(o[4 * e + 3]) * mul);
          }
        }
      }
    } else if (ok) {
      // bf16 gradients: stage in the K / V tiles (every MMA is done with them),
      // then one TMA store per panel.
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const float mul = which == 0 ? 1.f : prm.scale;
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {
          const int col = (D / 2) * hf + 32 * q;  // 32 columns: four 16-byte chunks of a panel row
          const uint32_t panel = sbase + (which == 0 ? L::OFF_V : L::OFF_K) + (uint32_t)(col >> 6) * L::PANEL;
          uint32_t o[32];
          acc_cols(which, col, o);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float* f = reinterpret_cast<const float*>(&o[8 * q4]);
            st_shared_v4(panel + sw128_offset(r, ((col & 63) >> 3) + q4), pack_bf16x2(f[0] * mul, f[1] * mul),
                         pack_bf16x2(f[2] * mul, f[3] * mul), pack_bf16x2(f[4] * mul, f[5] * mul),
                         pack_bf16x2(f[6] * mul, f[7] * mul));
          }
        }
      }
    }
    fence_async_smem();
    named_bar_sync(1, 256);
    if (threadIdx.x == 0 && ok && !prm.grad_f32) {
      for (int hb = 0; hb < (ky >= 0 ? 2 : 1); ++hb)
        for (int p = 0; p < L::DP; ++p) {
          tma_store_4d(&tmdV, smem + L::OFF_V + p * L::PANEL + hb * 8192, 64 * p, h, base + 64 * kload[hb], bc);
          tma_store_4d(&tmdK, smem + L::OFF_K + p * L::PANEL + hb * 8192, 64 * p, h, base + 64 * kload[hb], bc);
        }
      bulk_commit();
      bulk_wait_all();
    }
  } else {
    // ------------------------------------------------------------ dQ drain warps 10-13
    // Thread = dQ^T row d (TMEM lane); a warp's 32 lanes hit 32 consecutive dQ
    // elements of one query row, so every reduction below is one coalesced
    // 128-byte request. At head dim 64 the warps of lane quarters 0 and 1
    // drain; the other two hold no dQ^T rows and stop here.
    const int quarter = warp & 3;
    const int d = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int n = 0; n < NT && 32 * quarter < D; ++n) {  // n: global step
      const int hq = step_head(n);  // query head
      const int i0 = step_block(n);
      const bool second = i0 + 1 <= last;  // the step's second query block is in the list range
      if (!__all_sync(0xffffffffu, mbar_wait(dq_full, (uint32_t)n & 1, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      float* dst = prm.dq_acc + (hrow0 + (size_t)hq * prm.S + 64 * (size_t)i0) * L::D + d;
      // Read all 128 columns first, so R_d is released before any reduction is
      // issued (the reductions run at the L2's rate and would otherwise hold
      // up the next dP^T).
      uint32_t va[64], vb[64];
      tmem_ld64(t_lane + L::T_RD, va);
      tmem_ld64(t_lane + L::T_RD + 64, vb);
      tc_fence_before();
      mbar_arrive(dq_free);
      // The reductions are spread over the step: a short pause after every 16
      // (measured 3-7 % faster than bursts, which crowd the P / dS warps' own
      // memory traffic on the same SM; pauses much longer than this let the
      // drain fall behind the next step).
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        red_add_f32(dst + (size_t)c * L::D, __uint_as_float(va[c]));
        if ((c & 15) == 15 && c < 63) __nanosleep(200);
      }
      // Loads before the second half of the reductions: the Q / dO copies of
      // step n+2 (issued once dK(n) freed their stage) go through L2 first, so
      // the next S^T is not starved by this step's reductions.
      if (n + 2 < NT &&
          !__all_sync(0xffffffffu, mbar_wait(&qq_full[n & 1], (uint32_t)((n + 2) >> 1) & 1, abort_flag, err,
                                             kErrBwdWait)))
        break;
      if (second) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          red_add_f32(dst + (size_t)(64 + c) * L::D, __uint_as_float(vb[c]));
          if ((c & 15) == 15 && c < 63) __nanosleep(200);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int D, bool GQA>
static cudaError_t launch_bwd128_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                      const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                                      const BwdParams& prm, int B, cudaStream_t stream) {
  using L = Bwd128Layout<D>;
  cudaError_t e = cudaFuncSetAttribute(lg_bwd128_kernel<D, GQA>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  // With the heavy tile split, each head has its other nkt - 1 tiles and n_chunks chunks.
  dim3 grid((prm.n_chunks > 0 ? prm.nkt - 1 + prm.n_chunks : prm.nkt) * prm.Hkv, B);
  lg_bwd128_kernel<D, GQA><<<grid, 448, L::ALLOC, stream>>>(tq, tk, tv, tdo, tdk, tdv, prm);
  return cudaGetLastError();
}

cudaError_t launch_bwd128(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                          const CUtensorMap& tdk, const CUtensorMap& tdv, const BwdParams& prm, int B,
                          cudaStream_t stream) {
  const bool gqa = prm.H != prm.Hkv;
  if (prm.D == 64)
    return gqa ? launch_bwd128_impl<64, true>(tq, tk, tv, tdo, tdk, tdv, prm, B, stream)
               : launch_bwd128_impl<64, false>(tq, tk, tv, tdo, tdk, tdv, prm, B, stream);
  if (prm.D != 128) return cudaErrorInvalidValue;
  return gqa ? launch_bwd128_impl<128, true>(tq, tk, tv, tdo, tdk, tdv, prm, B, stream)
             : launch_bwd128_impl<128, false>(tq, tk, tv, tdo, tdk, tdv, prm, B, stream);
}

}  // namespace lg
