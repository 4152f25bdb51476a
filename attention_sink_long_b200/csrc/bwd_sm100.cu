// bwd_sm100.cu -- LongGen sparse causal attention, training backward, for sm_100a.
//
// "A Little Goes a Long Way" (LongGen), atlas.scime.ai summary, "Approach"
// (training with a FlashAttention-2-based kernel) and "Key results" (1.55x
// training speedup at 128K). Three launches:
//   1. preprocess: Delta = rowsum(dO * O) per query row, and zero the fp32 dQ
//      accumulator;
//   2. main: KV-tile-parallel dK, dV with dQ accumulated through bulk fp32
//      reduce-add (see lg_bwd_kernel);
//   3. convert: dQ = scale * dQ_acc to bf16 in the [B, S, H, D] layout.
#include "lg_common.cuh"
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

// ---------------------------------------------------------------------------
// 1. Delta and dQ_acc clearing. One thread per 8 elements of a row.
// ---------------------------------------------------------------------------
template <int D, bool OF32>
__global__ void __launch_bounds__(256) lg_bwd_pre_kernel(const void* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         float* __restrict__ delta, float* __restrict__ dq_acc,
                                                         const float* __restrict__ lse, float* __restrict__ lse2,
                                                         int B, int S, int H) {
  constexpr int TPR = D / 8;
  const long long rows = (long long)B * S * H;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = t / TPR;  // memory order of O: ((b * S + s) * H + h)
  const int c = (int)(t % TPR);
  float acc = 0.f;
  if (row < rows) {
    float of[8];
    if constexpr (OF32) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(o) + row * D + 8 * c);
      const float4 x0 = src[0], x1 = src[1];
      of[0] = x0.x; of[1] = x0.y; of[2] = x0.z; of[3] = x0.w;
      of[4] = x1.x; of[5] = x1.y; of[6] = x1.z; of[7] = x1.w;
    } else {
      const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + row * D + 8 * c);
      const uint32_t aa[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        of[2 * e] = __uint_as_float(aa[e] << 16);
        of[2 * e + 1] = __uint_as_float(aa[e] & 0xffff0000u);
      }
    }
    const uint4 g = *reinterpret_cast<const uint4*>(dout + row * D + 8 * c);
    const uint32_t gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(of[2 * e], __uint_as_float(gg[e] << 16), acc);
      acc = fmaf(of[2 * e + 1], __uint_as_float(gg[e] & 0xffff0000u), acc);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows) {
    const int h = (int)(row % H);
    const long long bs = row / H;
    const int s = (int)(bs % S);
    const int b = (int)(bs / S);
    const long long drow = ((long long)b * H + h) * S + s;
    if (c == 0) delta[drow] = acc;
    if (c == 1) lse2[drow] = lse[drow] * 1.4426950408889634f;  // log2 units, for exp2 in the backward
    float4* z = reinterpret_cast<float4*>(dq_acc + drow * D + 8 * c);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

cudaError_t launch_bwd_pre(const void* o, int o_f32, const void* dout, float* delta, float* dq_acc, const float* lse,
                           float* lse2, int B, int S,
                           int H, int D, cudaStream_t stream) {
  const long long threads = (long long)B * S * H * (D / 8);
  const unsigned int blocks = (unsigned int)((threads + 255) / 256);
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(dout);
  if (D == 64) {
    if (o_f32) lg_bwd_pre_kernel<64, true><<<blocks, 256, 0, stream>>>(o, g, delta, dq_acc, lse, lse2, B, S, H);
    else lg_bwd_pre_kernel<64, false><<<blocks, 256, 0, stream>>>(o, g, delta, dq_acc, lse, lse2, B, S, H);
  } else {
    if (o_f32) lg_bwd_pre_kernel<128, true><<<blocks, 256, 0, stream>>>(o, g, delta, dq_acc, lse, lse2, B, S, H);
    else lg_bwd_pre_kernel<128, false><<<blocks, 256, 0, stream>>>(o, g, delta, dq_acc, lse, lse2, B, S, H);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 3. dQ = scale * dQ_acc, [B, H, S, D] fp32 -> [B, S, H, D] bf16.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) lg_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                        __nv_bfloat16* __restrict__ dq, float* __restrict__ dq_f32,
                                                        float scale, int B, int S, int H) {
  constexpr int TPR = D / 8;
  const long long rows = (long long)B * S * H;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = t / TPR;  // output memory order ((b * S + s) * H + h)
  const int c = (int)(t % TPR);
  if (row >= rows) return;
  const int h = (int)(row % H);
  const long long bs = row / H;
  const int s = (int)(bs % S);
  const int b = (int)(bs / S);
  const long long srow = ((long long)b * H + h) * S + s;
  const float4* src = reinterpret_cast<const float4*>(dq_acc + srow * D + 8 * c);
  const float4 x0 = src[0], x1 = src[1];
  if (dq_f32 != nullptr) {
    float4* dst = reinterpret_cast<float4*>(dq_f32 + row * D + 8 * c);
    dst[0] = make_float4(x0.x * scale, x0.y * scale, x0.z * scale, x0.w * scale);
    dst[1] = make_float4(x1.x * scale, x1.y * scale, x1.z * scale, x1.w * scale);
    return;
  }
  uint4 out;
  out.x = pack_bf16x2(x0.x * scale, x0.y * scale);
  out.y = pack_bf16x2(x0.z * scale, x0.w * scale);
  out.z = pack_bf16x2(x1.x * scale, x1.y * scale);
  out.w = pack_bf16x2(x1.z * scale, x1.w * scale);
  *reinterpret_cast<uint4*>(dq + row * D + 8 * c) = out;
}

cudaError_t launch_bwd_dq(const float* dq_acc, void* dq, int dq_f32, float scale, int B, int S, int H, int D,
                          cudaStream_t stream) {
  const long long threads = (long long)B * S * H * (D / 8);
  const unsigned int blocks = (unsigned int)((threads + 255) / 256);
  __nv_bfloat16* qb = dq_f32 ? nullptr : static_cast<__nv_bfloat16*>(dq);
  float* qf = dq_f32 ? static_cast<float*>(dq) : nullptr;
  if (D == 64)
    lg_bwd_dq_kernel<64><<<blocks, 256, 0, stream>>>(dq_acc, qb, qf, scale, B, S, H);
  else
    lg_bwd_dq_kernel<128><<<blocks, 256, 0, stream>>>(dq_acc, qb, qf, scale, B, S, H);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 2. main kernel for head dim 64 (head dim 128 runs lg_bwd128_kernel, in
// bwd128_sm100.cu). The template keeps D general; only D = 64 is instantiated.
//
// CTA per (128-row KV tile = KV blocks 2u and 2u+1, KV head, batch); it walks
// the union of the two blocks' query-block lists (a contiguous range, see
// QIter) for every query head of the KV head's group, one 64-row query block
// per step. Per step, all on tcgen05 with fp32 accumulation in TMEM:
//   S^T  = K Q_i^T          (M=128 kv, N=64 q, K=D)
//   dP^T = V dO_i^T         (M=128,    N=64,   K=D)
//   dV  += P^T dO_i         (M=128,    N=D,    K=64; P^T read from TMEM)
//   dK  += dS^T Q_i         (M=128,    N=D,    K=64; dS^T read from TMEM)
//   dQ_i^T = K^T dS^T       (M=D,      N=64,   K=128; dS^T from shared memory)
// with P^T = exp(scale S^T - LSE) on the mask and dS^T = P^T (dP^T - Delta),
// computed by eight warps, two per 32 KV rows (TMEM lanes). They write
// bf16 P^T and dS^T back into TMEM over the S^T / dP^T columns they have
// read (A operands of the dV / dK products), and dS^T also to shared memory
// (B operand of dQ^T). dQ_i^T lands in the middle 64 columns of the same
// step's TMEM buffer, which the P^T / dS^T writes leave free; four more warps
// read it and add it to the fp32 dQ accumulator with coalesced global
// reductions (a warp's 32 lanes cover 32 consecutive dQ elements of one row).
// The per-step TMEM buffer (S^T | dP^T) is double-buffered, so S^T / dP^T of
// step n+1 run while the warps work on step n, and the gradient GEMMs of
// step n run while they work on step n+1.
// With GQA (H / Hkv > 1) dV and dK sum over the group's query heads and grow
// with it, so P^T and dS^T then also enter dV / dK as the bf16 residual
// bf16(x - bf16(x)) from shared memory: dV and dK then carry no bf16 rounding
// of P or dS (a single bf16 operand costs ~2^-9 relative per term, which at
// |dK| ~ 4 is the whole 1e-2 error budget). Without GQA the plain five GEMMs
// are used.
//
// Warps: 0-7 P/dS + epilogue (two per TMEM lane quarter, 32 query columns
// each), 8 TMA producer, 9 TMEM owner + MMA issuer, 10-13 dQ drain. TMEM columns: dV [0,D), dK [D,2D), step buffer b at
// 2D + 128b: S^T [0,64) then P^T in [0,32); dP^T [64,128) then dS^T in
// [96,128); dQ^T in [32,96).
// ---------------------------------------------------------------------------
template <int D, bool SPLIT>
struct BwdLayout {
  static constexpr int QS = 3;                   // Q / dO stages
  static constexpr int KV_BYTES = 128 * D * 2;   // K or V tile (128 rows)
  static constexpr int QB_BYTES = 64 * D * 2;    // Q or dO block (64 rows)
  static constexpr int PT_BYTES = 128 * 64 * 2;  // a [128 x 64] bf16 tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;          // QS stages
  static constexpr int OFF_DO = OFF_Q + QS * QB_BYTES;    // QS stages
  static constexpr int OFF_DST = OFF_DO + QS * QB_BYTES;  // bf16(dS^T), 2 buffers
  static constexpr int OFF_PL = OFF_DST + 2 * PT_BYTES;   // GQA: bf16(P^T - bf16(P^T))
  static constexpr int OFF_DSL = OFF_PL + PT_BYTES;       // GQA: bf16(dS^T - bf16(dS^T))
  static constexpr int OFF_LSE = OFF_DSL + (SPLIT ? PT_BYTES : 0) - (SPLIT ? 0 : PT_BYTES);  // QS x 64 fp32
  static constexpr int OFF_DEL = OFF_LSE + QS * 256;      // QS stages x 64 fp32
  static constexpr int OFF_BAR = OFF_DEL + QS * 256;
  static constexpr int NBAR = 1 + 2 * QS + 19;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DV = 0, T_DK = D, T_BUF = 2 * D;
};


template <int D, bool SPLIT>
__global__ void __launch_bounds__(448, 1)
    lg_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                  const BwdParams prm) {
  using L = BwdLayout<D, SPLIT>;
  constexpr int DP = D / 64;
  constexpr int QS = L::QS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;        // [QS]
  uint64_t* q_empty = bars + 1 + QS;  // [QS]
  uint64_t* s_full = bars + 1 + 2 * QS;  // [2]
  uint64_t* dp_full = s_full + 2;        // [2]
  uint64_t* p_full = s_full + 4;         // [2]
  uint64_t* ds_full = s_full + 6;        // [2]
  uint64_t* dq_full = s_full + 8;        // [2]
  uint64_t* dq_free = s_full + 10;       // [2]
  uint64_t* dss_free = s_full + 12;      // [2]
  uint64_t* acc_done = s_full + 14;
  uint64_t* s_read = s_full + 15;   // [2] every P/dS warp has read S^T of the buffer
  uint64_t* dp_read = s_full + 17;  // [2] every P/dS warp has read dP^T of the buffer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_del = reinterpret_cast<const float*>(smem + L::OFF_DEL);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Launch order: first the heavy KV tiles (those a sink or strided block makes
  // visible to many more queries, listed by the host) of every head, then the
  // other tiles head by head in ascending order -- so the long CTAs start in
  // the first waves while CTAs running together still share one head's Q, dO
  // and dQ accumulator rows in L2.
  int u, kvh;
  {
    const int L = blockIdx.x;
    const int nh = prm.n_heavy;
    if (L < nh * prm.Hkv) {
      u = prm.heavy[L / prm.Hkv];
      kvh = L % prm.Hkv;
    } else {
      const int rest = prm.nkt - nh;
      const int L2 = L - nh * prm.Hkv;
      kvh = L2 / rest;
      u = L2 % rest;
      for (int k = 0; k < nh; ++k) u += (prm.heavy[k] <= u) ? 1 : 0;  // skip the heavy tiles
    }
  }
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
  const size_t hrow0 = prm.cu_seqlens != nullptr ? (size_t)base : (size_t)b * prm.H * prm.S;
  const long long lin0 = prm.cu_seqlens != nullptr ? (long long)base : (long long)b * prm.S;
  const int G = prm.H / prm.Hkv;
  const int j_lo = 2 * u;
  if (j_lo >= nqb) return;  // past a shorter sequence's last tile (uniform exit)
  const int j_hi = imin(2 * u + 1, nqb - 1);
  const QIter qit(prm.pat, j_lo, j_hi, nqb);
  const int cnt = qit.count();
  const int N = G * cnt;
  constexpr bool split = SPLIT;
  unsigned int* err = prm.err;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1 + 256);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&dp_full[s], 1);
      mbar_init(&p_full[s], 256);
      mbar_init(&ds_full[s], 256);
      mbar_init(&dq_full[s], 1);
      mbar_init(&dq_free[s], 128);
      mbar_init(&dss_free[s], 1);
      mbar_init(&s_read[s], 256);
      mbar_init(&dp_read[s], 256);
    }
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
      mbar_arrive_expect_tx(kv_full, 2 * L::KV_BYTES);
      // Two 64-row boxes per panel; rows past the sequence stay masked.
      for (int hb = 0; hb < 2; ++hb)
        for (int p = 0; p < DP; ++p) {
          tma_load_4d(smem + L::OFF_K + p * 16384 + hb * 8192, &tmK, kv_full, 64 * p, kvh, base + 128 * u + 64 * hb,
                      bc);
          tma_load_4d(smem + L::OFF_V + p * 16384 + hb * 8192, &tmV, kv_full, 64 * p, kvh, base + 128 * u + 64 * hb,
                      bc);
        }
      for (int n = 0; n < N; ++n) {
        const int h = kvh * G + n / cnt;
        const int i = qit.first_blk + n % cnt;
        const int st = n % QS;
        const uint32_t use = (uint32_t)(n / QS);
        if (use > 0 && !mbar_wait(&q_empty[st], (use - 1) & 1, abort_flag, err, kErrBwdWait)) break;
        mbar_arrive_expect_tx(&q_full[st], 2 * L::QB_BYTES + 512);
        for (int p = 0; p < DP; ++p) {
          tma_load_4d(smem + L::OFF_Q + st * L::QB_BYTES + p * 8192, &tmQ, &q_full[st], 64 * p, h, base + 64 * i, bc);
          tma_load_4d(smem + L::OFF_DO + st * L::QB_BYTES + p * 8192, &tmdO, &q_full[st], 64 * p, h, base + 64 * i, bc);
        }
        const size_t row = hrow0 + (size_t)h * prm.S + 64 * (size_t)i;
        bulk_load(smem + L::OFF_LSE + st * 256, prm.lse + row, 256, &q_full[st]);
        bulk_load(smem + L::OFF_DEL + st * 256, prm.delta + row, 256, &q_full[st]);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_g = idesc_bf16(128, D, false, true);
      constexpr uint32_t idesc_q = idesc_bf16(D, 64, true, true);
      const uint32_t aK = sbase + L::OFF_K, aV = sbase + L::OFF_V;
      auto grad = [&](int m) -> bool {
        const int bb = m & 1;
        const int st = m % QS;
        const uint32_t use = (uint32_t)(m >> 1);
        const uint32_t tb = tmem + L::T_BUF + 128 * bb;
        const uint32_t aQ = sbase + L::OFF_Q + st * L::QB_BYTES;
        const uint32_t aDO = sbase + L::OFF_DO + st * L::QB_BYTES;
        const uint32_t aDS = sbase + L::OFF_DST + bb * L::PT_BYTES;
        if (!mbar_wait(&p_full[bb], use & 1, abort_flag, err, kErrBwdWait)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts(tmem + L::T_DV, tb + 8 * kk, sdesc_sw128(aDO + kk * 2048, 8192, 1024), idesc_g,
                    (m > 0 || kk > 0) ? 1u : 0u);
        if (split) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_ss(tmem + L::T_DV, sdesc_sw128(sbase + L::OFF_PL + kk * 32, 16, 1024),
                      sdesc_sw128(aDO + kk * 2048, 8192, 1024), idesc_g, 1u);
        }
        if (!mbar_wait(&ds_full[bb], use & 1, abort_flag, err, kErrBwdWait)) return false;
        tc_fence_after();
        // dK and dQ^T are independent accumulations: interleave their k-steps so
        // the tensor pipe has two chains in flight (one dependent chain of
        // M=128 MMAs is latency-bound).
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          tc_mma_ts(tmem + L::T_DK, tb + 96 + 8 * kk, sdesc_sw128(aQ + kk * 2048, 8192, 1024), idesc_g,
                    (m > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            const int kq = 2 * kk + q2;
            tc_mma_ss(tb + 32, sdesc_sw128(aK + kq * 2048, 16384, 1024), sdesc_sw128(aDS + kq * 2048, 8192, 1024),
                      idesc_q, kq > 0 ? 1u : 0u);
          }
        }
        if (split) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_ss(tmem + L::T_DK, sdesc_sw128(sbase + L::OFF_DSL + kk * 32, 16, 1024),
                      sdesc_sw128(aQ + kk * 2048, 8192, 1024), idesc_g, 1u);
        }
        tc_commit(&dq_full[bb]);
        tc_commit(&dss_free[bb]);
        tc_commit(&q_empty[st]);
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, err, kErrBwdWait);
      for (int n = 0; n < N && ok; ++n) {
        const int bb = n & 1;
        const int st = n % QS;
        const uint32_t tb = tmem + L::T_BUF + 128 * bb;
        if (!mbar_wait(&q_full[st], (uint32_t)(n / QS) & 1, abort_flag, err, kErrBwdWait)) { ok = false; break; }
        // Buffer bb last held step n-2: its dQ^T must have been drained.
        if (n >= 2 && !mbar_wait(&dq_free[bb], (uint32_t)((n >> 1) - 1) & 1, abort_flag, err, kErrBwdWait)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aQ = sbase + L::OFF_Q + st * L::QB_BYTES;
        const uint32_t aDO = sbase + L::OFF_DO + st * L::QB_BYTES;
        // S^T and dP^T are independent: interleave their k-steps (two chains in flight).
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t kb = (kk >> 2) * 8192 + (kk & 3) * 32;
          tc_mma_ss(tb, sdesc_sw128(aK + ka, 16, 1024), sdesc_sw128(aQ + kb, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          tc_mma_ss(tb + 64, sdesc_sw128(aV + ka, 16, 1024), sdesc_sw128(aDO + kb, 16, 1024), idesc_s,
                    kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[bb]);
        tc_commit(&dp_full[bb]);
        if (n >= 1 && !grad(n - 1)) { ok = false; break; }
      }
      if (ok && N > 0) ok = grad(N - 1);
      tc_commit(acc_done);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P / dS warps
    // Two warps per TMEM lane quarter: warp w owns KV rows 32 (w % 4) .. +31
    // and query columns [32 (w / 4), +32) of the step.
    const int hf = warp >> 2;
    const int c0 = 32 * hf;
    const int r = (warp & 3) * 32 + lane;  // KV row of the tile == TMEM lane
    const int kvb = 2 * u + (r >> 6);
    const int rr = r & 63;
    const bool krow_live = kvb < nqb;
    const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = prm.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    int n = 0;
    for (; n < N; ++n) {
      const int i = qit.first_blk + n % cnt;
      const int st = n % QS;
      const int bb = n & 1;
      const uint32_t use = (uint32_t)(n >> 1);
      const uint32_t tl = t_lane + L::T_BUF + 128 * bb;
      const bool vis = krow_live && in_list(prm.pat, i, kvb);  // warp-uniform
      const bool diag = (i == kvb);
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[st], (uint32_t)(n / QS) & 1, abort_flag, err, kErrBwdWait)))
        break;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[bb], use & 1, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      float pf[32];
      {
        uint32_t sr[32];
        tmem_ld32(tl + c0, sr);
        tc_fence_before();
        mbar_arrive(&s_read[bb]);
        const float* lse = s_lse + st * 64 + c0;
        if (vis) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float p = ex2_approx(fmaf(__uint_as_float(sr[e]), sl2, -lse[e] * kLog2e));
            pf[e] = (diag && c0 + e < rr) ? 0.f : p;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) pf[e] = 0.f;
        }
      }
      // P^T goes over S^T columns [0, 32), which hold S^T the other warp of this
      // lane quarter may still be reading: wait until every warp has read S^T.
      if (!__all_sync(0xffffffffu, mbar_wait(&s_read[bb], use & 1, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      {
        uint32_t hi[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) hi[e] = pack_bf16x2(pf[2 * e], pf[2 * e + 1]);
        tmem_st16(tl + 16 * hf, hi);  // P^T over S^T columns [0, 32)
        if (split) {
          // The single residual buffer is free once the gradient GEMMs of step n-1 completed.
          if (n >= 1 && !__all_sync(0xffffffffu, mbar_wait(&dss_free[bb ^ 1], (uint32_t)((n - 1) >> 1) & 1,
                                                           abort_flag, err, kErrBwdWait)))
            break;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              lo[e] = pack_bf16x2(pf[8 * c + 2 * e] - __uint_as_float(hi[4 * c + e] << 16),
                                  pf[8 * c + 2 * e + 1] - __uint_as_float(hi[4 * c + e] & 0xffff0000u));
            st_shared_v4(sbase + L::OFF_PL + sw128_offset(r, 4 * hf + c), lo[0], lo[1], lo[2], lo[3]);
          }
          fence_async_smem();
        }
      }
      tc_fence_before();
      mbar_arrive(&p_full[bb]);
      if (!__all_sync(0xffffffffu, mbar_wait(&dp_full[bb], use & 1, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      {
        uint32_t dpr[32];
        tmem_ld32(tl + 64 + c0, dpr);
        tc_fence_before();
        mbar_arrive(&dp_read[bb]);
        const float* del = s_del + st * 64 + c0;
#pragma unroll
        for (int e = 0; e < 32; ++e) pf[e] = pf[e] * (__uint_as_float(dpr[e]) - del[e]);  // pf now holds dS^T
      }
      // dS^T goes over dP^T columns [32, 64): same hazard as for P^T.
      if (!__all_sync(0xffffffffu, mbar_wait(&dp_read[bb], use & 1, abort_flag, err, kErrBwdWait))) break;
      tc_fence_after();
      uint32_t hi[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) hi[e] = pack_bf16x2(pf[2 * e], pf[2 * e + 1]);
      tmem_st16(tl + 96 + 16 * hf, hi);  // dS^T over dP^T columns [32, 64)
      // The shared dS^T buffer bb last fed dQ^T of step n-2.
      if (n >= 2 &&
          !__all_sync(0xffffffffu, mbar_wait(&dss_free[bb], (use - 1) & 1, abort_flag, err, kErrBwdWait)))
        break;
      const uint32_t drow = sbase + L::OFF_DST + bb * L::PT_BYTES;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        st_shared_v4(drow + sw128_offset(r, 4 * hf + c), hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
        if (split) {
          uint32_t lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            lo[e] = pack_bf16x2(pf[8 * c + 2 * e] - __uint_as_float(hi[4 * c + e] << 16),
                                pf[8 * c + 2 * e + 1] - __uint_as_float(hi[4 * c + e] & 0xffff0000u));
          st_shared_v4(sbase + L::OFF_DSL + sw128_offset(r, 4 * hf + c), lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&ds_full[bb]);
      mbar_arrive(&q_empty[st]);
    }

    // ------------------------------------------------------------ dK, dV epilogue
    // Warp (quarter, half) writes rows of its quarter, columns [half * D/2, +D/2).
    bool ok = (n == N) && !*abort_flag;
    if (ok) ok = mbar_wait(acc_done, 0, abort_flag, err, kErrBwdWait);
    ok = __all_sync(0xffffffffu, ok);
    constexpr int CH = D / 64;  // 32-column chunks per half
    if (ok && prm.grad_f32) {
      // fp32 gradients: each thread stores its part of a KV row straight from TMEM.
      tc_fence_after();
      const int krow = 128 * u + r;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tcol = which == 0 ? L::T_DV : L::T_DK;
        const float mul = which == 0 ? 1.f : prm.scale;
        float* dst = (which == 0 ? prm.dv_f32 : prm.dk_f32) + (((size_t)lin0 + krow) * prm.Hkv + kvh) * D;
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          const int col = hf * (D / 2) + 32 * q;
          uint32_t o[32];
          tmem_ld32(t_lane + tcol + col, o);
          if (krow < len) {
            float4* d4 = reinterpret_cast<float4*>(dst + col);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(o[4 * e]) * mul, __uint_as_float(o[4 * e + 1]) * mul,
                                  __uint_as_float(o[4 * e + 2]) * mul, __uint_as_float(o[4 * e + 3]) * mul);
          }
        }
      }
    } else if (ok) {
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tcol = which == 0 ? L::T_DV : L::T_DK;
        const float mul = which == 0 ? 1.f : prm.scale;
        const uint32_t dst = sbase + (which == 0 ? L::OFF_V : L::OFF_K);
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          const int col = hf * (D / 2) + 32 * q;
          uint32_t o[32];
          tmem_ld32(t_lane + tcol + col, o);
          const uint32_t panel = dst + (uint32_t)(col >> 6) * 16384;
          const int cq = (col & 63) >> 3;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float* f = reinterpret_cast<const float*>(&o[8 * q4]);
            st_shared_v4(panel + sw128_offset(r, cq + q4), pack_bf16x2(f[0] * mul, f[1] * mul),
                         pack_bf16x2(f[2] * mul, f[3] * mul), pack_bf16x2(f[4] * mul, f[5] * mul),
                         pack_bf16x2(f[6] * mul, f[7] * mul));
          }
        }
      }
    }
    fence_async_smem();
    named_bar_sync(1, 256);
    if (threadIdx.x == 0 && !*abort_flag && !prm.grad_f32) {
      // One 64-row box per block inside the sequence: never into the next packed sequence.
      for (int hb = 0; hb < (2 * u + 1 < nqb ? 2 : 1); ++hb)
        for (int p = 0; p < DP; ++p) {
          tma_store_4d(&tmdV, smem + L::OFF_V + p * 16384 + hb * 8192, 64 * p, kvh, base + 128 * u + 64 * hb, bc);
          tma_store_4d(&tmdK, smem + L::OFF_K + p * 16384 + hb * 8192, 64 * p, kvh, base + 128 * u + 64 * hb, bc);
        }
      bulk_commit();
      bulk_wait_all();
    }
  } else {
    // ------------------------------------------------------------ dQ drain warps 10-13
    const int quarter = warp & 3;
    // dQ^T row (= d) held by this thread: M = D rows; for M = 64 the rows sit in
    // lanes 0-15 of each 32-lane quarter.
    const int d = (D == 128) ? quarter * 32 + lane : quarter * 16 + lane;
    const bool dvalid = (D == 128) || lane < 16;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int n = 0; n < N; ++n) {
      const int h = kvh * G + n / cnt;
      const int i = qit.first_blk + n % cnt;
      const int bb = n & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&dq_full[bb], (uint32_t)(n >> 1) & 1, abort_flag, err, kErrBwdWait)))
        break;
      tc_fence_after();
      uint32_t v[64];
      tmem_ld64(t_lane + L::T_BUF + 128 * bb + 32, v);
      tc_fence_before();
      mbar_arrive(&dq_free[bb]);
      if (dvalid) {
        float* dst = prm.dq_acc + (hrow0 + (size_t)h * prm.S + 64 * (size_t)i) * D + d;
#pragma unroll
        for (int c = 0; c < 64; ++c) red_add_f32(dst + (size_t)c * D, __uint_as_float(v[c]));
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

template <int D, bool SPLIT>
static cudaError_t launch_bwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                   const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                                   const BwdParams& prm, int B, cudaStream_t stream) {
  using L = BwdLayout<D, SPLIT>;
  static_assert(L::ALLOC <= 232448, "shared memory budget");
  cudaError_t e =
      cudaFuncSetAttribute(lg_bwd_kernel<D, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(prm.nkt * prm.Hkv, B);
  lg_bwd_kernel<D, SPLIT><<<grid, 448, L::ALLOC, stream>>>(tq, tk, tv, tdo, tdk, tdv, prm);
  return cudaGetLastError();
}

cudaError_t launch_bwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const BwdParams& prm,
                       int B, cudaStream_t stream) {
  // Head dim 128 (with or without query-head groups) runs the 128-row-step
  // kernel; this one serves head dim 64.
  if (D == 128) return launch_bwd128(tq, tk, tv, tdo, tdk, tdv, prm, B, stream);
  if (prm.split_lo) return launch_bwd_impl<64, true>(tq, tk, tv, tdo, tdk, tdv, prm, B, stream);
  return launch_bwd_impl<64, false>(tq, tk, tv, tdo, tdk, tdv, prm, B, stream);
}

}  // namespace lg
