// bwd_sm100.cu -- LongGen sparse causal attention, training backward, for sm_100a.
//
// "A Little Goes a Long Way" (LongGen), atlas.scime.ai summary, "Approach"
// (training with a FlashAttention-2-based kernel) and "Key results" (1.55x
// training speedup at 128K). Three launches:
//   1. preprocess: Delta = rowsum(dO * O) per query row, and zero the fp32 dQ
//      accumulator;
//   2. main: KV-tile-parallel dK, dV with dQ accumulated through fp32
//      reductions (lg_bwd128_kernel, bwd128_sm100.cu);
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

cudaError_t launch_bwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const BwdParams& prm,
                       int B, cudaStream_t stream) {
  // Both head dims run the 128-row-step kernel (bwd128_sm100.cu).
  if (D != prm.D) return cudaErrorInvalidValue;
  return launch_bwd128(tq, tk, tv, tdo, tdk, tdv, prm, B, stream);
}

}  // namespace lg
