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
template <int D>
__global__ void __launch_bounds__(256) lg_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         float* __restrict__ delta, float* __restrict__ dq_acc,
                                                         int B, int S, int H) {
  constexpr int TPR = D / 8;
  const long long rows = (long long)B * S * H;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = t / TPR;  // memory order of O: ((b * S + s) * H + h)
  const int c = (int)(t % TPR);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + 8 * c);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + row * D + 8 * c);
    const uint32_t aa[4] = {a.x, a.y, a.z, a.w};
    const uint32_t gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(aa[e] << 16), __uint_as_float(gg[e] << 16), acc);
      acc = fmaf(__uint_as_float(aa[e] & 0xffff0000u), __uint_as_float(gg[e] & 0xffff0000u), acc);
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
    float4* z = reinterpret_cast<float4*>(dq_acc + drow * D + 8 * c);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

cudaError_t launch_bwd_pre(const void* o, const void* dout, float* delta, float* dq_acc, int B, int S, int H, int D,
                           cudaStream_t stream) {
  const long long threads = (long long)B * S * H * (D / 8);
  const unsigned int blocks = (unsigned int)((threads + 255) / 256);
  if (D == 64)
    lg_bwd_pre_kernel<64><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                      static_cast<const __nv_bfloat16*>(dout), delta, dq_acc, B, S, H);
  else
    lg_bwd_pre_kernel<128><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                       static_cast<const __nv_bfloat16*>(dout), delta, dq_acc, B, S,
                                                       H);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 3. dQ = scale * dQ_acc, [B, H, S, D] fp32 -> [B, S, H, D] bf16.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) lg_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                        __nv_bfloat16* __restrict__ dq, float scale, int B, int S,
                                                        int H) {
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
  uint4 out;
  out.x = pack_bf16x2(x0.x * scale, x0.y * scale);
  out.y = pack_bf16x2(x0.z * scale, x0.w * scale);
  out.z = pack_bf16x2(x1.x * scale, x1.y * scale);
  out.w = pack_bf16x2(x1.z * scale, x1.w * scale);
  *reinterpret_cast<uint4*>(dq + row * D + 8 * c) = out;
}

cudaError_t launch_bwd_dq(const float* dq_acc, void* dq, float scale, int B, int S, int H, int D,
                          cudaStream_t stream) {
  const long long threads = (long long)B * S * H * (D / 8);
  const unsigned int blocks = (unsigned int)((threads + 255) / 256);
  if (D == 64)
    lg_bwd_dq_kernel<64><<<blocks, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), scale, B, S, H);
  else
    lg_bwd_dq_kernel<128><<<blocks, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), scale, B, S, H);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 2. main kernel -- not yet available.
// ---------------------------------------------------------------------------
cudaError_t launch_bwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const BwdParams& prm,
                       int B, cudaStream_t stream) {
  (void)D; (void)tq; (void)tk; (void)tv; (void)tdo; (void)tdk; (void)tdv; (void)prm; (void)B; (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace lg
