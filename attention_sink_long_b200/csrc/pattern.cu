// pattern.cu -- device-side run of the block iterators the attention kernels use,
// recorded so the host can compare it bit for bit with the CSR / CSC expansion
// ("A Little Goes a Long Way", atlas.scime.ai summary, "Approach": static,
// block-wise access).
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

__global__ void lg_pattern_iterate_kernel(lg_pattern_t p, int nqb, int tile_blocks, int transpose, int32_t* out,
                                          int cap) {
  const int ntiles = (nqb + tile_blocks - 1) / tile_blocks;
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= ntiles) return;
  const int lo = u * tile_blocks;
  const int hi = imin(lo + tile_blocks - 1, nqb - 1);
  int32_t* dst = out + (size_t)u * (cap + 1);
  int n = 0;
  if (!transpose) {
    const KvIter it(p, lo, hi);
    for (int j = it.first(); j >= 0; j = it.next(j)) {
      int mem = 0;
      for (int t = 0; t <= hi - lo; ++t)
        if (in_list(p, lo + t, j)) mem |= 1 << t;
      if (n < cap) dst[1 + n] = (j << 2) | mem;
      ++n;
    }
    // The kernels size their loops with count(); flag any disagreement.
    if (n != it.count()) n = -1 - n;
  } else {
    const QIter it(p, lo, hi, nqb);
    for (int i = it.first_blk; i <= it.last_blk; ++i) {
      int mem = 0;
      for (int t = 0; t <= hi - lo; ++t)
        if (in_list(p, i, lo + t)) mem |= 1 << t;
      if (n < cap) dst[1 + n] = (i << 2) | mem;
      ++n;
    }
    if (n != it.count()) n = -1 - n;
  }
  dst[0] = n;
}

cudaError_t launch_pattern_iterate(const lg_pattern_t& p, int seqlen, int tile_blocks, int transpose, int32_t* out,
                                   int cap, cudaStream_t stream) {
  const int nqb = seqlen / p.block_size;
  const int ntiles = (nqb + tile_blocks - 1) / tile_blocks;
  lg_pattern_iterate_kernel<<<(ntiles + 127) / 128, 128, 0, stream>>>(p, nqb, tile_blocks, transpose, out, cap);
  return cudaGetLastError();
}

}  // namespace lg
