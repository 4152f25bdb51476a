// pattern.cu -- device-side run of the block iterators the attention kernels use,
// recorded so the host can compare it bit for bit with the CSR / CSC expansion
// ("A Little Goes a Long Way", atlas.scime.ai summary, "Approach": static,
// block-wise access).
#include "lg_kernels.h"
#include "lg_pattern.cuh"

namespace lg {

// One thread per tile. Entries are (block << 8) | membership: bit t of the
// membership says whether the entry is in the list of the tile's t-th block
// (mode 3: bit 0 / bit 1 for the tile's two paired KV blocks).
__global__ void lg_pattern_iterate_kernel(lg_pattern_t p, int nqb, int tile_blocks, int mode, int32_t* out, int cap) {
  const int ntiles = mode == 3 ? BlockPairing(p, nqb).tiles() : (nqb + tile_blocks - 1) / tile_blocks;
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= ntiles) return;
  int32_t* dst = out + (size_t)u * (cap + 1);
  int n = 0;
  auto put = [&](int32_t x) {
    if (n < cap) dst[1 + n] = x;
    ++n;
  };
  const int lo = u * tile_blocks;
  const int hi = imin(lo + tile_blocks - 1, nqb - 1);
  if (mode == 0) {  // forward: the union of the tile's query blocks' KV lists
    const KvIter it(p, lo, hi);
    for (int j = it.first(); j >= 0; j = it.next(j)) {
      int mem = 0;
      for (int t = 0; t <= hi - lo; ++t)
        if (in_list(p, lo + t, j)) mem |= 1 << t;
      put((j << 8) | mem);
    }
    // The kernels size their loops with count(); flag any disagreement.
    if (n != it.count()) n = -1 - n;
  } else if (mode == 1) {  // backward: the union of the tile's KV blocks' query lists
    const QIter it(p, lo, hi, nqb);
    for (int i = it.first_blk; i <= it.last_blk; ++i) {
      int mem = 0;
      for (int t = 0; t <= hi - lo; ++t)
        if (in_list(p, i, lo + t)) mem |= 1 << t;
      put((i << 8) | mem);
    }
    if (n != it.count()) n = -1 - n;
  } else if (mode == 2) {  // the forward's chunked walk: two entries per chunk, the second -1 for a lone block
    const KvChunks chunks(p, lo, hi);
    int nb = 1;
    for (int j = chunks.first(); j >= 0;) {
      int j2 = -1;
      const int jn = chunks.span(j, &nb, &j2);
      const int js[2] = {j, j2};
      for (int e = 0; e < 2; ++e) {
        if (e >= nb) {
          put(-1);
          continue;
        }
        int mem = 0;
        for (int t = 0; t <= hi - lo; ++t)
          if (in_list(p, lo + t, js[e])) mem |= 1 << t;
        put((js[e] << 8) | mem);
      }
      j = jn;
    }
  } else {  // mode 3: the backward's KV tile u: its paired blocks, the query range it walks, the walk
    const BlockPairing bp(p, nqb);
    int kx, ky;
    bp.pair(u, &kx, &ky);
    const int q_first = ky >= 0 ? imin(kx, ky) : kx;
    const int last = ky >= 0 ? imax(bp.reach(kx), bp.reach(ky)) : bp.reach(kx);
    put(kx);
    put(ky);
    put(q_first);
    put(last);
    for (int i = q_first; i <= last; ++i)
      put((i << 8) | (in_list(p, i, kx) ? 1 : 0) | (ky >= 0 && in_list(p, i, ky) ? 2 : 0));
  }
  dst[0] = n;
}

cudaError_t launch_pattern_iterate(const lg_pattern_t& p, int seqlen, int tile_blocks, int mode, int32_t* out, int cap,
                                   cudaStream_t stream) {
  const int nqb = seqlen / p.block_size;
  const int ntiles = mode == 3 ? BlockPairing(p, nqb).tiles() : (nqb + tile_blocks - 1) / tile_blocks;
  lg_pattern_iterate_kernel<<<(ntiles + 127) / 128, 128, 0, stream>>>(p, nqb, tile_blocks, mode, out, cap);
  return cudaGetLastError();
}

}  // namespace lg
