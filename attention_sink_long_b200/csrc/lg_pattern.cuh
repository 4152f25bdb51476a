// lg_pattern.cuh -- the static block pattern and its closed-form block iterators.
//
// "A Little Goes a Long Way" (LongGen), Abstract insight 1 and the atlas.scime.ai
// summary, "Approach": sparse layers attend to sink blocks, a local window of
// recent blocks and strided blocks, with static, block-wise access. Because the
// pattern is static and made of at most three arithmetic ranges, the per-query-
// block KV-block list (and its transpose) is enumerated here in closed form
// instead of being stored: the kernels visit exactly the listed blocks, in
// increasing order, and never touch a masked block.
#pragma once

#include <stdint.h>

#include "../../include/lg_attn.h"

#if defined(__CUDACC__)
#define LG_HD __host__ __device__ __forceinline__
#else
#define LG_HD inline
#endif

namespace lg {

LG_HD int imin(int a, int b) { return a < b ? a : b; }
LG_HD int imax(int a, int b) { return a > b ? a : b; }
LG_HD int ceil_div_nonneg(int a, int b) { return (a + b - 1) / b; }

// Is KV block j in the list of query block i?
LG_HD bool in_list(const lg_pattern_t& p, int i, int j) {
  if (j < 0 || j > i) return false;
  if (j < p.sink_blocks) return true;
  if (i - j < p.local_blocks) return true;
  if (p.stride > 0 && (j % p.stride) == 0) return true;
  return false;
}

// Union of the KV-block lists of the consecutive query blocks [i_lo, i_hi], in
// increasing order: sink blocks below the window, strided blocks below the
// window, then the window [i_lo - local + 1, i_hi] (which covers every
// diagonal). next(j) is the smallest listed block > j, or -1.
struct KvIter {
  int lo, hi, sink, stride;

  LG_HD KvIter(const lg_pattern_t& p, int i_lo, int i_hi) {
    const long long w = (long long)i_lo - (long long)p.local_blocks + 1;
    lo = w < 0 ? 0 : (int)w;
    hi = i_hi;
    sink = p.sink_blocks;
    stride = p.stride;
  }
  LG_HD int first() const { return next(-1); }
  LG_HD int next(int j) const {
    const int c = j + 1;
    if (c >= lo) return c <= hi ? c : -1;
    if (c < sink) return c;
    if (stride > 0) {
      const int m = ceil_div_nonneg(c, stride) * stride;
      if (m < lo) return m;
    }
    return lo <= hi ? lo : -1;
  }
  LG_HD int count() const {
    const int a = imin(imax(sink, 0), lo);  // sink blocks strictly below the window
    int n = a;
    if (stride > 0) n += ceil_div_nonneg(lo, stride) - ceil_div_nonneg(a, stride);
    return n + (hi - lo + 1);
  }
  // The n-th listed block (0 <= n < count()) in closed form: the sink blocks
  // below the window, then the strided blocks below it, then the window.
  LG_HD int nth(int n) const {
    const int a = imin(imax(sink, 0), lo);
    if (n < a) return n;
    n -= a;
    if (stride > 0) {
      const int s0 = ceil_div_nonneg(a, stride);
      const int ns = ceil_div_nonneg(lo, stride) - s0;
      if (n < ns) return (s0 + n) * stride;
      n -= ns;
    }
    return lo + n;
  }
};

// The KvIter sequence grouped into chunks of two consecutive listed blocks
// (adjacent or not: a sink block pairs with the first window block, isolated
// strided blocks pair with each other), the last chunk holding one block when
// the list is odd. span(j, &nb, &j2) takes a chunk start j, sets nb to its
// block count and j2 to its second block (-1 when nb == 1) and returns the
// next chunk start (or -1).
struct KvChunks {
  KvIter it;
  LG_HD KvChunks(const lg_pattern_t& p, int i_lo, int i_hi) : it(p, i_lo, i_hi) {}
  LG_HD int first() const { return it.first(); }
  LG_HD int span(int j, int* nb, int* j2) const {
    const int n2 = it.next(j);
    if (n2 >= 0) {
      *nb = 2;
      *j2 = n2;
      return it.next(n2);
    }
    *nb = 1;
    *j2 = -1;
    return -1;
  }
};

// The backward's pairing of KV blocks into 128-row tiles. Blocks that every
// later query sees ("global": sink blocks and strided blocks) come first in
// ascending order, then the window-only ("local") blocks in ascending order;
// tile t holds elements 2t and 2t+1 of that sequence. Two global blocks, or two
// nearby local blocks, share nearly the same query range, so few rows of a
// tile are masked while the CTA walks it (pairing block 32a with 32a+1 instead
// would mask half the tile for most queries of a strided pattern).
struct BlockPairing {
  int nqb, sink, stride, local;
  int nG;  // global blocks below nqb
  LG_HD BlockPairing(const lg_pattern_t& p, int nqb_) : nqb(nqb_), sink(p.sink_blocks), stride(p.stride),
                                                        local(p.local_blocks) {
    const int s = imin(imax(sink, 0), nqb);
    nG = s;
    if (stride > 0 && s < nqb) nG += ceil_div_nonneg(nqb, stride) - ceil_div_nonneg(s, stride);
  }
  LG_HD bool is_global(int kb) const { return kb < sink || (stride > 0 && kb % stride == 0); }
  LG_HD int tiles() const { return (nqb + 1) / 2; }
  // n-th global block (n < nG).
  LG_HD int global_nth(int n) const {
    const int s = imin(imax(sink, 0), nqb);
    if (n < s) return n;
    return (ceil_div_nonneg(s, stride) + (n - s)) * stride;
  }
  // n-th local block (n < nqb - nG): blocks >= sink that are not multiples of stride.
  LG_HD int local_nth(int n) const {
    const int s = imin(imax(sink, 0), nqb);
    if (stride <= 0) return s + n;
    const int m0 = ceil_div_nonneg(s, stride) * stride;  // first multiple >= s
    if (n < m0 - s) return s + n;
    n -= m0 - s;
    // after m0, each period of `stride` blocks holds stride - 1 local blocks
    return m0 + (n / (stride - 1)) * stride + 1 + n % (stride - 1);
  }
  LG_HD int seq(int n) const { return n < nG ? global_nth(n) : local_nth(n - nG); }
  // Blocks of tile t: *x always, *y = -1 when the tile holds one block.
  LG_HD void pair(int t, int* x, int* y) const {
    *x = seq(2 * t);
    *y = 2 * t + 1 < nqb ? seq(2 * t + 1) : -1;
  }
  // Last query block that sees KV block kb.
  LG_HD int reach(int kb) const {
    if (is_global(kb)) return nqb - 1;
    const long long r = (long long)kb + local - 1;
    return (int)(r < nqb - 1 ? r : nqb - 1);
  }
};

// Union of the query-block lists (transpose) of the consecutive KV blocks
// [j_lo, j_hi], given nqb query blocks. A sink or strided KV block is seen by
// every later query block; any other by the local_blocks query blocks starting
// at itself. The union is the contiguous range [j_lo, last].
struct QIter {
  int first_blk, last_blk;

  LG_HD QIter(const lg_pattern_t& p, int j_lo, int j_hi, int nqb) {
    first_blk = j_lo;
    int last = -1;
    for (int j = j_lo; j <= j_hi; ++j) {
      const bool global = (j < p.sink_blocks) || (p.stride > 0 && (j % p.stride) == 0);
      const long long reach = global ? (long long)nqb - 1 : (long long)j + p.local_blocks - 1;
      const int r = (int)(reach < (long long)nqb - 1 ? reach : (long long)nqb - 1);
      last = imax(last, r);
    }
    last_blk = last;
  }
  LG_HD int count() const { return last_blk >= first_blk ? last_blk - first_blk + 1 : 0; }
};

}  // namespace lg
