// decode_noalloc.cu -- lg_sparse_decode_noalloc: split-KV decode that allocates nothing.
//
// Some callers cannot hand the library a workspace: a host framework or plugin
// that owns all device memory through its own pool and forbids side
// allocations, a latency-critical decode loop where cudaMalloc / cudaFree
// would synchronise the device and stall every other stream, or a thin C / FFI
// caller with no device allocator of its own. This entry point runs the same
// decode kernel as lg_sparse_decode, but keeps the split partials and tickets
// in a fixed array compiled into the library, so the caller passes only its
// inputs and outputs. The paper has no counterpart; this is a deployment
// convenience.
//
// The array is LG_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) per device, held from
// the moment the library is loaded on a device until the process exits. Its
// name is a host-side stand-in in host code, not a device address, so the
// device address is looked up with cudaGetSymbolAddress once per device (with
// that device current) on the first call, and cached. Every call shares the
// array and it keeps the last call's contents: the tickets are cleared on the
// stream at every call, and calls that overlap on the GPU (other streams, other
// host threads) race on it -- serialise them.
#include <mutex>

#include "lg_kernels.h"

static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[LG_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxNoallocDevices = 64;

size_t r256(size_t x) { return (x + 255) & ~size_t(255); }

size_t scratch_need(int B, int H, int Hkv, int D, int ns) {
  if (ns <= 1) return 0;
  return r256((size_t)B * H * ns * D * 4) + r256((size_t)B * H * ns * 4) + r256((size_t)B * Hkv * 4);
}

// Device address of the scratch array on the current device; resolved on the
// first call per device, with that device current.
unsigned char* scratch_address(lg_status_t* st) {
  static std::mutex mu;
  static unsigned char* addr[kMaxNoallocDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoallocDevices) {
    *st = LG_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *st = LG_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = static_cast<unsigned char*>(p);
  }
  *st = LG_OK;
  return addr[dev];
}

}  // namespace

extern "C" lg_status_t lg_sparse_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                const int32_t* cache_lens, void* o, float* lse, int32_t B, int32_t H,
                                                int32_t Hkv, int32_t D, int32_t Lmax, int32_t num_splits,
                                                float scale, lg_stream_t stream) {
  if (!q || !k_cache || !v_cache || !cache_lens || !o) return LG_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0 || num_splits < 0) return LG_ERR_INVALID_ARG;
  if (H % Hkv != 0) return LG_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return LG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return LG_ERR_UNSUPPORTED;
  const int G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return LG_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return LG_ERR_UNSUPPORTED;
  const auto mis16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis16(q) || mis16(k_cache) || mis16(v_cache) || mis16(o) || (reinterpret_cast<uintptr_t>(cache_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return LG_ERR_UNSUPPORTED;

  // Same split rule as lg_sparse_decode; in automatic mode the split count is
  // lowered until the partials fit the fixed array, an explicit count that does
  // not fit is rejected.
  int32_t ns = 1;
  lg_status_t st = lg_sparse_decode_splits(B, H, Hkv, D, Lmax, num_splits, &ns);
  if (st != LG_OK) return st;
  if (scratch_need(B, H, Hkv, D, ns) > (size_t)LG_DECODE_NOALLOC_SCRATCH_BYTES) {
    if (num_splits > 0) return LG_ERR_WORKSPACE;
    while (ns > 1 && scratch_need(B, H, Hkv, D, ns) > (size_t)LG_DECODE_NOALLOC_SCRATCH_BYTES) --ns;
  }
  int rps = (Lmax + ns - 1) / ns;
  ns = (Lmax + rps - 1) / rps;

  unsigned char* scratch = scratch_address(&st);
  if (st != LG_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lg::DecodeParams prm;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.lens = cache_lens;
  prm.o = o;
  prm.lse = lse;
  prm.part_o = nullptr;
  prm.part_lse = nullptr;
  prm.tickets = nullptr;
  if (ns > 1) {
    unsigned char* w = scratch;
    prm.part_o = reinterpret_cast<float*>(w);
    w += r256((size_t)B * H * ns * D * 4);
    prm.part_lse = reinterpret_cast<float*>(w);
    w += r256((size_t)B * H * ns * 4);
    prm.tickets = reinterpret_cast<unsigned int*>(w);
    // Tickets must start at zero; the array keeps whatever the last call left.
    if (cudaMemsetAsync(prm.tickets, 0, (size_t)B * Hkv * 4, s) != cudaSuccess) return LG_ERR_CUDA;
  }
  prm.B = B;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.Lmax = Lmax;
  prm.ns = ns;
  prm.rows_per_split = rps;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = nullptr;  // the decode kernel has no device-side waits
  return lg::launch_decode(D, G, prm, s) == cudaSuccess ? LG_OK : LG_ERR_CUDA;
}
