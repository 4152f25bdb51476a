// decode_noalloc.cu -- lg_sparse_decode_noalloc: split-KV decode that allocates nothing.
//
// Some callers cannot hand the library a workspace: a host framework or plugin
// that owns all device memory through its own pool and forbids side
// allocations, a latency-critical decode loop where cudaMalloc / cudaFree
// would synchronise the device and stall every other stream, or a thin C / FFI
// caller with no device allocator of its own. This entry point runs the same
// validation, split rule and decode kernel as lg_sparse_decode (decode_call in
// api.cu), but keeps the split partials and tickets in a fixed array compiled
// into the library, so the caller passes only its inputs and outputs. The
// paper has no counterpart; this is a deployment convenience.
//
// The array is LG_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) per device, held from
// the moment the library is loaded on a device until the process exits. Its
// name is a host-side stand-in in host code, not a device address, so the
// device address is looked up with cudaGetSymbolAddress (with the device
// current) on the first call on a device and cached together with the
// device's current context; a new context (after cudaDeviceReset) triggers a
// fresh look-up. Every call shares the array and it keeps the last call's
// contents: the tickets are cleared on the stream at every call, and calls
// that overlap on the GPU (other streams, other host threads) race on it --
// serialise them.
#include <cudaTypedefs.h>

#include <mutex>

#include "lg_kernels.h"

static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[LG_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxNoallocDevices = 64;

// The driver's cuCtxGetCurrent, reached through the runtime (nothing links libcuda).
PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  });
  return fn;
}

// Device address of the scratch array on device dev, which is current.
unsigned char* scratch_address(int dev, lg_status_t* st) {
  static std::mutex mu;
  static unsigned char* addr[kMaxNoallocDevices] = {};
  static CUcontext ctx_of[kMaxNoallocDevices] = {};
  *st = LG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxNoallocDevices) return nullptr;
  PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return nullptr;
  // cudaSetDevice makes the device's primary context current (and creates it if needed).
  if (cudaSetDevice(dev) != cudaSuccess) return nullptr;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || ctx_of[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = static_cast<unsigned char*>(p);
    ctx_of[dev] = ctx;
  }
  *st = LG_OK;
  return addr[dev];
}

}  // namespace

extern "C" lg_status_t lg_sparse_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                const int32_t* cache_lens, void* o, int32_t o_dtype, float* lse,
                                                int32_t B, int32_t H, int32_t Hkv, int32_t D, int32_t Lmax,
                                                int32_t num_splits, float scale, lg_stream_t stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The scratch address belongs to the current device, so the stream and the
  // query must be on it too: a kernel given another device's array would read
  // and write memory that is not its own.
  int dev = -1, sdev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LG_ERR_CUDA;
  if (cudaStreamGetDevice(s, &sdev) != cudaSuccess) return LG_ERR_INVALID_ARG;
  if (sdev != dev) return LG_ERR_INVALID_ARG;
  if (q != nullptr) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, q) != cudaSuccess) return LG_ERR_INVALID_ARG;
    if ((a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) || a.device != dev)
      return LG_ERR_INVALID_ARG;
  }
  lg_status_t st = LG_OK;
  unsigned char* scratch = scratch_address(dev, &st);
  if (st != LG_OK) return st;
  // Same validation, split rule and launch as lg_sparse_decode. An automatic
  // split count is lowered until the partials fit the array; an explicit one
  // that does not fit returns LG_ERR_WORKSPACE before anything is launched.
  return lg::decode_call(q, k_cache, v_cache, cache_lens, nullptr, 0, 0, o, o_dtype, lse, B, H, Hkv, D, Lmax,
                         num_splits, scale, scratch, LG_DECODE_NOALLOC_SCRATCH_BYTES, true, s);
}
