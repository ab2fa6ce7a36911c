// lh_noalloc.cu -- lh_subseq_attn_bwd_noalloc: the sub-sequence attention
// backward for callers that can neither allocate device memory nor pass a
// workspace.  Its only scratch (the per-row softmax statistics, -lse*log2(e)
// and -rowsum(dos * os), two floats per row with rows padded to whole
// 128-row tiles) lives in a fixed, file-scope device array instead of caller
// memory.  It runs exactly the kernels lh_subseq_attn_bwd runs (the shared
// attn_bwd helper), so its results are bitwise those of the workspace call.
//
// Costs and limits, stated for users of the library:
//   * every GPU that loads this library holds 2 * kNoAllocRows floats (8 MiB)
//     for this array until the process exits, whether or not the call is used;
//   * one call handles at most kNoAllocRows padded rows (B * H * ceil(S/128) *
//     128); larger shapes are rejected with LH_ERR_WORKSPACE before anything
//     is enqueued;
//   * all calls on a device share the one array: two calls whose kernels
//     overlap on the GPU (different streams, no ordering between them) race
//     on it.  Calls ordered on one stream are safe.  The array keeps the last
//     call's contents; every element a call reads was first written by that
//     same call, so nothing needs clearing;
//   * the first call in each CUDA context of a device (normally one per
//     device; a new one after cudaDeviceReset) looks up the array's device
//     address (cudaGetSymbolAddress, with that device current) and caches it
//     under the context's unique id; make that first call before any stream
//     capture.
#include <cuda.h>

#include <mutex>

#include "lh_internal.cuh"

namespace lh {
namespace {

constexpr size_t kNoAllocRows = (size_t)1 << 20;

static __device__ __align__(256) float g_noalloc_stats[2 * kNoAllocRows];

// The current context's process-unique id (cuCtxGetId never reuses an id, unlike
// a CUcontext handle, which a context created after a reset may get again), or
// 0 when there is no current context or the driver lacks the call.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

constexpr int kMaxDevices = 64;
struct CachedAddress {
  unsigned long long ctx_id = 0;  // 0: nothing cached
  float* ptr = nullptr;
};
CachedAddress g_cache[kMaxDevices];
std::mutex g_cache_mutex;

// Device address of the array in the current context of the current device
// (host code cannot use the symbol itself: in host code it names a host-side
// stand-in, not device memory).
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_cache_mutex);
  const unsigned long long id = current_context_id();
  if (id != 0 && g_cache[dev].ctx_id == id) {
    *out = g_cache[dev].ptr;
    return cudaSuccess;
  }
  float* p = nullptr;
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_stats);
  if (e != cudaSuccess) return e;
  // the lookup makes the device's context current if it was not; key the cache
  // on it (no id: nothing is cached and every call looks the address up)
  g_cache[dev].ctx_id = current_context_id();
  g_cache[dev].ptr = p;
  *out = p;
  return cudaSuccess;
}

inline bool al16(const void* p) { return p && (((uintptr_t)p) & 15u) == 0; }

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" lh_status lh_subseq_attn_bwd_noalloc(const lh_shape* shape, const void* qs,
                                                const void* ks, const void* vs, const void* os,
                                                const float* lse, const void* dos, float scale,
                                                float* dqs, float* dks, float* dvs,
                                                lh_stream_t stream) {
  lh_status s = lh_validate(shape, LH_BF16);
  if (s != LH_OK) return s;
  if (!al16(qs) || !al16(ks) || !al16(vs) || !al16(os) || !al16(lse) || !al16(dos) ||
      !al16(dqs) || !al16(dks) || !al16(dvs))
    return LH_ERR_INVALID_ARG;
  const Geom g = make_geom(*shape);
  if (attn_stats_floats(g) > 2 * kNoAllocRows) return LH_ERR_WORKSPACE;
  float* stats = nullptr;
  if (noalloc_scratch(&stats) != cudaSuccess) return LH_ERR_CUDA;
  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)g.d);
  return attn_bwd(g, static_cast<const __half*>(qs), static_cast<const __half*>(ks),
                  static_cast<const __half*>(vs), static_cast<const __half*>(os), lse,
                  static_cast<const __half*>(dos), sc, dqs, dks, dvs, stats, stream);
}
