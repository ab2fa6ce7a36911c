// lh_noalloc.cu -- lh_subseq_attn_bwd_noalloc: the sub-sequence attention
// backward for callers that can neither allocate device memory nor pass a
// workspace.  Its only scratch (the per-row softmax statistics, -lse*log2(e)
// and -rowsum(dos * os), two floats per row with rows padded to whole
// 128-row tiles) lives in a fixed, file-scope device array instead of caller
// memory.
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
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make
//     that first call before any stream capture.
#include <atomic>

#include "lh_internal.cuh"

namespace lh {
namespace {

constexpr size_t kNoAllocRows = (size_t)1 << 20;

static __device__ __align__(256) float g_noalloc_stats[2 * kNoAllocRows];

constexpr int kMaxDevices = 64;
std::atomic<float*> g_noalloc_ptr[kMaxDevices];

// Device address of the array on the current device (host code cannot use the
// symbol itself: in host code it names a host-side stand-in, not device memory).
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  float* p = g_noalloc_ptr[dev].load();
  if (!p) {
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_stats);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev].store(p);
  }
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
  auto* q = static_cast<const __half*>(qs);
  auto* k = static_cast<const __half*>(ks);
  auto* v = static_cast<const __half*>(vs);
  auto* o = static_cast<const __half*>(os);
  auto* go = static_cast<const __half*>(dos);
  if (launch_attn_stats(g, o, go, lse, stats, stream) != cudaSuccess) return LH_ERR_CUDA;
  cudaError_t e = attn_bwd_uses_tc()
                      ? launch_attn_bwd_tc(g, q, k, v, go, stats, sc, dqs, dks, dvs, stream)
                      : launch_attn_bwd_mma(g, q, k, v, go, stats, sc, dqs, dks, dvs, stream);
  return e == cudaSuccess ? LH_OK : LH_ERR_CUDA;
}
