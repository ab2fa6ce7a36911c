// lh_api.cu -- the extern "C" entry points declared in include/lighthouse.h:
// host-side argument checks, the layout of the saved and workspace buffers,
// and the order in which the stage kernels are enqueued.
#include <atomic>
#include <cmath>

#include "lh_internal.cuh"

namespace lh {

Geom make_geom(const lh_shape& s) {
  Geom g;
  g.U = s.B * s.H;
  g.N = s.N;
  g.d = s.d;
  g.p = s.p;
  g.L = s.L;
  g.S = s.S;
  int64_t pw = 1, off = 0;
  for (int l = 0; l <= kMaxLevels; ++l) {
    g.pw[l] = pw;
    g.off[l] = off;
    if (l < s.L) off += s.N / pw;
    if (pw <= s.N) pw *= s.p;  // powers past the pyramid are never used to index
  }
  g.M = g.off[s.L];
  for (int l = s.L + 1; l <= kMaxLevels; ++l) g.off[l] = g.M;
  return g;
}

namespace {

std::atomic<int> g_attn_impl{-1};  // -1 automatic, 0 tcgen05, 1 mma.sync

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Sequential layout of named regions, each 256-byte aligned.
struct Layout {
  size_t off[12] = {};
  size_t total = 0;
  int n = 0;
  size_t add(size_t bytes) {
    off[n++] = total;
    total += align_up(bytes);
    return off[n - 1];
  }
};

enum SavedRegion { kIdx = 0, kPos, kSlot, kQs, kKs, kVs, kOs, kLse, kInvCnt, kNumSaved };

Layout saved_layout(const Geom& g) {
  Layout L;
  const size_t US = (size_t)g.U * g.S;
  L.add(US * 4);                       // idx
  L.add(US * 4);                       // pos
  L.add((size_t)g.U * g.M * 4);        // slot
  for (int i = 0; i < 4; ++i) L.add(US * g.d * 2);  // qs ks vs os
  L.add(US * 4);                       // lse
  L.add((size_t)g.U * g.N * 4);        // inverse contributor count
  return L;
}

enum FwdRegion { kPq = 0, kPk, kPv, kScore, kTopk };
Layout fwd_ws_layout(const Geom& g) {
  Layout L;
  const size_t pyr = (size_t)g.U * (g.M - g.N) * g.d * 4;
  L.add(pyr);
  L.add(pyr);
  L.add(pyr);
  L.add((size_t)g.U * g.M * 4);
  L.add(topk_passes_workspace_bytes(g));  // the selection's device-wide passes
  return L;
}

enum BwdRegion { kDos = 0, kStats, kDqs, kDks, kDvs };
Layout bwd_ws_layout(const Geom& g) {
  Layout L;
  const size_t US = (size_t)g.U * g.S;
  L.add(US * g.d * 2);                // dos
  L.add(attn_stats_floats(g) * 4);   // softmax statistics, tile-padded
  for (int i = 0; i < 3; ++i) L.add(US * g.d * 4);
  return L;
}

lh_status check_shape(const lh_shape* s) {
  if (!s) return LH_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->N < 1) return LH_ERR_SHAPE;
  if (s->d != 64 && s->d != 128) return LH_ERR_SHAPE;
  if (s->p < 2 || s->L < 1 || s->L > kMaxLevels) return LH_ERR_SHAPE;
  if (s->B > ((int64_t)1 << 24) || s->H > ((int64_t)1 << 24)) return LH_ERR_SHAPE;
  int64_t pw = 1, M = 0;
  for (int l = 0; l < s->L; ++l) {
    if (l > 0) {
      if (pw > s->N / s->p) return LH_ERR_SHAPE;  // p^l > N
      pw *= s->p;
    }
    if (s->N % pw != 0) return LH_ERR_SHAPE;
    M += s->N / pw;
  }
  if (M >= ((int64_t)1 << 31)) return LH_ERR_SHAPE;
  if (s->S < 1 || (int64_t)s->S > M) return LH_ERR_SHAPE;
  const int64_t U = s->B * s->H;
  if (U > ((int64_t)1 << 40) / M) return LH_ERR_SHAPE;
  return LH_OK;
}

inline bool aligned16(const void* p) { return p && (((uintptr_t)p) & 15u) == 0; }

bool use_tc() {
  int v = g_attn_impl.load();
  if (v == 1) return false;
  return attn_tc_available();
}

}  // namespace

bool attn_fwd_uses_tc() { return use_tc(); }
bool attn_bwd_uses_tc() { return use_tc() && attn_tc_bwd_available(); }

namespace {

inline lh_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LH_OK : LH_ERR_CUDA; }

#define LH_TRY(expr)                           \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return LH_ERR_CUDA; \
  } while (0)

float resolve_scale(const Geom& g, float scale) {
  return scale > 0.0f ? scale : 1.0f / sqrtf((float)g.d);
}

lh_status attn_fwd(const Geom& g, const __half* qs, const __half* ks,
                   const __half* vs, float scale, __half* os, float* lse,
                   cudaStream_t st) {
  if (attn_fwd_uses_tc()) return cuda_status(launch_attn_fwd_tc(g, qs, ks, vs, scale, os, lse, st));
  return cuda_status(launch_attn_fwd_mma(g, qs, ks, vs, scale, os, lse, st));
}

// How lh_forward gathers the sub-sequence.  The pyramid path writes every fp32
// level (12 (M - N) d bytes per unit) and reads S rows back; the pooled path
// writes no level and reads, for each selected entry of level l, its p^l input
// rows.  The selection is unknown when the path is chosen (no host sync), so the
// rule takes the worst case, all S entries at the coarsest level: the pooled
// path when S p^(L-1) rows of Q, K, V, with a margin of 4 for the pooled
// kernel's per-span reads, cost less than the level writes.  For the
// benchmark workloads the selections cover 1.27-1.38 N rows of spans and the
// pyramid path is the faster one (measured: 0.29 vs 1.21 ms at the pretraining
// shape), which the rule picks; small budgets over long inputs take the pooled path.
bool use_pooled_gather(const Geom& g, lh_dtype dt) {
  if (g.L == 1) return false;
  const double s = dt == LH_BF16 ? 2.0 : 4.0;
  const double worst = 4.0 * (double)g.S * (double)g.pw[g.L - 1] * 3.0 * g.d * s;
  const double levels = 12.0 * (double)(g.M - g.N) * g.d;
  return worst < levels;
}

// How lh_forward selects: device-wide passes (launch_topk_passes, its later
// passes dependent launches).  Measured against one cluster per unit (launch_topk):
// 98,304 tokens 69 -> 62 us, 524,288 tokens 410 -> 160 us, where the cluster
// kernel needs 16-CTA clusters, of which a B200 runs only 7 at once.
bool use_topk_passes(const Geom& g) {
  (void)g;
  return true;
}

// The geometry of a shape with the variant options applied (options validated).
Geom geom_with(const lh_shape& shape, const lh_options* opt) {
  Geom g = make_geom(shape);
  if (opt) {
    g.score_mode = opt->score_mode;
    g.keep_top = opt->keep_coarsest;
    g.scatter_mode = opt->scatter_mode;
  }
  return g;
}

}  // namespace

lh_status attn_bwd(const Geom& g, const __half* qs, const __half* ks,
                   const __half* vs, const __half* os, const float* lse,
                   const __half* dos, float scale, float* dqs, float* dks, float* dvs,
                   float* stats, cudaStream_t st, int full) {
  if (full && !attn_bwd_uses_tc()) return LH_ERR_UNSUPPORTED;  // checked before any launch
  LH_TRY(launch_attn_stats(g, os, dos, lse, stats, st));
  if (attn_bwd_uses_tc())
    return cuda_status(launch_attn_bwd_tc(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, st, full));
  return cuda_status(launch_attn_bwd_mma(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, st));
}

}  // namespace lh

using namespace lh;

extern "C" {

const char* lh_status_string(lh_status s) {
  switch (s) {
    case LH_OK: return "LH_OK";
    case LH_ERR_INVALID_ARG: return "LH_ERR_INVALID_ARG: null or misaligned pointer, or bad enum";
    case LH_ERR_SHAPE: return "LH_ERR_SHAPE: shape outside the supported limits";
    case LH_ERR_UNSUPPORTED: return "LH_ERR_UNSUPPORTED: no kernel for this device/configuration";
    case LH_ERR_WORKSPACE: return "LH_ERR_WORKSPACE: workspace smaller than required";
    case LH_ERR_CUDA: return "LH_ERR_CUDA: a CUDA call or kernel launch failed";
    case LH_ERR_DEVICE_STATUS:
      return "LH_ERR_DEVICE_STATUS: a kernel reported a timed-out wait or an fp16 saturation";
  }
  return "LH_ERR_UNKNOWN";
}

lh_status lh_validate(const lh_shape* shape, lh_dtype dtype) {
  if (dtype != LH_F32 && dtype != LH_BF16) return LH_ERR_INVALID_ARG;
  return check_shape(shape);
}

int64_t lh_num_entries(const lh_shape* shape) {
  if (check_shape(shape) != LH_OK) return -1;
  return make_geom(*shape).M;
}

size_t lh_saved_bytes(const lh_shape* shape) {
  if (check_shape(shape) != LH_OK) return 0;
  return saved_layout(make_geom(*shape)).total;
}

int64_t lh_saved_offset(const lh_shape* shape, int which) {
  if (check_shape(shape) != LH_OK || which < 0 || which >= kNumSaved) return -1;
  return (int64_t)saved_layout(make_geom(*shape)).off[which];
}

size_t lh_workspace_bytes(const lh_shape* shape, lh_dtype dtype, int with_backward) {
  if (lh_validate(shape, dtype) != LH_OK) return 0;
  const Geom g = make_geom(*shape);
  size_t f = fwd_ws_layout(g).total;
  if (!with_backward) return f;
  size_t b = bwd_ws_layout(g).total;
  return f > b ? f : b;
}

size_t lh_topk_workspace_bytes(const lh_shape* shape) {
  if (check_shape(shape) != LH_OK) return 0;
  return topk_passes_workspace_bytes(make_geom(*shape));
}

size_t lh_attn_bwd_workspace_bytes(const lh_shape* shape) {
  if (check_shape(shape) != LH_OK) return 0;
  const Geom g = make_geom(*shape);
  return align_up(attn_stats_floats(g) * 4);
}

lh_status lh_validate_options(const lh_shape* shape, const lh_options* opt) {
  lh_status s = check_shape(shape);
  if (s != LH_OK) return s;
  if (opt == nullptr) return LH_OK;
  if (opt->reserved != 0) return LH_ERR_INVALID_ARG;
  if (opt->score_mode < LH_SCORE_SUM || opt->score_mode > LH_SCORE_CONCAT) return LH_ERR_INVALID_ARG;
  if (opt->scatter_mode < LH_SCATTER_MEAN || opt->scatter_mode > LH_SCATTER_LAST)
    return LH_ERR_INVALID_ARG;
  if (opt->keep_coarsest != 0 && opt->keep_coarsest != 1) return LH_ERR_INVALID_ARG;
  if (opt->keep_coarsest) {
    const Geom g = make_geom(*shape);
    if (g.N / g.pw[g.L - 1] > g.S) return LH_ERR_SHAPE;  // the coarsest level alone exceeds S
  }
  return LH_OK;
}

lh_status lh_build_pyramid(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                           const void* v, float* pq, float* pk, float* pv, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return LH_ERR_INVALID_ARG;
  if (shape->L == 1) return LH_OK;  // no level above the input
  if (!aligned16(pq) || !aligned16(pk) || !aligned16(pv)) return LH_ERR_INVALID_ARG;
  const Geom g = make_geom(*shape);
  return cuda_status(launch_pyramid_score(g, dtype, q, k, v, pq, pk, pv, nullptr, stream));
}

lh_status lh_build_pyramid_score_ex(const lh_shape* shape, lh_dtype dtype, const void* q,
                                    const void* k, const void* v, float* pq, float* pk, float* pv,
                                    float* score, const lh_options* opt, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(score))
    return LH_ERR_INVALID_ARG;
  if (shape->L > 1 && (!aligned16(pq) || !aligned16(pk) || !aligned16(pv)))
    return LH_ERR_INVALID_ARG;
  const Geom g = geom_with(*shape, opt);
  if (g.L == 1) pq = pk = pv = nullptr;
  return cuda_status(launch_pyramid_score(g, dtype, q, k, v, pq, pk, pv, score, stream));
}

lh_status lh_build_pyramid_score(const lh_shape* shape, lh_dtype dtype, const void* q,
                                 const void* k, const void* v, float* pq, float* pk, float* pv,
                                 float* score, lh_stream_t stream) {
  return lh_build_pyramid_score_ex(shape, dtype, q, k, v, pq, pk, pv, score, nullptr, stream);
}

lh_status lh_score_ex(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                      float* score, const lh_options* opt, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(score)) return LH_ERR_INVALID_ARG;
  const Geom g = geom_with(*shape, opt);
  return cuda_status(
      launch_pyramid_score(g, dtype, q, k, nullptr, nullptr, nullptr, nullptr, score, stream));
}

lh_status lh_score(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                   float* score, lh_stream_t stream) {
  return lh_score_ex(shape, dtype, q, k, score, nullptr, stream);
}

lh_status lh_topk_select_ex(const lh_shape* shape, const float* score, int32_t* idx,
                            int32_t* pos, int32_t* slot, void* ws, size_t ws_bytes,
                            const lh_options* opt, lh_stream_t stream) {
  lh_status s = check_shape(shape);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(score) || !aligned16(idx) || !aligned16(pos) || !aligned16(slot) ||
      (ws != nullptr && !aligned16(ws)))
    return LH_ERR_INVALID_ARG;
  const Geom g = geom_with(*shape, opt);
  if (ws == nullptr)  // no workspace: one thread-block cluster per unit
    return cuda_status(launch_topk(g, score, idx, pos, slot, stream));
  if (ws_bytes < topk_passes_workspace_bytes(g)) return LH_ERR_WORKSPACE;
  return cuda_status(launch_topk_passes(g, score, idx, pos, slot, ws, stream));
}

lh_status lh_topk_select(const lh_shape* shape, const float* score, int32_t* idx, int32_t* pos,
                         int32_t* slot, void* ws, size_t ws_bytes, lh_stream_t stream) {
  return lh_topk_select_ex(shape, score, idx, pos, slot, ws, ws_bytes, nullptr, stream);
}

lh_status lh_gather(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                    const void* v, const float* pq, const float* pk, const float* pv,
                    const int32_t* idx, void* qs, void* ks, void* vs, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(qs) ||
      !aligned16(ks) || !aligned16(vs))
    return LH_ERR_INVALID_ARG;
  if (shape->L > 1 && (!aligned16(pq) || !aligned16(pk) || !aligned16(pv)))
    return LH_ERR_INVALID_ARG;
  return cuda_status(launch_gather(make_geom(*shape), dtype, q, k, v, pq, pk, pv, idx,
                                   static_cast<__half*>(qs),
                                   static_cast<__half*>(ks),
                                   static_cast<__half*>(vs), stream));
}

lh_status lh_gather_pooled(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                           const void* v, const int32_t* idx, void* qs, void* ks, void* vs,
                           lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(qs) ||
      !aligned16(ks) || !aligned16(vs))
    return LH_ERR_INVALID_ARG;
  return cuda_status(launch_gather_pooled(make_geom(*shape), dtype, q, k, v, idx,
                                          static_cast<__half*>(qs), static_cast<__half*>(ks),
                                          static_cast<__half*>(vs), stream));
}

lh_status lh_subseq_attn_fwd(const lh_shape* shape, const void* qs, const void* ks,
                             const void* vs, float scale, void* os, float* lse,
                             lh_stream_t stream) {
  lh_status s = check_shape(shape);
  if (s != LH_OK) return s;
  if (!aligned16(qs) || !aligned16(ks) || !aligned16(vs) || !aligned16(os) || !aligned16(lse))
    return LH_ERR_INVALID_ARG;
  const Geom g = make_geom(*shape);
  return attn_fwd(g, static_cast<const __half*>(qs), static_cast<const __half*>(ks),
                  static_cast<const __half*>(vs), resolve_scale(g, scale),
                  static_cast<__half*>(os), lse, stream);
}

lh_status lh_subseq_attn_bwd(const lh_shape* shape, const void* qs, const void* ks,
                             const void* vs, const void* os, const float* lse, const void* dos,
                             float scale, float* dqs, float* dks, float* dvs, void* ws,
                             size_t ws_bytes, lh_stream_t stream) {
  lh_status s = check_shape(shape);
  if (s != LH_OK) return s;
  if (!aligned16(qs) || !aligned16(ks) || !aligned16(vs) || !aligned16(os) || !aligned16(lse) ||
      !aligned16(dos) || !aligned16(dqs) || !aligned16(dks) || !aligned16(dvs))
    return LH_ERR_INVALID_ARG;
  if (ws_bytes < lh_attn_bwd_workspace_bytes(shape)) return LH_ERR_WORKSPACE;
  if (!aligned16(ws)) return LH_ERR_INVALID_ARG;
  const Geom g = make_geom(*shape);
  return attn_bwd(g, static_cast<const __half*>(qs), static_cast<const __half*>(ks),
                  static_cast<const __half*>(vs), static_cast<const __half*>(os),
                  lse, static_cast<const __half*>(dos), resolve_scale(g, scale), dqs, dks,
                  dvs, static_cast<float*>(ws), stream);
}

lh_status lh_scatter_back_ex(const lh_shape* shape, lh_dtype dtype, const void* os,
                             const int32_t* slot, void* o, float* inv_count, const lh_options* opt,
                             lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(os) || !aligned16(slot) || !aligned16(o)) return LH_ERR_INVALID_ARG;
  if (inv_count && !aligned16(inv_count)) return LH_ERR_INVALID_ARG;
  return cuda_status(launch_scatter(geom_with(*shape, opt), dtype,
                                    static_cast<const __half*>(os), slot, o, inv_count,
                                    stream));
}

lh_status lh_scatter_back(const lh_shape* shape, lh_dtype dtype, const void* os,
                          const int32_t* slot, void* o, float* inv_count, lh_stream_t stream) {
  return lh_scatter_back_ex(shape, dtype, os, slot, o, inv_count, nullptr, stream);
}

lh_status lh_scatter_back_bwd_ex(const lh_shape* shape, lh_dtype dtype, const void* dO,
                                 const int32_t* slot, const float* inv_count, void* dos,
                                 const lh_options* opt, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(dO) || !aligned16(slot) || !aligned16(dos)) return LH_ERR_INVALID_ARG;
  if (inv_count && !aligned16(inv_count)) return LH_ERR_INVALID_ARG;
  return cuda_status(launch_scatter_bwd(geom_with(*shape, opt), dtype, dO, slot, inv_count,
                                        static_cast<__half*>(dos), stream));
}

lh_status lh_scatter_back_bwd(const lh_shape* shape, lh_dtype dtype, const void* dO,
                              const int32_t* slot, const float* inv_count, void* dos,
                              lh_stream_t stream) {
  return lh_scatter_back_bwd_ex(shape, dtype, dO, slot, inv_count, dos, nullptr, stream);
}

lh_status lh_gather_bwd(const lh_shape* shape, lh_dtype dtype, const float* dqs,
                        const float* dks, const float* dvs, const int32_t* slot, void* dq,
                        void* dk, void* dv, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if (!aligned16(dqs) || !aligned16(dks) || !aligned16(dvs) || !aligned16(slot) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return LH_ERR_INVALID_ARG;
  return cuda_status(
      launch_gather_bwd(make_geom(*shape), dtype, dqs, dks, dvs, slot, dq, dk, dv, stream));
}

lh_status lh_forward(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                     const void* v, float scale, void* o, void* saved, void* ws,
                     size_t ws_bytes, lh_stream_t stream) {
  return lh_forward_ex(shape, dtype, q, k, v, scale, o, saved, ws, ws_bytes, nullptr, stream);
}

lh_status lh_forward_ex(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                        const void* v, float scale, void* o, void* saved, void* ws,
                        size_t ws_bytes, const lh_options* opt, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(saved) ||
      !aligned16(ws))
    return LH_ERR_INVALID_ARG;
  if (ws_bytes < lh_workspace_bytes(shape, dtype, 0)) return LH_ERR_WORKSPACE;
  const Geom g = geom_with(*shape, opt);
  const Layout sl = saved_layout(g), wl = fwd_ws_layout(g);
  char* sv = static_cast<char*>(saved);
  char* w = static_cast<char*>(ws);
  int32_t* idx = reinterpret_cast<int32_t*>(sv + sl.off[kIdx]);
  int32_t* pos = reinterpret_cast<int32_t*>(sv + sl.off[kPos]);
  int32_t* slot = reinterpret_cast<int32_t*>(sv + sl.off[kSlot]);
  auto* qs = reinterpret_cast<__half*>(sv + sl.off[kQs]);
  auto* ks = reinterpret_cast<__half*>(sv + sl.off[kKs]);
  auto* vs = reinterpret_cast<__half*>(sv + sl.off[kVs]);
  auto* os = reinterpret_cast<__half*>(sv + sl.off[kOs]);
  float* lse = reinterpret_cast<float*>(sv + sl.off[kLse]);
  float* ic = reinterpret_cast<float*>(sv + sl.off[kInvCnt]);
  float* pq = g.L > 1 ? reinterpret_cast<float*>(w + wl.off[kPq]) : nullptr;
  float* pk = g.L > 1 ? reinterpret_cast<float*>(w + wl.off[kPk]) : nullptr;
  float* pv = g.L > 1 ? reinterpret_cast<float*>(w + wl.off[kPv]) : nullptr;
  float* score = reinterpret_cast<float*>(w + wl.off[kScore]);
  void* tws = w + wl.off[kTopk];

  if (use_pooled_gather(g, dtype)) {
    // scores only (no pyramid level written), then each selected coarse entry
    // pooled from its span of input rows: the same bits as the pyramid gather
    LH_TRY(launch_pyramid_score(g, dtype, q, k, nullptr, nullptr, nullptr, nullptr, score, stream));
    LH_TRY(use_topk_passes(g) ? launch_topk_passes(g, score, idx, pos, slot, tws, stream)
                              : launch_topk(g, score, idx, pos, slot, stream));
    LH_TRY(launch_gather_pooled(g, dtype, q, k, v, idx, qs, ks, vs, stream));
  } else {
    LH_TRY(launch_pyramid_score(g, dtype, q, k, v, pq, pk, pv, score, stream));
    LH_TRY(use_topk_passes(g) ? launch_topk_passes(g, score, idx, pos, slot, tws, stream)
                              : launch_topk(g, score, idx, pos, slot, stream));
    LH_TRY(launch_gather(g, dtype, q, k, v, pq, pk, pv, idx, qs, ks, vs, stream));
  }
  s = attn_fwd(g, qs, ks, vs, resolve_scale(g, scale), os, lse, stream);
  if (s != LH_OK) return s;
  LH_TRY(launch_scatter(g, dtype, os, slot, o, ic, stream));
  return LH_OK;
}

lh_status lh_backward(const lh_shape* shape, lh_dtype dtype, const void* saved, const void* dO,
                      float scale, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                      lh_stream_t stream) {
  return lh_backward_ex(shape, dtype, saved, dO, scale, dq, dk, dv, ws, ws_bytes, nullptr, stream);
}

lh_status lh_backward_ex(const lh_shape* shape, lh_dtype dtype, const void* saved, const void* dO,
                         float scale, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                         const lh_options* opt, lh_stream_t stream) {
  lh_status s = lh_validate(shape, dtype);
  if (s != LH_OK) return s;
  if ((s = lh_validate_options(shape, opt)) != LH_OK) return s;
  if (!aligned16(saved) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned16(ws))
    return LH_ERR_INVALID_ARG;
  if (ws_bytes < bwd_ws_layout(make_geom(*shape)).total) return LH_ERR_WORKSPACE;
  const Geom g = geom_with(*shape, opt);
  const Layout sl = saved_layout(g), wl = bwd_ws_layout(g);
  const char* sv = static_cast<const char*>(saved);
  char* w = static_cast<char*>(ws);
  const int32_t* slot = reinterpret_cast<const int32_t*>(sv + sl.off[kSlot]);
  auto* qs = reinterpret_cast<const __half*>(sv + sl.off[kQs]);
  auto* ks = reinterpret_cast<const __half*>(sv + sl.off[kKs]);
  auto* vs = reinterpret_cast<const __half*>(sv + sl.off[kVs]);
  auto* os = reinterpret_cast<const __half*>(sv + sl.off[kOs]);
  const float* lse = reinterpret_cast<const float*>(sv + sl.off[kLse]);
  const float* ic = reinterpret_cast<const float*>(sv + sl.off[kInvCnt]);
  auto* dos = reinterpret_cast<__half*>(w + wl.off[kDos]);
  float* stats = reinterpret_cast<float*>(w + wl.off[kStats]);
  float* dqs = reinterpret_cast<float*>(w + wl.off[kDqs]);
  float* dks = reinterpret_cast<float*>(w + wl.off[kDks]);
  float* dvs = reinterpret_cast<float*>(w + wl.off[kDvs]);

  LH_TRY(launch_scatter_bwd(g, dtype, dO, slot, ic, dos, stream));
  s = attn_bwd(g, qs, ks, vs, os, lse, dos, resolve_scale(g, scale), dqs, dks, dvs, stats, stream);
  if (s != LH_OK) return s;
  LH_TRY(launch_gather_bwd(g, dtype, dqs, dks, dvs, slot, dq, dk, dv, stream));
  return LH_OK;
}

lh_status lh_read_device_status(lh_stream_t stream, uint32_t* code) {
  uint32_t v = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LH_ERR_CUDA;
  cudaError_t (*const words[])(uint32_t*) = {device_status_read_clear, subseq_status_read_clear,
                                             pyramid_status_read_clear, topk_status_read_clear,
                                             mma_status_read_clear};
  for (auto read_clear : words) {
    uint32_t w = 0;
    if (read_clear(&w) != cudaSuccess) return LH_ERR_CUDA;
    v |= w;
  }
  if (code) *code = v;
  return v ? LH_ERR_DEVICE_STATUS : LH_OK;
}

int lh_forward_topk_path(const lh_shape* shape) {
  if (check_shape(shape) != LH_OK) return -1;
  return use_topk_passes(make_geom(*shape)) ? 1 : 0;
}

int lh_forward_gather_path(const lh_shape* shape, lh_dtype dtype) {
  if (lh_validate(shape, dtype) != LH_OK) return -1;
  return use_pooled_gather(make_geom(*shape), dtype) ? 1 : 0;
}

int lh_set_attention_impl(int impl) {
  if (impl != 0 && impl != 1) impl = -1;
  return g_attn_impl.exchange(impl);
}

int lh_attention_impl_in_use(void) {
  const bool f = attn_fwd_uses_tc(), b = attn_bwd_uses_tc();
  return f && b ? 0 : (!f && !b ? 1 : 2);
}

int lh_kernel_launches(const lh_shape* shape, lh_dtype dtype, int backward) {
  if (check_shape(shape) != LH_OK) return -1;
  if (dtype != LH_BF16 && dtype != LH_F32) return -1;
  const Geom g = make_geom(*shape);
  const int chunks = (int)((g.U + 65534) / 65535);  // grid.y limit per launch
  if (!backward) {
    // pyramid+score, top-k (per chunk), gather, attention (per chunk), scatter (per chunk)
    return pyramid_launches(g, dtype) + (use_topk_passes(g) ? topk_passes_launches(g) : chunks) + 1 +
           (attn_fwd_uses_tc() ? attn_tc_fwd_launches(g) : chunks) + chunks;
  }
  // scatter-back bwd, softmax statistics, attention bwd, gather bwd (per chunk)
  return 1 + 1 + (attn_bwd_uses_tc() ? attn_tc_bwd_launches(g) : 2 * chunks) + chunks;
}

}  // extern "C"
