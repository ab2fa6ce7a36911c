// k_gather_scatter.cu -- gather into the dense sub-sequence, scatter-back, and
// the adjoints of both.
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.C: the selected triplets form one dense
// sequence (gather) and a deterministic kernel returns the attention outputs to
// their original positions (scatter-back); §2.B: gradients flow back through
// scatter-back, the attention and the gather only.  "Contributors" per original
// position: phase 1 of bitsgeniais.com.br "Adeus Custo Quadrático! ...".
//
// Every kernel gives a group of G = d/8 consecutive lanes one row (or one
// coarsest span) and lane c columns [8c, 8c+8): all HBM traffic is 128-bit and
// coalesced, and every output element is written by exactly one thread in a
// fixed order of additions (no atomics), so results are bitwise reproducible.
#include <type_traits>

#include "lh_internal.cuh"

namespace lh {

// Status word of the kernels in this file: kStatusFp16Saturated when a finite
// value written into the fp16 sub-sequence (qs, ks, vs by the gather, dos by
// the scatter-back adjoint) was beyond +-65504 and clipped; in the debug build
// also the bounds checks (kStatusBounds).
__device__ uint32_t g_subseq_status = 0;
#define LH_STATUS_WORD g_subseq_status

cudaError_t subseq_status_read_clear(uint32_t* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_subseq_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_subseq_status, &zero, sizeof(zero));
}

namespace {

__device__ __forceinline__ void report_saturation(uint32_t sat) {
  if (sat) atomicOr(&g_subseq_status, kStatusFp16Saturated);
}

// Per-unit geometry with 32-bit indices (M < 2^31 is a checked limit); unit
// offsets stay 64-bit.  log2p >= 0 when p is a power of two: then the level-l
// index of token t is a shift instead of a division.
struct Lv {
  int32_t N, M, S;
  int32_t L, p, log2p;
  int32_t mode;  // lh_scatter_mode of the scatter-back (mean, sum, last token)
  int32_t off[kMaxLevels + 1];
  int32_t pw[kMaxLevels + 1];
};

Lv make_lv(const Geom& g) {
  Lv v;
  v.N = (int32_t)g.N;
  v.M = (int32_t)g.M;
  v.S = g.S;
  v.L = g.L;
  v.p = g.p;
  v.log2p = ((g.p & (g.p - 1)) == 0) ? __builtin_ctz((unsigned)g.p) : -1;
  v.mode = g.scatter_mode;
  for (int l = 0; l <= kMaxLevels; ++l) {
    v.off[l] = (int32_t)g.off[l];
    v.pw[l] = (int32_t)(g.pw[l] > 0x7fffffff ? 0x7fffffff : g.pw[l]);
  }
  return v;
}

// Slot-map entry X of a unit, sl = the unit's map.  The debug build checks that
// X lies in [0, M) and the value in [-1, S) and reads a bad one as -1 (skipped).
__device__ __forceinline__ int32_t ld_slot(const int32_t* __restrict__ sl, int32_t X, const Lv& lv,
                                           uint32_t bits) {
  if (!LH_CHECK(dbg::in_range(X, lv.M), bits)) return -1;
  const int32_t s = __ldg(sl + X);
  return LH_CHECK(dbg::slot_ok(s, lv.S), bits) ? s : -1;
}

// index at level l of the entry covering token t: floor(t / p^l)
__device__ __forceinline__ int32_t lvl_index(const Lv& lv, int32_t t, int l) {
  return lv.log2p >= 0 ? (t >> (l * lv.log2p)) : (int32_t)((uint32_t)t / (uint32_t)lv.pw[l]);
}

inline unsigned blocks_for(int64_t threads, int block) {
  return (unsigned)((threads + block - 1) / block);
}

// ------------------------------------------------------------------ gather
// xs[u,k] = fp16_rne(level row of gid idx[u,k]), saturating; level 0 from the input.
template <typename Tin, int D>
__global__ void __launch_bounds__(256) k_gather(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const float* __restrict__ pq, const float* __restrict__ pk, const float* __restrict__ pv,
    const int32_t* __restrict__ idx, __half* __restrict__ qs, __half* __restrict__ ks,
    __half* __restrict__ vs, const Lv lv, int64_t rows) {
  pdl_enter();
  constexpr int G = D / 8;
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gt / G;  // u * S + slot
  if (row >= rows) return;
  const int c = (int)(gt % G);
  const int64_t u = row / lv.S;
  const int32_t gid = __ldg(idx + row);
  if (!LH_CHECK(dbg::in_range(gid, lv.M), kBoundsGather)) return;
  float xq[8], xk[8], xv[8];
  if (gid < lv.N) {
    const int64_t o = (u * lv.N + gid) * D + 8 * c;
    load8(q + o, xq);
    load8(k + o, xk);
    load8(v + o, xv);
  } else {
    const int64_t o = (u * (int64_t)(lv.M - lv.N) + (gid - lv.N)) * D + 8 * c;
    load8(pq + o, xq);
    load8(pk + o, xk);
    load8(pv + o, xv);
  }
  const int64_t d = row * D + 8 * c;
  uint32_t sat = 0;
  store8_h(qs + d, xq, sat);
  store8_h(ks + d, xk, sat);
  store8_h(vs + d, xv, sat);
  report_saturation(sat);
}

// ------------------------------------------------------------ pooled gather
// Same result as k_gather on a pyramid, without the pyramid: a selected entry of
// level l >= 1 is pooled from its span of level-0 rows with exactly the pyramid
// kernel's arithmetic (children summed in order from 0.0f with fp32 adds, the
// sum divided by p, level by level), so every value has the same bits.  Only
// the rows of selected spans are read; no pooled level is written to HBM.
constexpr int kPoolBatch = 4;  // level-0 rows whose loads are in flight together

template <typename Tin, int D, int L>
__device__ __forceinline__ void pool_span(const Tin* __restrict__ src, int lev, const Lv& lv,
                                          float (&out)[8]) {
  // src: first row of the span (this lane's 8 columns); p^lev rows at stride D;
  // acc[l] is the running sum of the children of the current level-(l+1) entry
  constexpr int NL = (L > 1) ? (L - 1) : 1;
  float acc[NL][8];
  int cnt[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) {
    cnt[l] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[l][i] = 0.0f;
  }
  const int rows = lv.pw[lev];
  const float fp = (float)lv.p;
  for (int r0 = 0; r0 < rows; r0 += kPoolBatch) {
    float x[kPoolBatch][8];
#pragma unroll
    for (int b = 0; b < kPoolBatch; ++b)
      if (r0 + b < rows) load8(src + (int64_t)(r0 + b) * D, x[b]);
#pragma unroll
    for (int b = 0; b < kPoolBatch; ++b) {
      if (r0 + b >= rows) break;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[0][i] = __fadd_rn(acc[0][i], x[b][i]);
      cnt[0] += 1;
#pragma unroll
      for (int l = 0; l < NL; ++l) {
        if (l + 1 > lev || cnt[l] != lv.p) break;
        // level l+1 complete: its mean feeds level l+2 (or is the answer)
        float m[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = __fdiv_rn(acc[l][i], fp);
        if (l + 1 == lev) {
#pragma unroll
          for (int i = 0; i < 8; ++i) out[i] = m[i];
        } else if (l + 1 < NL) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[l + 1][i] = __fadd_rn(acc[l + 1][i], m[i]);
          cnt[l + 1] += 1;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[l][i] = 0.0f;
        cnt[l] = 0;
      }
    }
  }
}

template <typename Tin, int D, int L>
__global__ void __launch_bounds__(256) k_gather_pooled(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const int32_t* __restrict__ idx, __half* __restrict__ qs, __half* __restrict__ ks,
    __half* __restrict__ vs, const Lv lv, int64_t rows) {
  pdl_enter();
  constexpr int G = D / 8;
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gt / G;  // u * S + slot
  if (row >= rows) return;
  const int c = (int)(gt % G);
  const int64_t u = row / lv.S;
  const int32_t gid = __ldg(idx + row);
  if (!LH_CHECK(dbg::in_range(gid, lv.M), kBoundsGather)) return;
  int lev = 0;
  while (lev + 1 < lv.L && gid >= lv.off[lev + 1]) ++lev;
  const int32_t j = gid - lv.off[lev];
  const int64_t first = (u * lv.N + (int64_t)j * lv.pw[lev]) * D + 8 * c;  // span start
  const int64_t d = row * D + 8 * c;
  const Tin* srcs[3] = {q + first, k + first, v + first};
  __half* dsts[3] = {qs + d, ks + d, vs + d};
  uint32_t sat = 0;
#pragma unroll
  for (int x = 0; x < 3; ++x) {
    float val[8];
    if (lev == 0)
      load8(srcs[x], val);
    else
      pool_span<Tin, D, L>(srcs[x], lev, lv, val);
    store8_h(dsts[x], val, sat);
  }
  report_saturation(sat);
}

// ------------------------------------------------------------- scatter-back
// O[t] = (sum over selected entries covering t, ascending level, of os[slot]) / c_t.
// Grid: x = blocks of kRows tokens of one unit, y = unit (offset u0).
// 1/c rounded to fp32 for the contributor counts c = 0..kMaxLevels (entry 0 unused)
__constant__ float kRcpCount[kMaxLevels + 1] = {0.0f,        1.0f,        1.0f / 2.0f,
                                                1.0f / 3.0f, 1.0f / 4.0f, 1.0f / 5.0f,
                                                1.0f / 6.0f, 1.0f / 7.0f, 1.0f / 8.0f};

// One thread: column chunk c of R consecutive tokens t0..t0+R-1 (R divides p,
// t0 a multiple of R), which share every entry of level >= 1; so each thread
// issues R + L - 1 slot loads and at most as many row loads, all independent.
__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = h_lo(w.x); x[1] = h_hi(w.x);
  x[2] = h_lo(w.y); x[3] = h_hi(w.y);
  x[4] = h_lo(w.z); x[5] = h_hi(w.z);
  x[6] = h_lo(w.w); x[7] = h_hi(w.w);
}

template <typename Tout, int D, int L, int R>
__global__ void __launch_bounds__(256) k_scatter(const __half* __restrict__ os,
                                                 const int32_t* __restrict__ slot,
                                                 Tout* __restrict__ o, float* __restrict__ inv_count,
                                                 const Lv lv, int64_t u0) {
  pdl_enter();
  constexpr int G = D / 8, kGroups = 256 / G;
  constexpr int LC = (L > 1) ? L - 1 : 1;  // coarse levels (array size)
  const int32_t t0 = ((int32_t)blockIdx.x * kGroups + (int32_t)(threadIdx.x / G)) * R;
  if (t0 >= lv.N) return;
  const int c = (int)(threadIdx.x % G);
  const int64_t u = u0 + blockIdx.y;
  const int32_t* sl = slot + u * lv.M;
  const __half* src = os + u * lv.S * D + 8 * c;
  int32_t s0[R], sc[LC];
#pragma unroll
  for (int r = 0; r < R; ++r) s0[r] = ld_slot(sl, t0 + r, lv, kBoundsScatter);
#pragma unroll
  for (int l = 1; l < L; ++l) sc[l - 1] = ld_slot(sl, lv.off[l] + lvl_index(lv, t0, l), lv, kBoundsScatter);
  uint4 w0[R], wc[LC];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    w0[r] = make_uint4(0u, 0u, 0u, 0u);
    if (s0[r] >= 0) w0[r] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)s0[r] * D));
  }
#pragma unroll
  for (int l = 1; l < L; ++l) {
    wc[l - 1] = make_uint4(0u, 0u, 0u, 0u);
    if (sc[l - 1] >= 0) wc[l - 1] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)sc[l - 1] * D));
  }
  // branch-free: an unselected level adds +0 (exact; at most the sign of a zero differs)
  float xc[LC][8];
  int cc = 0;
#pragma unroll
  for (int l = 1; l < L; ++l) {
    unpack8(wc[l - 1], xc[l - 1]);
    cc += sc[l - 1] >= 0 ? 1 : 0;
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float acc[8];
    unpack8(w0[r], acc);  // zeros when not selected
#pragma unroll
    for (int l = 1; l < L; ++l)  // ascending level, as defined
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], xc[l - 1][i]);
    const int cnt = cc + (s0[r] >= 0 ? 1 : 0);
    if (cnt > 0 && lv.mode != LH_SCATTER_SUM) {  // sums of fp16 values: 0 or |acc| >= 2^-24, inside div_small's range
      const float y = kRcpCount[cnt], cf = (float)cnt;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = div_small(acc[i], cf, y);
    }
    const int64_t row = u * lv.N + t0 + r;
    store8_stream(o + row * D + 8 * c, acc);
    // the weight of dO[t] in the adjoint: 1/c rounded (mean), 1 (sum); 0 when c = 0
    if (inv_count && c == 0) inv_count[row] = lv.mode == LH_SCATTER_SUM ? (cnt > 0 ? 1.0f : 0.0f) : kRcpCount[cnt];
  }
}

constexpr int ipow(int b, int e) { return e == 0 ? 1 : b * ipow(b, e - 1); }

// 8 output elements packed once and stored any number of times (streaming).
template <typename T>
struct Packed8;
template <>
struct Packed8<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void pack(const float (&x)[8]) {
    w = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                   pack_bf16(x[6], x[7]));
  }
  __device__ __forceinline__ void store(__nv_bfloat16* p) const { __stcs(reinterpret_cast<uint4*>(p), w); }
};
template <>
struct Packed8<float> {
  float4 a, b;
  __device__ __forceinline__ void pack(const float (&x)[8]) {
    a = make_float4(x[0], x[1], x[2], x[3]);
    b = make_float4(x[4], x[5], x[6], x[7]);
  }
  __device__ __forceinline__ void store(float* p) const {
    __stcs(reinterpret_cast<float4*>(p), a);
    __stcs(reinterpret_cast<float4*>(p) + 1, b);
  }
};

// Same result as k_scatter (the same additions in the same order), for p = P in
// {2, 4} known at compile time.  A thread owns NE consecutive level-1 entries
// (P tokens each) and walks them with the next entry's slot loads in flight while
// the current entry's rows load, so each entry costs one memory round trip.
// A token not selected at level 0 sums 0 + x_1 + x_2 + ... = x_1 + x_2 + ...,
// the same value for all P tokens of its level-1 entry, so that sum, its
// division and its packing are done once per entry and stored P times; only the
// (few) tokens selected at level 0 form their own chain.  Grid: x = blocks of
// level-1 entries of one unit, y = unit (offset u0).
constexpr int kScatterEntries = 4;  // level-1 entries per thread

template <typename Tout, int D, int L, int P>
__global__ void __launch_bounds__(128) k_scatter_pp(const __half* __restrict__ os,
                                                    const int32_t* __restrict__ slot,
                                                    Tout* __restrict__ o, float* __restrict__ inv_count,
                                                    const Lv lv, int64_t u0) {
  pdl_enter();
  static_assert(L >= 2 && (P == 2 || P == 4), "specialised on p in {2, 4}, L >= 2");
  constexpr int G = D / 8, kGroups = 128 / G, NE = kScatterEntries;
  constexpr int NU = (L > 2) ? L - 2 : 1;  // levels >= 2: one entry each
  const int32_t n1 = lv.N / P;            // level-1 entries (N is a multiple of P)
  const int32_t e0 = ((int32_t)blockIdx.x * kGroups + (int32_t)(threadIdx.x / G)) * NE;
  if (e0 >= n1) return;
  const int c = (int)(threadIdx.x % G);
  const int64_t u = u0 + blockIdx.y;
  const int32_t* sl = slot + u * lv.M;
  const __half* src = os + u * lv.S * D + 8 * c;

  struct Slots {
    int32_t s0[P], s1, su[NU];
  };
  auto load_slots = [&](int32_t e, Slots& sv) {  // entry e < n1
    const int32_t t = e * P;
#pragma unroll
    for (int r = 0; r < P; ++r) sv.s0[r] = ld_slot(sl, t + r, lv, kBoundsScatter);
    sv.s1 = ld_slot(sl, lv.off[1] + e, lv, kBoundsScatter);
    static_for<2, L>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      sv.su[l - 2] = ld_slot(sl, lv.off[l] + (int32_t)((uint32_t)e / (uint32_t)ipow(P, l - 1)), lv, kBoundsScatter);
    });
  };
  auto row = [&](int32_t sidx) {
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (sidx >= 0) w = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)sidx * D));
    return w;
  };
  Slots cur;
  load_slots(e0, cur);
#pragma unroll
  for (int k = 0; k < NE; ++k) {
    const int32_t e = e0 + k;
    if (e >= n1) break;  // warp-uniform except in the last block of a unit
    uint4 w0[P], w1, wu[NU];
#pragma unroll
    for (int r = 0; r < P; ++r) w0[r] = row(cur.s0[r]);
    w1 = row(cur.s1);
#pragma unroll
    for (int l = 2; l < L; ++l) wu[l - 2] = row(cur.su[l - 2]);
    Slots nxt;
    if (k + 1 < NE && e + 1 < n1) load_slots(e + 1, nxt);  // in flight with this entry's rows

    // the chain of a token unselected at level 0: x_1 + x_2 + ... (0 + x_1 = x_1
    // exactly, up to the sign of a zero), ascending level
    float x1[8], base[8];
    unpack8(w1, x1);
#pragma unroll
    for (int i = 0; i < 8; ++i) base[i] = x1[i];
    int cb = cur.s1 >= 0 ? 1 : 0;
#pragma unroll
    for (int l = 2; l < L; ++l) {
      float xu[8];
      unpack8(wu[l - 2], xu);
#pragma unroll
      for (int i = 0; i < 8; ++i) base[i] = __fadd_rn(base[i], xu[i]);
      cb += cur.su[l - 2] >= 0 ? 1 : 0;
    }
    const bool mean = lv.mode != LH_SCATTER_SUM;
    if (cb > 0 && mean) {  // sums of fp16 values: 0 or |sum| >= 2^-24, inside div_small's range
      const float y = kRcpCount[cb], cf = (float)cb;
#pragma unroll
      for (int i = 0; i < 8; ++i) base[i] = div_small(base[i], cf, y);
    }
    Packed8<Tout> ob;
    ob.pack(base);
    Tout* out = o + (u * lv.N + (int64_t)e * P) * D + 8 * c;
    float icv[P];
#pragma unroll
    for (int r = 0; r < P; ++r) {
      if (cur.s0[r] >= 0) {  // selected at level 0: its own chain x_0 + x_1 + x_2 + ...
        float acc[8];
        unpack8(w0[r], acc);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], x1[i]);
#pragma unroll
        for (int l = 2; l < L; ++l) {
          float xu[8];
          unpack8(wu[l - 2], xu);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], xu[i]);
        }
        const int cnt = cb + 1;
        const float y = kRcpCount[cnt], cf = (float)cnt;
        if (mean) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = div_small(acc[i], cf, y);
        }
        Packed8<Tout> pr;
        pr.pack(acc);
        pr.store(out + r * D);
        icv[r] = mean ? y : 1.0f;
      } else {
        ob.store(out + r * D);
        icv[r] = mean ? kRcpCount[cb] : (cb > 0 ? 1.0f : 0.0f);
      }
    }
    if (inv_count && c == 0) {  // the entry's P counts, one aligned vector store
      float* ip = inv_count + u * lv.N + (int64_t)e * P;
      if constexpr (P == 4)
        *reinterpret_cast<float4*>(ip) = make_float4(icv[0], icv[1], icv[2], icv[3]);
      else
        *reinterpret_cast<float2*>(ip) = make_float2(icv[0], icv[1]);
    }
    if (k + 1 < NE) cur = nxt;
  }
}

// ---------------------------------------------------------- scatter-back bwd
// dos[k] = sum_{t in span(k)} dO[t] / c_t, as a sum-pyramid of w[t] = dO[t]/c_t
// over each coarsest span: dO is read once, each selected row written once.
// RG row-groups of d/8 lanes share a span (RG = p, or 1): row-group r walks the
// r-th level-(L-2) entry of the span, and the span's top-level sum is formed
// from the RG partial sums in order with shuffles -- the same additions, in the
// same order, as one group walking the whole span (0 + s_0 = s_0 exactly).
template <typename Tin, int D, int L, int RG>
__global__ void __launch_bounds__(256) k_scatter_bwd(const Tin* __restrict__ dO,
                                                     const int32_t* __restrict__ slot,
                                                     const float* __restrict__ inv_count,
                                                     __half* __restrict__ dos, const Lv lv,
                                                     int64_t spans, int64_t groups) {
  pdl_enter();
  constexpr int G = D / 8;
  constexpr int NL = (L > 1) ? (L - 1) : 1;
  constexpr int RB = 4;  // rows of dO whose loads are in flight together
  static_assert(RG == 1 || (L > 1 && G * RG <= 32), "row-groups of a span share one warp");
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t group = gt / (G * RG);  // span
  if (group >= groups) return;          // whole spans leave together (G * RG divides 32)
  const int c = (int)(gt % G);
  const int rg = (int)((gt / G) % RG);
  const int32_t Ptop = lv.pw[L - 1] / RG;  // rows this row-group walks
  const int64_t u = group / spans;
  const int32_t t0 = (int32_t)(group - u * spans) * lv.pw[L - 1] + rg * Ptop;
  const int32_t* sl = slot + u * lv.M;
  const Tin* src = dO + (u * lv.N + t0) * D + 8 * c;
  __half* dst = dos + u * lv.S * D + 8 * c;
  uint32_t sat = 0;

  float acc[NL][8];
  int cnt[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) {
    cnt[l] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[l][i] = 0.0f;
  }
  for (int32_t r0 = 0; r0 < Ptop; r0 += RB) {
    float w[RB][8];
    float ic[RB];
    int32_t s0[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      if (r0 + b < Ptop) {
        const int32_t t = t0 + r0 + b;
        load8_stream(src + (int64_t)(r0 + b) * D, w[b]);
        s0[b] = ld_slot(sl, t, lv, kBoundsScatterBwd);
        if (inv_count) {
          ic[b] = __ldg(inv_count + u * lv.N + t);
        } else {
          int n = 0;
#pragma unroll
          for (int l = 0; l < L; ++l) n += (ld_slot(sl, lv.off[l] + lvl_index(lv, t, l), lv, kBoundsScatterBwd) >= 0) ? 1 : 0;
          ic[b] = lv.mode == LH_SCATTER_SUM ? (n > 0 ? 1.0f : 0.0f) : kRcpCount[n];
        }
      }
    }
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      if (r0 + b >= Ptop) break;
      const int32_t t = t0 + r0 + b;
#pragma unroll
      for (int i = 0; i < 8; ++i) w[b][i] = __fmul_rn(w[b][i], ic[b]);
      if (s0[b] >= 0) store8_h(dst + (int64_t)s0[b] * D, w[b], sat);
      if constexpr (L == 1) continue;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[0][i] = __fadd_rn(acc[0][i], w[b][i]);
      cnt[0] += 1;
#pragma unroll
      for (int l = 0; l < NL; ++l) {
        if (cnt[l] == lv.p) {
          const int lev = l + 1;
          const int32_t j = lvl_index(lv, t, lev);
          const int32_t s = ld_slot(sl, lv.off[lev] + j, lv, kBoundsScatterBwd);
          if (s >= 0) store8_h(dst + (int64_t)s * D, acc[l], sat);
          if (l + 1 < NL) {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[l + 1][i] = __fadd_rn(acc[l + 1][i], acc[l][i]);
            cnt[l + 1] += 1;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[l][i] = 0.0f;
          cnt[l] = 0;
        }
      }
    }
  }
  if constexpr (RG > 1) {
    // the span's level-(L-1) entry: its RG partial sums (each row-group's
    // acc[L-2] holds exactly one level-(L-2) sum) added in row-group order
    const int lane = threadIdx.x & 31;
    const int base = lane - rg * G;  // lane of row-group 0 with this chunk
    const unsigned mask = (G * RG == 32) ? 0xffffffffu
                                         : (((1u << (G * RG)) - 1u) << (lane & ~(G * RG - 1)));
    float tot[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) tot[i] = __shfl_sync(mask, acc[NL - 1][i], base);
#pragma unroll
    for (int r = 1; r < RG; ++r)
#pragma unroll
      for (int i = 0; i < 8; ++i) tot[i] = __fadd_rn(tot[i], __shfl_sync(mask, acc[NL - 1][i], base + r * G));
    if (rg == 0) {
      const int32_t j = (t0 + lv.pw[L - 1]) / lv.pw[L - 1] - 1;  // the span's entry at level L-1
      const int32_t s = ld_slot(sl, lv.off[L - 1] + j, lv, kBoundsScatterBwd);
      if (s >= 0) store8_h(dst + (int64_t)s * D, tot, sat);
    }
  }
  report_saturation(sat);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// 8 consecutive elements staged in shared memory (16 bytes of bf16, 32 of fp32) as fp32
__device__ __forceinline__ void staged8(const uint4* p, int stride, __nv_bfloat16*, float (&x)[8]) {
  const uint4 w = p[0];
  (void)stride;
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void staged8(const uint4* p, int stride, float*, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + stride);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

constexpr int kScatterBwdThreads = 128;

// Same sums as k_scatter_bwd (the same additions in the same order), for p = P
// in {2, 4} known at compile time and the saved 1/c_t.  A row-group walks its
// rows in batches of RB, two batches in flight: the rows of dO are copied by
// 16-byte cp.async into this thread's own slots of shared memory (consecutive
// threads take consecutive 16 bytes, so reads back are conflict-free), and each
// batch's slots, 1/c_t and the slots of the coarse entries that complete inside it
// are loaded into registers one batch ahead -- the stores of completed entries
// never wait on a slot load, and a thread keeps 2 * RB rows in flight without
// holding them in registers.
template <typename Tin, int D, int L, int P, int RG>
struct ScatterBwdCfg {
  static constexpr int G = D / 8;
  static constexpr int LW = (RG == 1) ? L - 1 : L - 2;  // coarse levels completed inside the walk
  static constexpr int Ptop = ipow(P, L - 1) / RG;        // rows one row-group walks
  static constexpr int CPR = sizeof(Tin) / 2;             // 16-byte copies per lane per row
  static constexpr int RBmax = 8 / CPR;
  static constexpr int RB = Ptop < RBmax ? Ptop : RBmax;  // rows per batch
  static constexpr int NB = Ptop / RB;                    // batches
  // level-l entries whose slot a batch loads: those inside it, or the one it ends in
  static constexpr int cnt(int l) { return ipow(P, l) <= RB ? RB / ipow(P, l) : 1; }
  static constexpr int first(int l) { return l <= 1 ? 0 : first(l - 1) + cnt(l - 1); }
  static constexpr int NCS = LW > 0 ? first(LW + 1) : 1;  // coarse slots per batch
  static constexpr size_t smem_bytes = (size_t)2 * RB * CPR * kScatterBwdThreads * 16;
};

// Grid: x = blocks of spans of one unit, y = unit (offset u0).
template <typename Tin, int D, int L, int P, int RG>
__global__ void __launch_bounds__(kScatterBwdThreads) k_scatter_bwd_pp(
    const Tin* __restrict__ dO, const int32_t* __restrict__ slot,
    const float* __restrict__ inv_count, __half* __restrict__ dos, const Lv lv, int32_t spans,
    int64_t u0) {
  pdl_enter();
  using C = ScatterBwdCfg<Tin, D, L, P, RG>;
  constexpr int G = C::G, LW = C::LW, Ptop = C::Ptop, CPR = C::CPR, RB = C::RB, NB = C::NB;
  constexpr int NCS = C::NCS, NA = LW > 0 ? LW : 1, NT = kScatterBwdThreads;
  static_assert(L >= 2 && (P == 2 || P == 4), "specialised on p in {2, 4}, L >= 2");
  static_assert(RG == 1 || (RG == P && G * RG <= 32), "row-groups of a span share one warp");
  static_assert(Ptop % RB == 0, "batches tile the walk");
  extern __shared__ uint4 sbuf[];  // [2 stages][RB][CPR][NT], this thread's column tid

  const int tid = (int)threadIdx.x;
  const int32_t gt = (int32_t)blockIdx.x * NT + tid;
  const int32_t span = gt / (G * RG);
  if (span >= spans) return;  // whole spans leave together (G * RG divides 32)
  const int c = gt % G;
  const int rg = (gt / G) % RG;
  const int64_t u = u0 + blockIdx.y;
  const int32_t t0 = span * ipow(P, L - 1) + rg * Ptop;
  const int32_t* sl = slot + u * lv.M;
  const float* icu = inv_count + u * lv.N;
  const Tin* src = dO + (u * lv.N + t0) * D + 8 * c;
  __half* dst = dos + u * lv.S * D + 8 * c;
  uint32_t sat = 0;

  auto issue = [&](int bi) {  // rows of batch bi into stage bi & 1
    uint4* st = sbuf + (bi & 1) * (RB * CPR * NT) + tid;
    const Tin* g = src + bi * (RB * D);
    static_for<0, RB>([&](auto bc) {
      constexpr int b = decltype(bc)::value;
      static_for<0, CPR>([&](auto qc) {
        constexpr int q = decltype(qc)::value;
        cp_async16(st + (b * CPR + q) * NT, g + b * D + 4 * q);
      });
    });
    cp_async_commit();
  };
  auto small_loads = [&](int bi, int32_t (&s0_)[RB], float (&ic_)[RB], int32_t (&cs_)[NCS]) {
    const int32_t tb = t0 + bi * RB;  // first token of the batch
    static_for<0, RB>([&](auto bc) {
      constexpr int b = decltype(bc)::value;
      s0_[b] = ld_slot(sl, tb + b, lv, kBoundsScatterBwd);
      ic_[b] = __ldg(icu + tb + b);
    });
    static_for<1, LW + 1>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      constexpr uint32_t pl = (uint32_t)ipow(P, l);
      constexpr int n = C::first(l), k = C::cnt(l);
      const int32_t j0 = (int32_t)((uint32_t)(tb + (pl <= (uint32_t)RB ? 0 : RB - 1)) / pl);
      static_for<0, k>([&](auto ic2) {
        constexpr int i = decltype(ic2)::value;
        cs_[n + i] = ld_slot(sl, lv.off[l] + j0 + i, lv, kBoundsScatterBwd);
      });
    });
  };
  int32_t s0[RB], cs[NCS];
  float ic[RB];
  issue(0);
  if (NB > 1) issue(1);
  small_loads(0, s0, ic, cs);

  float acc[NA][8];  // acc[l-1]: running sum of the current level-l entry
#pragma unroll
  for (int l = 0; l < NA; ++l)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[l][i] = 0.0f;
  float part[8];  // the walk's last completed entry (level LW; a row when LW = 0)

  for (int bi = 0; bi < NB; ++bi) {
    const int32_t r0 = bi * RB;
    int32_t s0n[RB], csn[NCS];
    float icn[RB];
    if (bi + 1 < NB) small_loads(bi + 1, s0n, icn, csn);
    if (bi + 1 < NB) cp_async_wait<1>(); else cp_async_wait<0>();
    const uint4* stg = sbuf + (bi & 1) * (RB * CPR * NT) + tid;
    static_for<0, RB>([&](auto bc) {
      constexpr int b = decltype(bc)::value;
      float w[8];
      staged8(stg + b * CPR * NT, NT, (Tin*)nullptr, w);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __fmul_rn(w[i], ic[b]);
      if (s0[b] >= 0) store8_h(dst + (int64_t)s0[b] * D, w, sat);
      if constexpr (LW == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) part[i] = w[i];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[0][i] = __fadd_rn(acc[0][i], w[i]);
        // entries completed by row r0 + b, finest first (each adds into the next level)
        static_for<1, LW + 1>([&](auto lc) {
          constexpr int l = decltype(lc)::value;
          constexpr int pl = ipow(P, l);
          constexpr bool inside = pl <= RB;  // the level's entries lie inside a batch
          constexpr int k = C::first(l) + (inside ? (b + 1) / pl - 1 : 0);
          bool done;
          if constexpr (inside)
            done = ((b + 1) % pl) == 0;
          else
            done = (b == RB - 1) && ((r0 + RB) % pl) == 0;
          if (done) {
            if (cs[k] >= 0) store8_h(dst + (int64_t)cs[k] * D, acc[l - 1], sat);
            if constexpr (l < LW) {
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[l][i] = __fadd_rn(acc[l][i], acc[l - 1][i]);
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) part[i] = acc[l - 1][i];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[l - 1][i] = 0.0f;
          }
        });
      }
    });
    if (bi + 2 < NB) issue(bi + 2);  // into the stage this thread just read
    if (bi + 1 < NB) {
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        s0[b] = s0n[b];
        ic[b] = icn[b];
      }
#pragma unroll
      for (int i = 0; i < NCS; ++i) cs[i] = csn[i];
    }
  }
  if constexpr (RG > 1) {
    // the span's level-(L-1) entry: the RG partial sums, added in row-group order
    const int lane = threadIdx.x & 31;
    const int base = lane - rg * G;  // lane of row-group 0 with this chunk
    const unsigned mask = (G * RG == 32) ? 0xffffffffu
                                         : (((1u << (G * RG)) - 1u) << (lane & ~(G * RG - 1)));
    float tot[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) tot[i] = __shfl_sync(mask, part[i], base);
#pragma unroll
    for (int r = 1; r < RG; ++r)
#pragma unroll
      for (int i = 0; i < 8; ++i) tot[i] = __fadd_rn(tot[i], __shfl_sync(mask, part[i], base + r * G));
    if (rg == 0) {
      const int32_t s = ld_slot(sl, lv.off[L - 1] + span, lv, kBoundsScatterBwd);
      if (s >= 0) store8_h(dst + (int64_t)s * D, tot, sat);
    }
  }
  report_saturation(sat);
}

// ------------------------------------------- scatter-back, last-token variant
// An entry delivers its output only to the last token of its span, pos(e); a
// token takes the mean of what reaches it (levels ascending): the level-0 entry
// at t and the entries of level l >= 1 whose span ends at t (p^l divides t + 1).
// One d/8-lane group per token; generic in p and L (an ablation, not the hot path).
__device__ __forceinline__ bool ends_at_t(const Lv& lv, int32_t t, int l) {
  return l == 0 || ((uint32_t)(t + 1) % (uint32_t)lv.pw[l]) == 0u;
}

template <typename Tout, int D>
__global__ void __launch_bounds__(256) k_scatter_last(const __half* __restrict__ os,
                                                      const int32_t* __restrict__ slot,
                                                      Tout* __restrict__ o, float* __restrict__ inv_count,
                                                      const Lv lv, int64_t u0) {
  pdl_enter();
  constexpr int G = D / 8, kGroups = 256 / G;
  const int32_t t = (int32_t)blockIdx.x * kGroups + (int32_t)(threadIdx.x / G);
  if (t >= lv.N) return;
  const int c = (int)(threadIdx.x % G);
  const int64_t u = u0 + blockIdx.y;
  const int32_t* sl = slot + u * lv.M;
  const __half* src = os + u * lv.S * D + 8 * c;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int cnt = 0;
  for (int l = 0; l < lv.L; ++l) {
    if (!ends_at_t(lv, t, l)) continue;
    const int32_t s = ld_slot(sl, lv.off[l] + lvl_index(lv, t, l), lv, kBoundsScatter);
    if (s < 0) continue;
    float x[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(src + (int64_t)s * D)), x);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], x[i]);
    ++cnt;
  }
  if (cnt > 0) {
    const float y = kRcpCount[cnt], cf = (float)cnt;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = div_small(acc[i], cf, y);
  }
  const int64_t row = u * lv.N + t;
  store8_stream(o + row * D + 8 * c, acc);
  if (inv_count && c == 0) inv_count[row] = kRcpCount[cnt];
}

// Adjoint: every selected entry is reached by exactly one token (its pos), so
// token t writes dO[t] / c_t to the slot of each entry that ends at it -- each
// row of dos exactly once, no accumulation.
template <typename Tin, int D>
__global__ void __launch_bounds__(256) k_scatter_bwd_last(const Tin* __restrict__ dO,
                                                          const int32_t* __restrict__ slot,
                                                          const float* __restrict__ inv_count,
                                                          __half* __restrict__ dos, const Lv lv,
                                                          int64_t u0) {
  pdl_enter();
  constexpr int G = D / 8, kGroups = 256 / G;
  const int32_t t = (int32_t)blockIdx.x * kGroups + (int32_t)(threadIdx.x / G);
  if (t >= lv.N) return;
  const int c = (int)(threadIdx.x % G);
  const int64_t u = u0 + blockIdx.y;
  const int32_t* sl = slot + u * lv.M;
  int32_t ss[kMaxLevels];
  int cnt = 0;
  for (int l = 0; l < lv.L; ++l) {
    ss[l] = ends_at_t(lv, t, l) ? ld_slot(sl, lv.off[l] + lvl_index(lv, t, l), lv, kBoundsScatterBwd) : -1;
    cnt += ss[l] >= 0 ? 1 : 0;
  }
  if (cnt == 0) return;
  const float w = inv_count ? __ldg(inv_count + u * lv.N + t) : kRcpCount[cnt];
  float x[8];
  load8(dO + (u * lv.N + t) * D + 8 * c, x);
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(x[i], w);
  __half* dst = dos + u * lv.S * D + 8 * c;
  uint32_t sat = 0;
  for (int l = 0; l < lv.L; ++l)
    if (ss[l] >= 0) store8_h(dst + (int64_t)ss[l] * D, x, sat);
  report_saturation(sat);
}

// --------------------------------------------------------------- gather bwd
// dX[t] = sum_{l ascending, selected} dxs[slot_l(t)] / p^l, X in {Q, K, V}.
// Grid: x = blocks of kRows tokens of one unit, y = unit (offset u0).
// One thread: column chunk c of R consecutive tokens sharing every entry of
// level >= 1 (as in the scatter); the slots are looked up once and the three
// arrays are done one after the other, each as one batch of independent loads.
template <typename Tout, int D, int L, int R>
__global__ void __launch_bounds__(256) k_gather_bwd(
    const float* __restrict__ dqs, const float* __restrict__ dks, const float* __restrict__ dvs,
    const int32_t* __restrict__ slot, Tout* __restrict__ dq, Tout* __restrict__ dk,
    Tout* __restrict__ dv, const Lv lv, int64_t u0) {
  pdl_enter();
  constexpr int G = D / 8, kGroups = 256 / G;
  constexpr int LC = (L > 1) ? L - 1 : 1;
  const int32_t t0 = ((int32_t)blockIdx.x * kGroups + (int32_t)(threadIdx.x / G)) * R;
  if (t0 >= lv.N) return;
  const int c = (int)(threadIdx.x % G);
  const int64_t u = u0 + blockIdx.y;
  const int32_t* sl = slot + u * lv.M;
  const int64_t base = u * lv.S * D + 8 * c;
  int32_t s0[R], sc[LC];
#pragma unroll
  for (int r = 0; r < R; ++r) s0[r] = ld_slot(sl, t0 + r, lv, kBoundsGatherBwd);
#pragma unroll
  for (int l = 1; l < L; ++l) sc[l - 1] = ld_slot(sl, lv.off[l] + lvl_index(lv, t0, l), lv, kBoundsGatherBwd);
  float inv[LC];
#pragma unroll
  for (int l = 1; l < L; ++l) inv[l - 1] = __frcp_rn((float)lv.pw[l]);
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const float* src = (a == 0 ? dqs : a == 1 ? dks : dvs) + base;
    Tout* dst = (a == 0 ? dq : a == 1 ? dk : dv) + (u * lv.N + t0) * D + 8 * c;
    float x0[R][8], xc[LC][8];
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (s0[r] >= 0) load8(src + (int64_t)s0[r] * D, x0[r]);
#pragma unroll
    for (int l = 1; l < L; ++l)
      if (sc[l - 1] >= 0) load8(src + (int64_t)sc[l - 1] * D, xc[l - 1]);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = s0[r] >= 0 ? x0[r][i] : 0.0f;  // level 0: weight 1
#pragma unroll
      for (int l = 1; l < L; ++l) {  // ascending level
        if (sc[l - 1] >= 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(xc[l - 1][i], inv[l - 1], acc[i]);
        }
      }
      store8_stream(dst + (int64_t)r * D, acc);
    }
  }
}

// Same result as k_gather_bwd (the same fused multiply-adds in the same order),
// for p = P in {2, 4} known at compile time.  One array per thread (grid z), and
// a thread walks kGatherEntries consecutive level-1 entries (P tokens each) with
// the next entry's slot loads in flight while the current entry's rows load, so
// an entry costs one memory round trip.  A token not selected at level 0 starts
// its chain from 0 (0 + x*w = x*w exactly in the first fused multiply-add), the
// same chain for all P tokens of its level-1 entry: done once, stored P times.
constexpr int kGatherEntries = 4;

template <typename Tout, int D, int L, int P>
__global__ void __launch_bounds__(128) k_gather_bwd_pp(
    const float* __restrict__ dqs, const float* __restrict__ dks, const float* __restrict__ dvs,
    const int32_t* __restrict__ slot, Tout* __restrict__ dq, Tout* __restrict__ dk,
    Tout* __restrict__ dv, const Lv lv, int64_t u0) {
  pdl_enter();
  static_assert(L >= 2 && (P == 2 || P == 4), "specialised on p in {2, 4}, L >= 2");
  constexpr int G = D / 8, kGroups = 128 / G, NE = kGatherEntries;
  constexpr int NU = (L > 2) ? L - 2 : 1;  // levels >= 2: one entry each
  const int32_t n1 = lv.N / P;
  const int32_t e0 = ((int32_t)blockIdx.x * kGroups + (int32_t)(threadIdx.x / G)) * NE;
  if (e0 >= n1) return;
  const int c = (int)(threadIdx.x % G);
  const int64_t u = u0 + blockIdx.y;
  const int a = (int)blockIdx.z;
  const int32_t* sl = slot + u * lv.M;
  const float* src = (a == 0 ? dqs : a == 1 ? dks : dvs) + u * lv.S * D + 8 * c;
  Tout* dst = (a == 0 ? dq : a == 1 ? dk : dv) + u * lv.N * D + 8 * c;

  struct Slots {
    int32_t s0[P], s1, su[NU];
  };
  auto load_slots = [&](int32_t e, Slots& sv) {
    const int32_t t = e * P;
#pragma unroll
    for (int r = 0; r < P; ++r) sv.s0[r] = ld_slot(sl, t + r, lv, kBoundsGatherBwd);
    sv.s1 = ld_slot(sl, lv.off[1] + e, lv, kBoundsGatherBwd);
    static_for<2, L>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      sv.su[l - 2] = ld_slot(sl, lv.off[l] + (int32_t)((uint32_t)e / (uint32_t)ipow(P, l - 1)), lv, kBoundsGatherBwd);
    });
  };
  auto row = [&](int32_t sidx, float (&x)[8]) {
    if (sidx >= 0) {
      load8(src + (int64_t)sidx * D, x);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.0f;
    }
  };
  Slots cur;
  load_slots(e0, cur);
#pragma unroll 1
  for (int k = 0; k < NE; ++k) {
    const int32_t e = e0 + k;
    if (e >= n1) break;
    float x0[P][8], x1[8], xu[NU][8];
#pragma unroll
    for (int r = 0; r < P; ++r) row(cur.s0[r], x0[r]);
    row(cur.s1, x1);
#pragma unroll
    for (int l = 2; l < L; ++l) row(cur.su[l - 2], xu[l - 2]);
    Slots nxt;
    if (k + 1 < NE && e + 1 < n1) load_slots(e + 1, nxt);  // in flight with this entry's rows
    // chain of a token unselected at level 0: 0, then + x_l / p^l for the
    // selected coarse levels, ascending (a level not selected adds nothing)
    float base[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) base[i] = 0.0f;
    if (cur.s1 >= 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) base[i] = __fmaf_rn(x1[i], 1.0f / (float)P, base[i]);
    }
    static_for<2, L>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      if (cur.su[l - 2] >= 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          base[i] = __fmaf_rn(xu[l - 2][i], 1.0f / (float)ipow(P, l), base[i]);
      }
    });
    Packed8<Tout> ob;
    ob.pack(base);
    Tout* out = dst + (int64_t)e * P * D;
#pragma unroll
    for (int r = 0; r < P; ++r) {
      if (cur.s0[r] >= 0) {  // selected at level 0: its own chain x_0 + x_1/p + ...
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = x0[r][i];
        if (cur.s1 >= 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(x1[i], 1.0f / (float)P, acc[i]);
        }
        static_for<2, L>([&](auto lc) {
          constexpr int l = decltype(lc)::value;
          if (cur.su[l - 2] >= 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              acc[i] = __fmaf_rn(xu[l - 2][i], 1.0f / (float)ipow(P, l), acc[i]);
          }
        });
        Packed8<Tout> pr;
        pr.pack(acc);
        pr.store(out + r * D);
      } else {
        ob.store(out + r * D);
      }
    }
    if (k + 1 < NE) cur = nxt;
  }
}

// ------------------------------------------- backward softmax statistics
// Tile-padded so that one bulk copy brings a 128-row tile's statistics: for
// unit u and tile t (T tiles per unit), row r = 128 t + c of the sub-sequence,
//   stats[(u T + t) 256 + c]       = -lse[r] log2(e)
//   stats[(u T + t) 256 + 128 + c] = -D[r],  D[r] = rowsum(dos[r] * os[r]);
// rows past S hold -inf and 0, which make every term they enter exactly zero.
template <int D>
__global__ void __launch_bounds__(256) k_attn_stats(const __half* __restrict__ os,
                                                    const __half* __restrict__ dos,
                                                    const float* __restrict__ lse,
                                                    float* __restrict__ stats, int S, int T,
                                                    int64_t prows) {
  pdl_enter();
  constexpr int G = D / 8;  // threads per row, 8 columns each
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t prow = gt / G;  // padded row over all units
  if (prow >= prows) return;    // whole groups leave together
  const int c = (int)(gt % G);
  const int64_t u = prow / ((int64_t)T * 128);
  const int rr = (int)(prow - u * T * 128);
  float* dst = stats + (u * T + (rr >> 7)) * 256 + (rr & 127);
  if (rr >= S) {
    if (c == 0) {
      dst[0] = -INFINITY;
      dst[128] = 0.0f;
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  const unsigned gmask = ((G == 32) ? 0xffffffffu : ((1u << G) - 1u)) << (lane & ~(G - 1));
  const int64_t row = u * S + rr;
  float a[8], b[8];
  load8(os + row * D + 8 * c, a);
  load8(dos + row * D + 8 * c, b);
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s = __fmaf_rn(a[i], b[i], s);
#pragma unroll
  for (int off = 1; off < G; off <<= 1) s = __fadd_rn(s, __shfl_xor_sync(gmask, s, off));
  if (c == 0) {
    dst[0] = -lse[row] * 1.4426950408889634f;
    dst[128] = -s;
  }
}

}  // namespace

cudaError_t launch_gather(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                          const float* pq, const float* pk, const float* pv, const int32_t* idx,
                          __half* qs, __half* ks, __half* vs, cudaStream_t st) {
  const Lv lv = make_lv(g);
  const int64_t rows = g.U * g.S;
  const unsigned nb = blocks_for(rows * (g.d / 8), 256);
  if (dt == LH_BF16) {
    auto* a = static_cast<const __nv_bfloat16*>(q);
    auto* b = static_cast<const __nv_bfloat16*>(k);
    auto* c = static_cast<const __nv_bfloat16*>(v);
    if (g.d == 64)
      (void)launch_pdl(k_gather<__nv_bfloat16, 64>, nb, 256, 0, st, a, b, c, pq, pk, pv, idx, qs, ks, vs, lv, rows);
    else
      (void)launch_pdl(k_gather<__nv_bfloat16, 128>, nb, 256, 0, st, a, b, c, pq, pk, pv, idx, qs, ks, vs, lv, rows);
  } else {
    auto* a = static_cast<const float*>(q);
    auto* b = static_cast<const float*>(k);
    auto* c = static_cast<const float*>(v);
    if (g.d == 64)
      (void)launch_pdl(k_gather<float, 64>, nb, 256, 0, st, a, b, c, pq, pk, pv, idx, qs, ks, vs, lv, rows);
    else
      (void)launch_pdl(k_gather<float, 128>, nb, 256, 0, st, a, b, c, pq, pk, pv, idx, qs, ks, vs, lv, rows);
  }
  return cudaGetLastError();
}

namespace {
template <typename Tin, int D>
cudaError_t gather_pooled_d(const Geom& g, const Tin* q, const Tin* k, const Tin* v,
                            const int32_t* idx, __half* qs, __half* ks, __half* vs,
                            cudaStream_t st) {
  const Lv lv = make_lv(g);
  const int64_t rows = g.U * g.S;
  const unsigned nb = blocks_for(rows * (D / 8), 256);
  switch (g.L) {
#define LH_CASE(LL)                                                                              \
  case LL:                                                                                       \
    (void)launch_pdl(k_gather_pooled<Tin, D, LL>, nb, 256, 0, st, q, k, v, idx, qs, ks, vs, lv, rows);        \
    break;
    LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_gather_pooled(const Geom& g, lh_dtype dt, const void* q, const void* k,
                                 const void* v, const int32_t* idx, __half* qs, __half* ks,
                                 __half* vs, cudaStream_t st) {
  if (dt == LH_BF16) {
    auto* a = static_cast<const __nv_bfloat16*>(q);
    auto* b = static_cast<const __nv_bfloat16*>(k);
    auto* c = static_cast<const __nv_bfloat16*>(v);
    return g.d == 64 ? gather_pooled_d<__nv_bfloat16, 64>(g, a, b, c, idx, qs, ks, vs, st)
                     : gather_pooled_d<__nv_bfloat16, 128>(g, a, b, c, idx, qs, ks, vs, st);
  }
  auto* a = static_cast<const float*>(q);
  auto* b = static_cast<const float*>(k);
  auto* c = static_cast<const float*>(v);
  return g.d == 64 ? gather_pooled_d<float, 64>(g, a, b, c, idx, qs, ks, vs, st)
                   : gather_pooled_d<float, 128>(g, a, b, c, idx, qs, ks, vs, st);
}

namespace {
// Runs f(std::integral_constant<int, L>) for the shape's level count.
template <typename F>
cudaError_t with_levels(int L, F&& f) {
  switch (L) {
    case 1: f(std::integral_constant<int, 1>{}); break;
    case 2: f(std::integral_constant<int, 2>{}); break;
    case 3: f(std::integral_constant<int, 3>{}); break;
    case 4: f(std::integral_constant<int, 4>{}); break;
    case 5: f(std::integral_constant<int, 5>{}); break;
    case 6: f(std::integral_constant<int, 6>{}); break;
    case 7: f(std::integral_constant<int, 7>{}); break;
    case 8: f(std::integral_constant<int, 8>{}); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// 2-D grid over (token blocks of one unit, units), units in chunks of 65535.
template <typename F>
void per_unit_chunks(int64_t U, F&& f) {
  for (int64_t u0 = 0; u0 < U; u0 += 65535) f(u0, (unsigned)(U - u0 < 65535 ? U - u0 : 65535));
}

// Tokens per thread for the scatter and the gather adjoint: R consecutive
// tokens share all coarser entries when R divides p (and L > 1).
inline int tokens_per_thread(const Geom& g) {
  if (g.L < 2) return 1;
  return g.p % 4 == 0 ? 4 : (g.p % 2 == 0 ? 2 : 1);
}

template <typename F>
cudaError_t with_tokens(int R, F&& f) {
  if (R == 4) return f(std::integral_constant<int, 4>{});
  if (R == 2) return f(std::integral_constant<int, 2>{});
  return f(std::integral_constant<int, 1>{});
}

template <typename Tout, int D>
cudaError_t scatter_t(const Geom& g, const __half* os, const int32_t* slot, Tout* o,
                      float* inv_count, cudaStream_t st) {
  const Lv lv = make_lv(g);
  if (g.scatter_mode == LH_SCATTER_LAST) {
    const unsigned bxl = blocks_for(g.N, 256 / (D / 8));
    per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
      (void)launch_pdl(k_scatter_last<Tout, D>, dim3(bxl, nu), 256, 0, st, os, slot, o, inv_count, lv, u0);
    });
    return cudaGetLastError();
  }
  if (g.L >= 2 && (g.p == 2 || g.p == 4)) {  // p known at compile time: p tokens a thread
    const unsigned bxp = blocks_for(g.N / g.p, (128 / (D / 8)) * kScatterEntries);
    return with_levels(g.L, [&](auto lc) {
      constexpr int LL = decltype(lc)::value;
      if constexpr (LL >= 2) {
        per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
          if (g.p == 4)
            (void)launch_pdl(k_scatter_pp<Tout, D, LL, 4>, dim3(bxp, nu), 128, 0, st, os, slot, o, inv_count, lv, u0);
          else
            (void)launch_pdl(k_scatter_pp<Tout, D, LL, 2>, dim3(bxp, nu), 128, 0, st, os, slot, o, inv_count, lv, u0);
        });
      }
    });
  }
  const int R = tokens_per_thread(g);
  const unsigned bx = blocks_for(g.N / R, 256 / (D / 8));
  return with_tokens(R, [&](auto rc) {
    return with_levels(g.L, [&](auto lc) {
      per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
        (void)launch_pdl(k_scatter<Tout, D, decltype(lc)::value, decltype(rc)::value>, dim3(bx, nu), 256, 0, st, os, slot, o, inv_count, lv, u0);
      });
    });
  });
}

template <typename Tout, int D>
cudaError_t gather_bwd_t(const Geom& g, const float* dqs, const float* dks, const float* dvs,
                         const int32_t* slot, Tout* dq, Tout* dk, Tout* dv, cudaStream_t st) {
  const Lv lv = make_lv(g);
  if (g.L >= 2 && (g.p == 2 || g.p == 4)) {  // p known at compile time, one array per thread
    const unsigned bxp = blocks_for(g.N / g.p, (128 / (D / 8)) * kGatherEntries);
    return with_levels(g.L, [&](auto lc) {
      constexpr int LL = decltype(lc)::value;
      if constexpr (LL >= 2) {
        per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
          if (g.p == 4)
            (void)launch_pdl(k_gather_bwd_pp<Tout, D, LL, 4>, dim3(bxp, nu, 3), 128, 0, st, dqs, dks, dvs, slot, dq, dk, dv, lv, u0);
          else
            (void)launch_pdl(k_gather_bwd_pp<Tout, D, LL, 2>, dim3(bxp, nu, 3), 128, 0, st, dqs, dks, dvs, slot, dq, dk, dv, lv, u0);
        });
      }
    });
  }
  const int R = tokens_per_thread(g);
  const unsigned bx = blocks_for(g.N / R, 256 / (D / 8));
  return with_tokens(R, [&](auto rc) {
    return with_levels(g.L, [&](auto lc) {
      per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
        (void)launch_pdl(k_gather_bwd<Tout, D, decltype(lc)::value, decltype(rc)::value>, dim3(bx, nu), 256, 0, st, dqs, dks, dvs, slot, dq, dk, dv, lv, u0);
      });
    });
  });
}
}  // namespace

cudaError_t launch_scatter(const Geom& g, lh_dtype dt, const __half* os,
                           const int32_t* slot, void* o, float* inv_count, cudaStream_t st) {
  if (dt == LH_BF16) {
    auto* out = static_cast<__nv_bfloat16*>(o);
    return g.d == 64 ? scatter_t<__nv_bfloat16, 64>(g, os, slot, out, inv_count, st)
                     : scatter_t<__nv_bfloat16, 128>(g, os, slot, out, inv_count, st);
  }
  auto* out = static_cast<float*>(o);
  return g.d == 64 ? scatter_t<float, 64>(g, os, slot, out, inv_count, st)
                   : scatter_t<float, 128>(g, os, slot, out, inv_count, st);
}

namespace {
template <typename Tin, int D>
cudaError_t scatter_bwd_d(const Geom& g, const Tin* dO, const int32_t* slot, const float* ic,
                          __half* dos, cudaStream_t st) {
  const Lv lv = make_lv(g);
  if (g.scatter_mode == LH_SCATTER_LAST) {
    const unsigned bxl = blocks_for(g.N, 256 / (D / 8));
    per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
      (void)launch_pdl(k_scatter_bwd_last<Tin, D>, dim3(bxl, nu), 256, 0, st, dO, slot, ic, dos, lv, u0);
    });
    return cudaGetLastError();
  }
  const int64_t spans = g.N / g.pw[g.L - 1];
  const int64_t groups = g.U * spans;
  // row-groups per span: p when p in {2, 4} and the span's lanes fit one warp
  const int RG = (g.L > 1 && (g.p == 2 || g.p == 4) && (D / 8) * g.p <= 32) ? g.p : 1;
  const unsigned nb = blocks_for(groups * (D / 8) * RG, 256);
  return with_levels(g.L, [&](auto lc) {
    constexpr int LL = decltype(lc)::value;
    if constexpr (LL > 1) {
      if (ic != nullptr && (g.p == 2 || g.p == 4)) {  // staged loads, p known at compile time
        auto go = [&](auto pc, auto rgc) {
          constexpr int PP = decltype(pc)::value, RR = decltype(rgc)::value;
          using C = ScatterBwdCfg<Tin, D, LL, PP, RR>;
          const unsigned bx = blocks_for(spans * (D / 8) * RR, kScatterBwdThreads);
          per_unit_chunks(g.U, [&](int64_t u0, unsigned nu) {
            (void)launch_pdl(k_scatter_bwd_pp<Tin, D, LL, PP, RR>, dim3(bx, nu), kScatterBwdThreads, C::smem_bytes, st, 
                dO, slot, ic, dos, lv, (int32_t)spans, u0);
          });
        };
        if (g.p == 4) {
          if (RG == 4) {
            if constexpr ((D / 8) * 4 <= 32)
              go(std::integral_constant<int, 4>{}, std::integral_constant<int, 4>{});
          } else {
            go(std::integral_constant<int, 4>{}, std::integral_constant<int, 1>{});
          }
        } else {
          go(std::integral_constant<int, 2>{}, std::integral_constant<int, 2>{});
        }
        return;
      }
      if (RG == 4) {
        if constexpr ((D / 8) * 4 <= 32) {
          (void)launch_pdl(k_scatter_bwd<Tin, D, LL, 4>, nb, 256, 0, st, dO, slot, ic, dos, lv, spans, groups);
          return;
        }
      }
      if (RG == 2) {
        (void)launch_pdl(k_scatter_bwd<Tin, D, LL, 2>, nb, 256, 0, st, dO, slot, ic, dos, lv, spans, groups);
        return;
      }
    }
    (void)launch_pdl(k_scatter_bwd<Tin, D, LL, 1>, nb, 256, 0, st, dO, slot, ic, dos, lv, spans, groups);
  });
}
}  // namespace

cudaError_t launch_scatter_bwd(const Geom& g, lh_dtype dt, const void* dO, const int32_t* slot,
                               const float* inv_count, __half* dos, cudaStream_t st) {
  if (dt == LH_BF16) {
    auto* a = static_cast<const __nv_bfloat16*>(dO);
    return g.d == 64 ? scatter_bwd_d<__nv_bfloat16, 64>(g, a, slot, inv_count, dos, st)
                     : scatter_bwd_d<__nv_bfloat16, 128>(g, a, slot, inv_count, dos, st);
  }
  auto* a = static_cast<const float*>(dO);
  return g.d == 64 ? scatter_bwd_d<float, 64>(g, a, slot, inv_count, dos, st)
                   : scatter_bwd_d<float, 128>(g, a, slot, inv_count, dos, st);
}

cudaError_t launch_gather_bwd(const Geom& g, lh_dtype dt, const float* dqs, const float* dks,
                              const float* dvs, const int32_t* slot, void* dq, void* dk, void* dv,
                              cudaStream_t st) {
  if (dt == LH_BF16) {
    auto* a = static_cast<__nv_bfloat16*>(dq);
    auto* b = static_cast<__nv_bfloat16*>(dk);
    auto* c = static_cast<__nv_bfloat16*>(dv);
    return g.d == 64 ? gather_bwd_t<__nv_bfloat16, 64>(g, dqs, dks, dvs, slot, a, b, c, st)
                     : gather_bwd_t<__nv_bfloat16, 128>(g, dqs, dks, dvs, slot, a, b, c, st);
  }
  auto* a = static_cast<float*>(dq);
  auto* b = static_cast<float*>(dk);
  auto* c = static_cast<float*>(dv);
  return g.d == 64 ? gather_bwd_t<float, 64>(g, dqs, dks, dvs, slot, a, b, c, st)
                   : gather_bwd_t<float, 128>(g, dqs, dks, dvs, slot, a, b, c, st);
}

cudaError_t launch_attn_stats(const Geom& g, const __half* os, const __half* dos,
                              const float* lse, float* stats, cudaStream_t st) {
  const int T = (int)((g.S + 127) / 128);
  const int64_t prows = g.U * T * 128;
  const unsigned nb = blocks_for(prows * (g.d / 8), 256);
  if (g.d == 64)
    (void)launch_pdl(k_attn_stats<64>, nb, 256, 0, st, os, dos, lse, stats, (int)g.S, T, prows);
  else
    (void)launch_pdl(k_attn_stats<128>, nb, 256, 0, st, os, dos, lse, stats, (int)g.S, T, prows);
  return cudaGetLastError();
}

}  // namespace lh
