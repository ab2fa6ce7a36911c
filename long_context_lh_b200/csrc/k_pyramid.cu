// k_pyramid.cu -- pyramid levels and entry scores in one pass over Q, K, V.
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.A (each level summarises p consecutive
// entries of the level below, Q, K and V alike) and §2.B (l2 norms of Q and K
// per entry, coarse levels inherit the max of their children); the averaging is
// phase 1 ("Pyramid Pool") of bitsgeniais.com.br "Adeus Custo Quadrático! ...".
//
// Work decomposition: a group of G = d/8 consecutive lanes owns one coarsest
// span (p^(L-1) tokens) of one unit; lane c owns columns [8c, 8c+8).  The group
// walks its span row by row with 128-bit loads, so every element of Q, K and V
// is read from HBM exactly once, and keeps one running sum per level in
// registers: when p children of level l are complete their mean is written and
// added to level l+1.  The level-0 score needs the whole row, so the G lanes
// combine their partial sums of squares with an xor-shuffle tree that yields
// the same bits in every lane.
//
// Score arithmetic (fixed, so the selection is reproducible bit for bit):
//   a_c = fmaf chain over x[8c+0..7]^2 from 0;  tree over c with offsets
//   1, 2, 4(, 8);  score = sqrt_rn(ss(Q)) + sqrt_rn(ss(K)).
#include "lh_internal.cuh"

namespace lh {
namespace {

struct PyrParams {
  int64_t N, M, spans, groups, Ptop;
  int p;
  int64_t off[kMaxLevels + 1];
  int64_t pw[kMaxLevels + 1];
};

template <typename T>
struct Raw;
template <>
struct Raw<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    w = __ldcs(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
    x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
    x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
  }
};
template <>
struct Raw<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldcs(reinterpret_cast<const float4*>(p));
    b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

__device__ __forceinline__ float sumsq8(const float (&x)[8]) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = __fmaf_rn(x[i], x[i], a);
  return a;
}

// Rows of the coarsest span processed per batch of loads (loads issued first).
constexpr int kRowBatch = 4;

template <typename Tin, int D, int L, bool kPyr, bool kScore>
__global__ void __launch_bounds__(256) k_pyramid_score(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    float* __restrict__ pq, float* __restrict__ pk, float* __restrict__ pv,
    float* __restrict__ score, const PyrParams prm) {
  constexpr int G = D / 8;
  constexpr int NL = (L > 1) ? (L - 1) : 1;  // accumulators for levels 1..L-1
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t group = gtid / G;
  const int c = (int)(gtid % G);
  if (group >= prm.groups) return;  // whole groups leave together (G | 32)
  const int lane = threadIdx.x & 31;
  const unsigned gmask = ((G == 32) ? 0xffffffffu : ((1u << G) - 1u)) << (lane & ~(G - 1));

  const int64_t u = group / prm.spans;
  const int64_t t0 = (group % prm.spans) * prm.Ptop;
  const int64_t row0 = (u * prm.N + t0) * D + 8 * c;
  const Tin* qp = q + row0;
  const Tin* kp = k + row0;
  const Tin* vp = v + row0;
  float* sc = score + u * prm.M;
  const int64_t pyr_unit = u * (prm.M - prm.N);

  float aq[NL][8], ak[NL][8], av[NL][8];
  float smax[NL];
  int cnt[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) {
    smax[l] = 0.0f;
    cnt[l] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) aq[l][i] = ak[l][i] = av[l][i] = 0.0f;
  }

  for (int64_t r0 = 0; r0 < prm.Ptop; r0 += kRowBatch) {
    Raw<Tin> rq[kRowBatch], rk[kRowBatch], rv[kRowBatch];
#pragma unroll
    for (int b = 0; b < kRowBatch; ++b) {
      if (r0 + b < prm.Ptop) {
        const int64_t o = (r0 + b) * D;
        rq[b].load(qp + o);
        rk[b].load(kp + o);
        if (kPyr) rv[b].load(vp + o);
      }
    }
#pragma unroll
    for (int b = 0; b < kRowBatch; ++b) {
      const int64_t r = r0 + b;
      if (r >= prm.Ptop) break;
      float xq[8], xk[8], xv[8];
      rq[b].unpack(xq);
      rk[b].unpack(xk);
      if (kPyr) rv[b].unpack(xv);
      // level-0 score (all lanes of the group end with identical bits)
      float s0 = 0.0f;
      if (kScore) {
        float ssq = sumsq8(xq), ssk = sumsq8(xk);
#pragma unroll
        for (int off = 1; off < G; off <<= 1) {
          ssq = __fadd_rn(ssq, __shfl_xor_sync(gmask, ssq, off));
          ssk = __fadd_rn(ssk, __shfl_xor_sync(gmask, ssk, off));
        }
        s0 = __fadd_rn(__fsqrt_rn(ssq), __fsqrt_rn(ssk));
        if (c == (int)(r % G)) sc[t0 + r] = s0;
      }
      if constexpr (L == 1) continue;
      // feed level 1
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (kPyr) {
          aq[0][i] = __fadd_rn(aq[0][i], xq[i]);
          ak[0][i] = __fadd_rn(ak[0][i], xk[i]);
          av[0][i] = __fadd_rn(av[0][i], xv[i]);
        }
      }
      smax[0] = fmaxf(smax[0], s0);
      cnt[0] += 1;
      // cascade completed levels upward
#pragma unroll
      for (int l = 0; l < NL; ++l) {
        if (cnt[l] == prm.p) {
          const int lev = l + 1;
          const int64_t j = (t0 + r + 1) / prm.pw[lev] - 1;
          const float fp = (float)prm.p;
          float mq[8], mk[8], mv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            mq[i] = __fdiv_rn(aq[l][i], fp);
            mk[i] = __fdiv_rn(ak[l][i], fp);
            mv[i] = __fdiv_rn(av[l][i], fp);
          }
          if (kPyr) {
            const int64_t prow = (pyr_unit + prm.off[lev] - prm.N + j) * D + 8 * c;
            store8(pq + prow, mq);
            store8(pk + prow, mk);
            store8(pv + prow, mv);
          }
          if (kScore && c == 0) sc[prm.off[lev] + j] = smax[l];
          if (l + 1 < NL) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              aq[l + 1][i] = __fadd_rn(aq[l + 1][i], mq[i]);
              ak[l + 1][i] = __fadd_rn(ak[l + 1][i], mk[i]);
              av[l + 1][i] = __fadd_rn(av[l + 1][i], mv[i]);
            }
            smax[l + 1] = fmaxf(smax[l + 1], smax[l]);
            cnt[l + 1] += 1;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) aq[l][i] = ak[l][i] = av[l][i] = 0.0f;
          smax[l] = 0.0f;
          cnt[l] = 0;
        }
      }
    }
  }
}

template <typename Tin, int D, int L>
cudaError_t launch_tl(const Geom& g, const void* q, const void* k, const void* v, float* pq,
                      float* pk, float* pv, float* score, cudaStream_t st) {
  PyrParams prm;
  prm.N = g.N;
  prm.M = g.M;
  prm.p = g.p;
  prm.Ptop = g.pw[g.L - 1];
  prm.spans = g.N / prm.Ptop;
  prm.groups = g.U * prm.spans;
  for (int l = 0; l <= kMaxLevels; ++l) {
    prm.off[l] = g.off[l];
    prm.pw[l] = g.pw[l];
  }
  const int64_t threads = prm.groups * (D / 8);
  const int block = 256;
  const int64_t grid = (threads + block - 1) / block;
  const Tin* tq = static_cast<const Tin*>(q);
  const Tin* tk = static_cast<const Tin*>(k);
  const Tin* tv = static_cast<const Tin*>(v);
  if (pq && score)
    k_pyramid_score<Tin, D, L, true, true><<<grid, block, 0, st>>>(tq, tk, tv, pq, pk, pv, score, prm);
  else if (pq)
    k_pyramid_score<Tin, D, L, true, false><<<grid, block, 0, st>>>(tq, tk, tv, pq, pk, pv, score, prm);
  else
    k_pyramid_score<Tin, D, L, false, true><<<grid, block, 0, st>>>(tq, tk, tv, pq, pk, pv, score, prm);
  return cudaGetLastError();
}

template <typename Tin, int D>
cudaError_t launch_t(const Geom& g, const void* q, const void* k, const void* v, float* pq,
                     float* pk, float* pv, float* score, cudaStream_t st) {
  switch (g.L) {
    case 1: return launch_tl<Tin, D, 1>(g, q, k, v, pq, pk, pv, score, st);
    case 2: return launch_tl<Tin, D, 2>(g, q, k, v, pq, pk, pv, score, st);
    case 3: return launch_tl<Tin, D, 3>(g, q, k, v, pq, pk, pv, score, st);
    case 4: return launch_tl<Tin, D, 4>(g, q, k, v, pq, pk, pv, score, st);
    case 5: return launch_tl<Tin, D, 5>(g, q, k, v, pq, pk, pv, score, st);
    case 6: return launch_tl<Tin, D, 6>(g, q, k, v, pq, pk, pv, score, st);
    case 7: return launch_tl<Tin, D, 7>(g, q, k, v, pq, pk, pv, score, st);
    case 8: return launch_tl<Tin, D, 8>(g, q, k, v, pq, pk, pv, score, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// pq/pk/pv == nullptr: scores only; score == nullptr: pyramid only.
cudaError_t launch_pyramid_score(const Geom& g, lh_dtype dt, const void* q, const void* k,
                                 const void* v, float* pq, float* pk, float* pv, float* score,
                                 cudaStream_t st) {
  if (dt == LH_BF16) {
    if (g.d == 64) return launch_t<__nv_bfloat16, 64>(g, q, k, v, pq, pk, pv, score, st);
    return launch_t<__nv_bfloat16, 128>(g, q, k, v, pq, pk, pv, score, st);
  }
  if (g.d == 64) return launch_t<float, 64>(g, q, k, v, pq, pk, pv, score, st);
  return launch_t<float, 128>(g, q, k, v, pq, pk, pv, score, st);
}

}  // namespace lh
