// k_pyramid.cu -- pyramid levels and entry scores in one pass over Q, K, V.
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.A (each level summarises p consecutive
// entries of the level below, Q, K and V alike) and §2.B (l2 norms of Q and K
// per entry, coarse levels inherit the max of their children); the averaging is
// phase 1 ("Pyramid Pool") of bitsgeniais.com.br "Adeus Custo Quadrático! ...".
//
// Work decomposition.  A block owns a chunk of CR consecutive tokens of one
// unit (CR = m p^J <= 64 rows and <= 8 KB per tensor, J the highest level
// whose entries fit in a chunk).
// It copies the chunk's rows of Q, K (and V) into shared memory with 16-byte
// asynchronous copies -- every element is read from HBM once, and the several
// blocks resident per SM keep enough copies in flight to cover the latency --
// then computes, from shared memory:
//   level 1   one thread per (entry, 8-column chunk c, tensor): the sum of the
//             p children in order, then the mean; for Q and K the same thread
//             also forms each child row's partial sum of squares a_c;
//   level 0   the scores, one thread per row, from the partials a_c;
//   level l   (2 <= l <= J) as level 1 from level l-1; scores: max of the
//             children.  Level l is kept in shared memory (fp32) for l+1.
// (Without level 1 in the chunk -- L = 1, or scores only -- G = d/8 lanes per
// row form the level-0 scores with a shuffle tree instead.)
// Levels above J (entries wider than a chunk) are built by a small kernel per
// level from the level below in HBM; when p^(L-1) fits a chunk there are none.
//
// Arithmetic (fixed, so the selection is reproducible bit for bit):
//   score:  a_c = fmaf chain over x[8c+0..7]^2 from 0; tree over c with offsets
//           1, 2, 4(, 8); score = sqrt_rn(ss(Q)) + sqrt_rn(ss(K)) (the default;
//           the ablations: their product, or sqrt_rn(ss(Q) + ss(K)));
//           coarse score = max(0, children in order) (scores are >= 0);
//   mean:   ((0 + c_0) + c_1) + ... + c_{p-1}, then / p (round to nearest; for
//           p a power of two the product with 1/p, which is the same number).
#include <type_traits>

#include "lh_internal.cuh"

namespace lh {

// Status word of the pyramid and score kernels (bounds checks of the debug build).
__device__ uint32_t g_pyramid_status = 0;
#define LH_STATUS_WORD g_pyramid_status

cudaError_t pyramid_status_read_clear(uint32_t* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_pyramid_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_pyramid_status, &zero, sizeof(zero));
}

namespace {

// Upper bound on CR: 64 rows and 8 KB of each tensor per chunk (64 rows of
// bf16 at d = 64).
inline int chunk_rows_cap(int d, size_t elem) {
  const int cap = (int)(8192 / ((size_t)d * elem));
  return cap < 64 ? cap : 64;
}

struct PyrPrm {
  int32_t N, M, CR, p, J, L;
  int32_t score_mode;  // lh_score_mode
  int32_t pow2;  // p is a power of two: mean = sum * inv_p exactly
  float inv_p;
  double inv_pd;  // 1/p in fp64 for the exact division (div_exact) otherwise
  int32_t off[kMaxLevels + 1];
  int32_t pw[kMaxLevels + 1];
};

// Level-0 score from the squared norms of the token's q and k rows: their norms'
// sum (default), product, or the norm of the concatenation [q; k].
__device__ __forceinline__ float combine_norms(float ssq, float ssk, int mode) {
  if (mode == LH_SCORE_PRODUCT) return __fmul_rn(__fsqrt_rn(ssq), __fsqrt_rn(ssk));
  if (mode == LH_SCORE_CONCAT) return __fsqrt_rn(__fadd_rn(ssq, ssk));
  return __fadd_rn(__fsqrt_rn(ssq), __fsqrt_rn(ssk));
}

template <int P>
__device__ __forceinline__ float mean_of(float sum, const PyrPrm& prm) {
  if constexpr (P > 0 && (P & (P - 1)) == 0) return sum * (1.0f / (float)P);
  return prm.pow2 ? sum * prm.inv_p : div_exact(sum, prm.inv_pd);
}

constexpr int ipow(int b, int e) { return e == 0 ? 1 : b * ipow(b, e - 1); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// 8 consecutive elements of a shared-memory row as float
__device__ __forceinline__ void smem8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void smem8(const float* p, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void put8(float* p, const float (&x)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

__device__ __forceinline__ float sumsq8(const float (&x)[8]) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = __fmaf_rn(x[i], x[i], a);
  return a;
}

// Shared memory of the chunk kernel, in bytes.
template <typename Tin, int D, bool kPyr>
struct ChunkSmem {
  static constexpr int NT = kPyr ? 3 : 2;
  static constexpr size_t in_bytes(int CR) { return (size_t)NT * CR * D * sizeof(Tin); }
  // two score rows of CR floats, padded so the fp32 level buffers stay 16-byte aligned
  static constexpr int score_floats(int CR) { return (2 * CR + 3) & ~3; }
  static constexpr size_t score_bytes(int CR) { return (size_t)score_floats(CR) * sizeof(float); }
  // ping-pong fp32 level buffers: A holds CR/p rows per tensor, B CR/p^2 (>= 1)
  static size_t lev_rows_a(int CR, int p) { return (size_t)(CR / p); }
  static size_t lev_rows_b(int CR, int p) { return (size_t)(CR / p / p > 0 ? CR / p / p : 1); }
  static size_t bytes(int CR, int p) {
    size_t b = in_bytes(CR) + score_bytes(CR);
    if (kPyr) {
      b += (size_t)3 * (lev_rows_a(CR, p) + lev_rows_b(CR, p)) * D * sizeof(float);
      b += (size_t)2 * CR * (D / 8) * sizeof(float);  // partial sums of squares
    }
    return b;
  }
};

// P > 0: p == P known at compile time (child loops unrolled, level widths
// constant); P == 0: any p.
template <typename Tin, int D, int P, bool kPyr, bool kScore>
__global__ void __launch_bounds__(256) k_pyr_chunk(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    float* __restrict__ pq, float* __restrict__ pk, float* __restrict__ pv,
    float* __restrict__ score, const PyrPrm prm, int64_t u0) {
  pdl_enter();
  using Sm = ChunkSmem<Tin, D, kPyr>;
  constexpr int G = D / 8;
  constexpr int NT = Sm::NT;
  extern __shared__ __align__(16) uint8_t smem[];
  const int CR = prm.CR;
  const int p = P > 0 ? P : prm.p;
  Tin* sIn = reinterpret_cast<Tin*>(smem);  // [NT][CR][D]
  float* sSc = reinterpret_cast<float*>(smem + Sm::in_bytes(CR));  // [2][CR] ping-pong
  float* sLa = sSc + Sm::score_floats(CR);                           // [3][CR/p][D]
  float* sLb = sLa + (size_t)3 * (CR / p) * D;                       // [3][CR/p^2][D]
  const int ra = CR / p, rb = (CR / p / p > 0) ? CR / p / p : 1;

  const int tid = threadIdx.x;
  const int32_t t0 = (int32_t)blockIdx.x * CR;
  const int64_t u = u0 + blockIdx.y;
  const int rows = (prm.N - t0 < CR) ? prm.N - t0 : CR;  // a multiple of p^J

  // ---- the chunk's rows into shared memory
  {
    const int64_t g0 = (u * prm.N + t0) * D;
    const int n16 = rows * D * (int)sizeof(Tin) / 16;  // 16-byte pieces per tensor
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>((t == 0 ? q : t == 1 ? k : v) + g0);
      uint8_t* dst = reinterpret_cast<uint8_t*>(sIn + (size_t)t * CR * D);
      for (int i = tid; i < n16; i += 256) cp_async16(dst + 16 * i, src + 16 * i);
    }
    cp_async_wait_all();
    __syncthreads();
  }
  float* sc = score + u * prm.M;
  float* sPart = sLb + (size_t)3 * rb * D;  // [2][CR][G] partial sums of squares (kPyr)
  const bool fused = kPyr && prm.J >= 1;    // scores from the level-1 pass

  // ---- level-0 scores without a level-1 pass: G lanes per row, shuffle tree
  if (kScore && !fused) {
    const int c = tid % G;
    const int lane = tid & 31;
    const unsigned gmask = ((G == 32) ? 0xffffffffu : ((1u << G) - 1u)) << (lane & ~(G - 1));
    for (int r = tid / G; r < rows; r += 256 / G) {  // whole groups iterate together
      float xq[8], xk[8];
      smem8(sIn + (size_t)r * D + 8 * c, xq);
      smem8(sIn + (size_t)(CR + r) * D + 8 * c, xk);
      float ssq = sumsq8(xq), ssk = sumsq8(xk);
#pragma unroll
      for (int off = 1; off < G; off <<= 1) {
        ssq = __fadd_rn(ssq, __shfl_xor_sync(gmask, ssq, off));
        ssk = __fadd_rn(ssk, __shfl_xor_sync(gmask, ssk, off));
      }
      if (c == 0) sSc[r] = combine_norms(ssq, ssk, prm.score_mode);
    }
    __syncthreads();
    for (int r = tid; r < rows; r += 256)
      if (LH_CHECK(dbg::in_range(t0 + r, prm.N), kBoundsPyramid)) sc[t0 + r] = sSc[r];
  }

  // ---- levels 1..J
  int nprev = rows;
#pragma unroll
  for (int l = 1; l < kMaxLevels; ++l) {  // unrolled: off[l] and pw[l] are constant indices
    if (l > prm.J) break;
    const int n = nprev / p;
    const int32_t pwl = P > 0 ? ipow(P > 0 ? P : 1, l) : prm.pw[l];
    const int32_t j0 = t0 / pwl;  // first entry of this chunk at level l
    const float* prevS = sSc + ((l - 1) & 1) * CR;
    float* curS = sSc + (l & 1) * CR;
    if (kPyr) {
      const float* prevL = (l & 1) ? sLb : sLa;  // level l-1 (l >= 2)
      float* curL = (l & 1) ? sLa : sLb;
      const int prow = (l & 1) ? rb : ra;        // rows per tensor of prevL
      const int crow = (l & 1) ? ra : rb;        // rows per tensor of curL
      const int nG = n * G;
      for (int it = tid; it < 3 * nG; it += 256) {
        const int t = it >= 2 * nG ? 2 : (it >= nG ? 1 : 0);
        const int rem = it - t * nG;
        const int e = rem / G, c = rem % G;
        float acc[8], x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int i = 0; i < p; ++i) {
          const int ch = e * p + i;
          if (l == 1) {
            smem8(sIn + ((size_t)t * CR + ch) * D + 8 * c, x);
            // the child row's partial a_c of its score (Q and K)
            if (kScore && t < 2) sPart[((size_t)t * CR + ch) * G + c] = sumsq8(x);
          } else {
            smem8(prevL + ((size_t)t * prow + ch) * D + 8 * c, x);
          }
#pragma unroll
          for (int z = 0; z < 8; ++z) acc[z] = __fadd_rn(acc[z], x[z]);
        }
#pragma unroll
        for (int z = 0; z < 8; ++z) acc[z] = mean_of<P>(acc[z], prm);
        float* dst = (t == 0 ? pq : t == 1 ? pk : pv);
        if (LH_CHECK(dbg::entry_ok(j0 + e, prm.off[l], prm.off[l + 1]), kBoundsPyramid))
          put8(dst + ((u * (prm.M - prm.N) + prm.off[l] - prm.N + j0 + e) * D + 8 * c), acc);
        if (l < prm.J && LH_CHECK(dbg::in_range(e, crow), kBoundsPyramid))
          put8(curL + ((size_t)t * crow + e) * D + 8 * c, acc);
      }
    }
    if (kScore) {
      if (l == 1 && fused) {
        __syncthreads();  // all partials written
        // level-0 scores, one thread per row: the same pairwise tree over the
        // partials a_0..a_{G-1} as the shuffle tree (offsets 1, 2, 4(, 8))
        for (int r = tid; r < rows; r += 256) {
          float a[G], b[G];
#pragma unroll
          for (int c = 0; c < G; c += 4) {  // 16-byte aligned: G is a multiple of 8
            const float4 x = *reinterpret_cast<const float4*>(sPart + (size_t)r * G + c);
            const float4 y = *reinterpret_cast<const float4*>(sPart + ((size_t)CR + r) * G + c);
            a[c] = x.x; a[c + 1] = x.y; a[c + 2] = x.z; a[c + 3] = x.w;
            b[c] = y.x; b[c + 1] = y.y; b[c + 2] = y.z; b[c + 3] = y.w;
          }
#pragma unroll
          for (int off = 1; off < G; off <<= 1)
#pragma unroll
            for (int c = 0; c < G; c += 2 * off) {
              a[c] = __fadd_rn(a[c], a[c + off]);
              b[c] = __fadd_rn(b[c], b[c + off]);
            }
          const float s0 = combine_norms(a[0], b[0], prm.score_mode);
          sSc[r] = s0;
          if (LH_CHECK(dbg::in_range(t0 + r, prm.N), kBoundsPyramid)) sc[t0 + r] = s0;
        }
        __syncthreads();
      }
      for (int e = tid; e < n; e += 256) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < p; ++i) m = fmaxf(m, prevS[e * p + i]);
        curS[e] = m;
        if (LH_CHECK(dbg::entry_ok(j0 + e, prm.off[l], prm.off[l + 1]), kBoundsPyramid))
          sc[prm.off[l] + j0 + e] = m;
      }
    }
    __syncthreads();
    nprev = n;
  }
}

// Level l > J from level l-1 in HBM (level 0 being the input): one thread per
// (entry, 8-column chunk, tensor) for the means, one per entry for the score.
template <typename Tin, int D, bool kPyr, bool kScore>
__global__ void __launch_bounds__(256) k_pyr_upper(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    float* __restrict__ pq, float* __restrict__ pk, float* __restrict__ pv,
    float* __restrict__ score, const PyrPrm prm, int l, int64_t u0) {
  pdl_enter();
  constexpr int G = D / 8;
  const int n = prm.N / prm.pw[l];  // entries of level l per unit
  const int it = (int)blockIdx.x * 256 + (int)threadIdx.x;
  const int64_t u = u0 + blockIdx.y;
  if (kPyr && it < 3 * n * G) {
    const int t = it / (n * G);
    const int rem = it - t * n * G;
    const int e = rem / G, c = rem - (rem / G) * G;
    float acc[8], x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int i = 0; i < prm.p; ++i) {
      const int ch = e * prm.p + i;  // child index at level l-1
      if (l == 1) {
        const Tin* src = (t == 0 ? q : t == 1 ? k : v) + (u * prm.N + ch) * D + 8 * c;
        load8(src, x);
      } else {
        const float* src = (t == 0 ? pq : t == 1 ? pk : pv) +
                           (u * (prm.M - prm.N) + prm.off[l - 1] - prm.N + ch) * D + 8 * c;
        load8(src, x);
      }
#pragma unroll
      for (int z = 0; z < 8; ++z) acc[z] = __fadd_rn(acc[z], x[z]);
    }
#pragma unroll
    for (int z = 0; z < 8; ++z) acc[z] = mean_of<0>(acc[z], prm);
    float* dst = (t == 0 ? pq : t == 1 ? pk : pv);
    float* o = dst + (u * (prm.M - prm.N) + prm.off[l] - prm.N + e) * D + 8 * c;
    if (LH_CHECK(dbg::entry_ok(e, prm.off[l], prm.off[l + 1]), kBoundsPyramid)) {
      *reinterpret_cast<float4*>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(o + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
  if (kScore && it < n) {
    float* sc = score + u * prm.M;
    float m = 0.0f;
    for (int i = 0; i < prm.p; ++i) m = fmaxf(m, sc[prm.off[l - 1] + it * prm.p + i]);
    if (LH_CHECK(dbg::entry_ok(it, prm.off[l], prm.off[l + 1]), kBoundsPyramid)) sc[prm.off[l] + it] = m;
  }
}

PyrPrm make_prm(const Geom& g, int cap) {
  PyrPrm prm;
  prm.N = (int32_t)g.N;
  prm.M = (int32_t)g.M;
  prm.p = g.p;
  prm.L = g.L;
  prm.score_mode = g.score_mode;
  prm.pow2 = (g.p & (g.p - 1)) == 0;
  prm.inv_p = 1.0f / (float)g.p;  // exact when p is a power of two
  prm.inv_pd = 1.0 / (double)g.p;
  for (int l = 0; l <= kMaxLevels; ++l) {
    prm.off[l] = (int32_t)g.off[l];
    prm.pw[l] = (int32_t)(g.pw[l] > 0x7fffffff ? 0x7fffffff : g.pw[l]);
  }
  int J = 0;
  while (J + 1 <= g.L - 1 && g.pw[J + 1] <= cap) ++J;
  prm.J = J;
  prm.CR = (int32_t)(g.pw[J] * (cap / g.pw[J]));
  return prm;
}

template <typename Tin, int D, int P, bool kPyr, bool kScore>
cudaError_t launch_flags(const Geom& g, const Tin* q, const Tin* k, const Tin* v, float* pq,
                         float* pk, float* pv, float* score, cudaStream_t st) {
  const PyrPrm prm = make_prm(g, chunk_rows_cap(D, sizeof(Tin)));
  const size_t smem = ChunkSmem<Tin, D, kPyr>::bytes(prm.CR, prm.p);
  auto* kc = k_pyr_chunk<Tin, D, P, kPyr, kScore>;
  cudaError_t e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned bx = (unsigned)((g.N + prm.CR - 1) / prm.CR);
  for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
    const unsigned nu = (unsigned)(g.U - u0 < 65535 ? g.U - u0 : 65535);
    (void)launch_pdl(kc, dim3(bx, nu), 256, smem, st, q, k, v, pq, pk, pv, score, prm, u0);
    for (int l = prm.J + 1; l <= g.L - 1; ++l) {
      const int64_t n = g.N / g.pw[l];
      const int64_t items = kPyr ? 3 * n * (D / 8) : n;
      const unsigned ub = (unsigned)((items + 255) / 256);
      (void)launch_pdl(k_pyr_upper<Tin, D, kPyr, kScore>, dim3(ub, nu), 256, 0, st, q, k, v, pq, pk, pv, score,
                                                                      prm, l, u0);
    }
  }
  return cudaGetLastError();
}

template <typename Tin, int D>
cudaError_t launch_t(const Geom& g, const void* q, const void* k, const void* v, float* pq,
                     float* pk, float* pv, float* score, cudaStream_t st) {
  const Tin* tq = static_cast<const Tin*>(q);
  const Tin* tk = static_cast<const Tin*>(k);
  const Tin* tv = static_cast<const Tin*>(v);
  auto go = [&](auto pc) {
    constexpr int P = decltype(pc)::value;
    if (pq && score) return launch_flags<Tin, D, P, true, true>(g, tq, tk, tv, pq, pk, pv, score, st);
    if (pq) return launch_flags<Tin, D, P, true, false>(g, tq, tk, tv, pq, pk, pv, score, st);
    return launch_flags<Tin, D, P, false, true>(g, tq, tk, tv, pq, pk, pv, score, st);
  };
  if (g.p == 4) return go(std::integral_constant<int, 4>{});
  if (g.p == 2) return go(std::integral_constant<int, 2>{});
  return go(std::integral_constant<int, 0>{});
}

}  // namespace

int pyramid_launches(const Geom& g, lh_dtype dt) {
  const PyrPrm prm = make_prm(g, chunk_rows_cap(g.d, dt == LH_BF16 ? 2 : 4));
  const int64_t chunks = (g.U + 65534) / 65535;
  return (int)(chunks * (1 + (g.L - 1 - prm.J)));
}

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
