// k_attn_mma.cu -- causal attention on the gathered sub-sequence with
// warp-level mma.sync (m16n8k16 fp16, fp32 accumulate).
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.C: stock causal attention on the dense
// sub-sequence; §2.B: its backward is the only path from the layer output back
// to the selected Q, K and V.
//
// This is the legacy-tensor-core implementation, kept as the comparison
// baseline for the tcgen05/TMEM kernels (k_attn_tc.cu) and selectable at run
// time.  Tiles: 64 query rows x 64 keys per step, 4 warps (16 rows each),
// online softmax in the exp2 domain, double-buffered cp.async tiles.
// Backward: a key-block pass (dK, dV) and a query-block pass (dQ), so every
// output element is accumulated by one thread in a fixed order: deterministic,
// no atomics.  Rows at or past S are zero-filled on load and never stored.
#include "lh_internal.cuh"

namespace lh {

// Status word of the mma.sync attention kernels (bounds checks of the debug build).
__device__ uint32_t g_mma_status = 0;
#define LH_STATUS_WORD g_mma_status

cudaError_t mma_status_read_clear(uint32_t* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_mma_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_mma_status, &zero, sizeof(zero));
}

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes: the 16 destination bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
               "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A * B + D; A 16x16 (4 regs), B 16x8 (2 regs), D 16x8 fp32 (4 regs).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
struct Tile {
  static constexpr int kStride = D + 8;  // halfs; +16 B keeps ldmatrix rows on distinct banks
};

// Copy rows [r0, r0+R) of a [S, D] fp16 matrix into smem (row stride D+8),
// zero-filling rows >= S.  All 128 threads participate.
template <int D, int R>
__device__ __forceinline__ void load_tile(__half* sm, const __half* g, int64_t r0,
                                          int64_t S) {
  constexpr int kChunks = R * D / 8;
#pragma unroll
  for (int i = threadIdx.x; i < kChunks; i += 128) {
    const int r = i / (D / 8), c = i % (D / 8);
    const bool ok = (r0 + r) < S;
    const __half* src = ok ? g + (r0 + r) * D + 8 * c : g;
    cp_async16(sm + r * Tile<D>::kStride + 8 * c, src, ok);
  }
}

// A-operand fragment (16 rows x 16 cols at (row0, col0)) of a row-major smem tile.
template <int D>
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const __half* sm, int row0,
                                       int col0) {
  const int l = threadIdx.x & 31;
  ldsm_x4(a, smem_u32(sm + (row0 + (l & 15)) * Tile<D>::kStride + col0 + (l >> 4) * 8));
}
// B fragments for two n-tiles where B[k][n] = T[n][k] (T row-major in smem):
// b[0],b[1] for n-tile n0, b[2],b[3] for n-tile n0+8; k in [k0, k0+16).
template <int D>
__device__ __forceinline__ void frag_b_nt(uint32_t (&b)[4], const __half* sm, int n0,
                                          int k0) {
  const int l = threadIdx.x & 31;
  ldsm_x4(b, smem_u32(sm + (n0 + (l & 7) + (l >> 4) * 8) * Tile<D>::kStride + k0 +
                      ((l >> 3) & 1) * 8));
}
// B fragments for two n-tiles where B[k][n] = T[k][n] (T row-major in smem).
template <int D>
__device__ __forceinline__ void frag_b_t(uint32_t (&b)[4], const __half* sm, int k0,
                                         int n0) {
  const int l = threadIdx.x & 31;
  ldsm_x4_t(b, smem_u32(sm + (k0 + (l & 7) + ((l >> 3) & 1) * 8) * Tile<D>::kStride + n0 +
                        (l >> 4) * 8));
}

// =================================================================== forward
template <int D>
__global__ void __launch_bounds__(128) k_attn_fwd_mma(const __half* __restrict__ qs,
                                                      const __half* __restrict__ ks,
                                                      const __half* __restrict__ vs,
                                                      __half* __restrict__ os,
                                                      float* __restrict__ lse, int64_t S,
                                                      float scale_log2, int ntiles) {
  constexpr int BM = 64, BN = 64, ST = Tile<D>::kStride;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __half* sQ = reinterpret_cast<__half*>(smem_raw);
  __half* sK = sQ + BM * ST;      // 2 stages
  __half* sV = sK + 2 * BN * ST;  // 2 stages

  // heaviest (last) query tiles first
  const int qt = ntiles - 1 - blockIdx.x;
  const int64_t u = blockIdx.y;
  if (!LH_CHECK(dbg::in_range((int64_t)qt * BM, S), kBoundsAttnFwd)) return;  // whole CTA
  const __half* Qg = qs + u * S * D;
  const __half* Kg = ks + u * S * D;
  const __half* Vg = vs + u * S * D;
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t q0 = (int64_t)qt * BM;

  load_tile<D, BM>(sQ, Qg, q0, S);
  load_tile<D, BN>(sK, Kg, 0, S);
  load_tile<D, BN>(sV, Vg, 0, S);
  cp_async_commit();

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.0f, 0.0f};
  uint32_t qf[D / 16][4];

  const int nkv = qt + 1;  // causal: key tiles 0..qt
  for (int j = 0; j < nkv; ++j) {
    const int stage = j & 1;
    if (j + 1 < nkv) {
      load_tile<D, BN>(sK + (stage ^ 1) * BN * ST, Kg, (int64_t)(j + 1) * BN, S);
      load_tile<D, BN>(sV + (stage ^ 1) * BN * ST, Vg, (int64_t)(j + 1) * BN, S);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) frag_a<D>(qf[kk], sQ, warp * 16, kk * 16);
    }
    const __half* cK = sK + stage * BN * ST;
    const __half* cV = sV + stage * BN * ST;
    float s[BN / 8][4];
#pragma unroll
    for (int i = 0; i < BN / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < BN / 8; nt += 2) {
        uint32_t b[4];
        frag_b_nt<D>(b, cK, nt * 8, kk * 16);
        mma16816(s[nt], qf[kk], b[0], b[1]);
        mma16816(s[nt + 1], qf[kk], b[2], b[3]);
      }
    }
    // scale into the log2 domain, causal mask on the diagonal tile
    const int64_t row_a = q0 + warp * 16 + (l >> 2), row_b = row_a + 8;
    float mx[2] = {m[0], m[1]};
#pragma unroll
    for (int nt = 0; nt < BN / 8; ++nt) {
      const int64_t col = (int64_t)j * BN + nt * 8 + 2 * (l & 3);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t r = (e < 2) ? row_a : row_b;
        const int64_t cc = col + (e & 1);
        float v = s[nt][e] * scale_log2;
        if (j == qt && cc > r) v = -INFINITY;
        s[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    }
    float alpha[2], rs[2] = {0.0f, 0.0f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      alpha[h] = exp2f(m[h] - mx[h]);  // m = -inf on the first tile gives 0
      m[h] = mx[h];
    }
    uint32_t pf[BN / 16][4];
#pragma unroll
    for (int nt = 0; nt < BN / 8; ++nt) {
      const float p0 = exp2f(s[nt][0] - m[0]), p1 = exp2f(s[nt][1] - m[0]);
      const float p2 = exp2f(s[nt][2] - m[1]), p3 = exp2f(s[nt][3] - m[1]);
      rs[0] += p0 + p1;
      rs[1] += p2 + p3;
      pf[nt >> 1][(nt & 1) * 2 + 0] = pack_h2(p0, p1);
      pf[nt >> 1][(nt & 1) * 2 + 1] = pack_h2(p2, p3);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) lsum[h] = lsum[h] * alpha[h] + rs[h];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < D / 8; nt += 2) {
        uint32_t b[4];
        frag_b_t<D>(b, cV, kk * 16, nt * 8);
        mma16816(o[nt], pf[kk], b[0], b[1]);
        mma16816(o[nt + 1], pf[kk], b[2], b[3]);
      }
    }
    __syncthreads();  // this stage is overwritten by the next prefetch
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], 1);
    lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], 2);
  }
  const int64_t row_a = q0 + warp * 16 + (l >> 2), row_b = row_a + 8;
  const float inv_a = 1.0f / lsum[0], inv_b = 1.0f / lsum[1];
  __half* Og = os + u * S * D;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int col = nt * 8 + 2 * (l & 3);
    if (row_a < S)
      *reinterpret_cast<uint32_t*>(Og + row_a * D + col) = pack_h2(o[nt][0] * inv_a, o[nt][1] * inv_a);
    if (row_b < S)
      *reinterpret_cast<uint32_t*>(Og + row_b * D + col) = pack_h2(o[nt][2] * inv_b, o[nt][3] * inv_b);
  }
  if ((l & 3) == 0) {
    if (row_a < S) lse[u * S + row_a] = (m[0] + log2f(lsum[0])) * kLn2;
    if (row_b < S) lse[u * S + row_b] = (m[1] + log2f(lsum[1])) * kLn2;
  }
}

// ============================================================ backward: dK, dV
// One CTA per 64-key block; loops over query blocks i >= key block.
// S^T = K Q^T, P^T = exp2(S^T c - lse2), dP^T = V dO^T, dS^T = P^T (dP^T - D),
// dV += P^T dO, dK += dS^T Q.
template <int D>
__global__ void __launch_bounds__(128) k_attn_bwd_dkdv_mma(
    const __half* __restrict__ qs, const __half* __restrict__ ks,
    const __half* __restrict__ vs, const __half* __restrict__ dos,
    const float* __restrict__ stats, float* __restrict__ dks,
    float* __restrict__ dvs, int64_t S, float scale, float scale_log2, int ntiles) {
  constexpr int BK = 64, BQ = 64, ST = Tile<D>::kStride;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __half* sK = reinterpret_cast<__half*>(smem_raw);
  __half* sV = sK + BK * ST;
  __half* sQ = sV + BK * ST;      // 2 stages
  __half* sdO = sQ + 2 * BQ * ST;  // 2 stages
  float* sL = reinterpret_cast<float*>(sdO + 2 * BQ * ST);  // 2 stages x BQ lse2
  float* sD = sL + 2 * BQ;                                   // 2 stages x BQ

  const int kt = ntiles - 1 - blockIdx.x;  // short loops last
  const int64_t u = blockIdx.y;
  if (!LH_CHECK(dbg::in_range((int64_t)kt * BK, S), kBoundsAttnBwd)) return;  // whole CTA
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t k0 = (int64_t)kt * BK;
  const __half* Qg = qs + u * S * D;
  const __half* dOg = dos + u * S * D;
  // tile-padded statistics of this unit: -lse2 and -D per 128-row tile
  const float* Stu = stats + u * ((S + 127) / 128) * 256;

  auto load_q = [&](int i, int stage) {
    load_tile<D, BQ>(sQ + stage * BQ * ST, Qg, (int64_t)i * BQ, S);
    load_tile<D, BQ>(sdO + stage * BQ * ST, dOg, (int64_t)i * BQ, S);
    if (threadIdx.x < BQ) {
      const int64_t r = (int64_t)i * BQ + threadIdx.x;
      // padded rows read lse2 = +inf (P = 0) and D = 0
      sL[stage * BQ + threadIdx.x] = -Stu[(r >> 7) * 256 + (r & 127)];
      sD[stage * BQ + threadIdx.x] = -Stu[(r >> 7) * 256 + 128 + (r & 127)];
    }
  };
  load_tile<D, BK>(sK, ks + u * S * D, k0, S);
  load_tile<D, BK>(sV, vs + u * S * D, k0, S);
  load_q(kt, 0);
  cp_async_commit();

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.0f;

  for (int i = kt; i < ntiles; ++i) {
    const int stage = (i - kt) & 1;
    if (i + 1 < ntiles) load_q(i + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const __half* cQ = sQ + stage * BQ * ST;
    const __half* cdO = sdO + stage * BQ * ST;
    const float* cL = sL + stage * BQ;
    const float* cD = sD + stage * BQ;
    float st[BQ / 8][4], dpt[BQ / 8][4];
#pragma unroll
    for (int n = 0; n < BQ / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];
      frag_a<D>(ka, sK, warp * 16, kk * 16);
      frag_a<D>(va, sV, warp * 16, kk * 16);
#pragma unroll
      for (int nt = 0; nt < BQ / 8; nt += 2) {
        uint32_t b[4];
        frag_b_nt<D>(b, cQ, nt * 8, kk * 16);
        mma16816(st[nt], ka, b[0], b[1]);
        mma16816(st[nt + 1], ka, b[2], b[3]);
        frag_b_nt<D>(b, cdO, nt * 8, kk * 16);
        mma16816(dpt[nt], va, b[0], b[1]);
        mma16816(dpt[nt + 1], va, b[2], b[3]);
      }
    }
    // rows of S^T are keys (kr), columns are queries (qc)
    const int64_t kr_a = k0 + warp * 16 + (l >> 2), kr_b = kr_a + 8;
    uint32_t pa[BQ / 16][4], dsa[BQ / 16][4];
#pragma unroll
    for (int nt = 0; nt < BQ / 8; ++nt) {
      const int qc_l = nt * 8 + 2 * (l & 3);
      float p[4], ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = qc_l + (e & 1);
        const int64_t qc = (int64_t)i * BQ + qi;
        const int64_t kr = (e < 2) ? kr_a : kr_b;
        float pv = exp2f(st[nt][e] * scale_log2 - cL[qi]);
        if (qc < kr) pv = 0.0f;
        p[e] = pv;
        ds[e] = pv * (dpt[nt][e] - cD[qi]);
      }
      pa[nt >> 1][(nt & 1) * 2 + 0] = pack_h2(p[0], p[1]);
      pa[nt >> 1][(nt & 1) * 2 + 1] = pack_h2(p[2], p[3]);
      dsa[nt >> 1][(nt & 1) * 2 + 0] = pack_h2(ds[0], ds[1]);
      dsa[nt >> 1][(nt & 1) * 2 + 1] = pack_h2(ds[2], ds[3]);
    }
#pragma unroll
    for (int kk = 0; kk < BQ / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < D / 8; nt += 2) {
        uint32_t b[4];
        frag_b_t<D>(b, cdO, kk * 16, nt * 8);
        mma16816(dv[nt], pa[kk], b[0], b[1]);
        mma16816(dv[nt + 1], pa[kk], b[2], b[3]);
        frag_b_t<D>(b, cQ, kk * 16, nt * 8);
        mma16816(dk[nt], dsa[kk], b[0], b[1]);
        mma16816(dk[nt + 1], dsa[kk], b[2], b[3]);
      }
    }
    __syncthreads();
  }
  const int64_t kr_a = k0 + warp * 16 + (l >> 2), kr_b = kr_a + 8;
  float* dKg = dks + u * S * D;
  float* dVg = dvs + u * S * D;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int col = nt * 8 + 2 * (l & 3);
    if (kr_a < S) {
      *reinterpret_cast<float2*>(dKg + kr_a * D + col) = make_float2(dk[nt][0] * scale, dk[nt][1] * scale);
      *reinterpret_cast<float2*>(dVg + kr_a * D + col) = make_float2(dv[nt][0], dv[nt][1]);
    }
    if (kr_b < S) {
      *reinterpret_cast<float2*>(dKg + kr_b * D + col) = make_float2(dk[nt][2] * scale, dk[nt][3] * scale);
      *reinterpret_cast<float2*>(dVg + kr_b * D + col) = make_float2(dv[nt][2], dv[nt][3]);
    }
  }
}

// ================================================================ backward: dQ
// One CTA per 64-query block; loops over key blocks j <= query block.
template <int D>
__global__ void __launch_bounds__(128) k_attn_bwd_dq_mma(
    const __half* __restrict__ qs, const __half* __restrict__ ks,
    const __half* __restrict__ vs, const __half* __restrict__ dos,
    const float* __restrict__ stats, float* __restrict__ dqs,
    int64_t S, float scale, float scale_log2, int ntiles) {
  constexpr int BM = 64, BN = 64, ST = Tile<D>::kStride;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __half* sQ = reinterpret_cast<__half*>(smem_raw);
  __half* sdO = sQ + BM * ST;
  __half* sK = sdO + BM * ST;     // 2 stages
  __half* sV = sK + 2 * BN * ST;  // 2 stages

  const int qt = ntiles - 1 - blockIdx.x;
  const int64_t u = blockIdx.y;
  if (!LH_CHECK(dbg::in_range((int64_t)qt * BM, S), kBoundsAttnBwd)) return;  // whole CTA
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t q0 = (int64_t)qt * BM;
  const __half* Kg = ks + u * S * D;
  const __half* Vg = vs + u * S * D;
  load_tile<D, BM>(sQ, qs + u * S * D, q0, S);
  load_tile<D, BM>(sdO, dos + u * S * D, q0, S);
  load_tile<D, BN>(sK, Kg, 0, S);
  load_tile<D, BN>(sV, Vg, 0, S);
  cp_async_commit();

  const int64_t row_a = q0 + warp * 16 + (l >> 2), row_b = row_a + 8;
  const float* Stu = stats + u * ((S + 127) / 128) * 256;
  const float l2a = -Stu[(row_a >> 7) * 256 + (row_a & 127)];
  const float l2b = -Stu[(row_b >> 7) * 256 + (row_b & 127)];
  const float Da = -Stu[(row_a >> 7) * 256 + 128 + (row_a & 127)];
  const float Db = -Stu[(row_b >> 7) * 256 + 128 + (row_b & 127)];

  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.0f;

  const int nkv = qt + 1;
  for (int j = 0; j < nkv; ++j) {
    const int stage = j & 1;
    if (j + 1 < nkv) {
      load_tile<D, BN>(sK + (stage ^ 1) * BN * ST, Kg, (int64_t)(j + 1) * BN, S);
      load_tile<D, BN>(sV + (stage ^ 1) * BN * ST, Vg, (int64_t)(j + 1) * BN, S);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const __half* cK = sK + stage * BN * ST;
    const __half* cV = sV + stage * BN * ST;
    float s[BN / 8][4], dp[BN / 8][4];
#pragma unroll
    for (int n = 0; n < BN / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t qa[4], ga[4];
      frag_a<D>(qa, sQ, warp * 16, kk * 16);
      frag_a<D>(ga, sdO, warp * 16, kk * 16);
#pragma unroll
      for (int nt = 0; nt < BN / 8; nt += 2) {
        uint32_t b[4];
        frag_b_nt<D>(b, cK, nt * 8, kk * 16);
        mma16816(s[nt], qa, b[0], b[1]);
        mma16816(s[nt + 1], qa, b[2], b[3]);
        frag_b_nt<D>(b, cV, nt * 8, kk * 16);
        mma16816(dp[nt], ga, b[0], b[1]);
        mma16816(dp[nt + 1], ga, b[2], b[3]);
      }
    }
    uint32_t dsa[BN / 16][4];
#pragma unroll
    for (int nt = 0; nt < BN / 8; ++nt) {
      const int64_t col = (int64_t)j * BN + nt * 8 + 2 * (l & 3);
      float ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t r = (e < 2) ? row_a : row_b;
        const int64_t cc = col + (e & 1);
        float pv = exp2f(s[nt][e] * scale_log2 - ((e < 2) ? l2a : l2b));
        if (cc > r) pv = 0.0f;
        ds[e] = pv * (dp[nt][e] - ((e < 2) ? Da : Db));
      }
      dsa[nt >> 1][(nt & 1) * 2 + 0] = pack_h2(ds[0], ds[1]);
      dsa[nt >> 1][(nt & 1) * 2 + 1] = pack_h2(ds[2], ds[3]);
    }
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < D / 8; nt += 2) {
        uint32_t b[4];
        frag_b_t<D>(b, cK, kk * 16, nt * 8);
        mma16816(dq[nt], dsa[kk], b[0], b[1]);
        mma16816(dq[nt + 1], dsa[kk], b[2], b[3]);
      }
    }
    __syncthreads();
  }
  float* dQg = dqs + u * S * D;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int col = nt * 8 + 2 * (l & 3);
    if (row_a < S)
      *reinterpret_cast<float2*>(dQg + row_a * D + col) = make_float2(dq[nt][0] * scale, dq[nt][1] * scale);
    if (row_b < S)
      *reinterpret_cast<float2*>(dQg + row_b * D + col) = make_float2(dq[nt][2] * scale, dq[nt][3] * scale);
  }
}

template <int D>
constexpr size_t fwd_smem() {
  return (size_t)(64 + 4 * 64) * Tile<D>::kStride * 2;
}
template <int D>
constexpr size_t dkdv_smem() {
  return (size_t)(2 * 64 + 4 * 64) * Tile<D>::kStride * 2 + 4 * 64 * 4;
}
template <int D>
constexpr size_t dq_smem() {
  return (size_t)(2 * 64 + 4 * 64) * Tile<D>::kStride * 2;
}

template <int D>
cudaError_t fwd_d(const Geom& g, const __half* qs, const __half* ks,
                  const __half* vs, float scale, __half* os, float* lse,
                  cudaStream_t st) {
  const int ntiles = (int)((g.S + 63) / 64);
  cudaError_t e = cudaFuncSetAttribute(k_attn_fwd_mma<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwd_smem<D>());
  if (e != cudaSuccess) return e;
  for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
    const int64_t nu = g.U - u0 < 65535 ? g.U - u0 : 65535;
    k_attn_fwd_mma<D><<<dim3(ntiles, (unsigned)nu), 128, fwd_smem<D>(), st>>>(
        qs + u0 * g.S * D, ks + u0 * g.S * D, vs + u0 * g.S * D, os + u0 * g.S * D,
        lse + u0 * g.S, g.S, scale * kLog2e, ntiles);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t bwd_d(const Geom& g, const __half* qs, const __half* ks,
                  const __half* vs, const __half* dos, const float* stats, float scale,
                  float* dqs, float* dks, float* dvs, cudaStream_t st) {
  const int ntiles = (int)((g.S + 63) / 64);
  const int64_t T = (g.S + 127) / 128;  // 128-row tiles of the statistics
  cudaError_t e = cudaFuncSetAttribute(k_attn_bwd_dkdv_mma<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)dkdv_smem<D>());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attn_bwd_dq_mma<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dq_smem<D>());
  if (e != cudaSuccess) return e;
  for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
    const int64_t nu = g.U - u0 < 65535 ? g.U - u0 : 65535;
    const int64_t o = u0 * g.S * D;
    k_attn_bwd_dkdv_mma<D><<<dim3(ntiles, (unsigned)nu), 128, dkdv_smem<D>(), st>>>(
        qs + o, ks + o, vs + o, dos + o, stats + u0 * T * 256, dks + o, dvs + o, g.S, scale,
        scale * kLog2e, ntiles);
    k_attn_bwd_dq_mma<D><<<dim3(ntiles, (unsigned)nu), 128, dq_smem<D>(), st>>>(
        qs + o, ks + o, vs + o, dos + o, stats + u0 * T * 256, dqs + o, g.S, scale,
        scale * kLog2e, ntiles);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_mma(const Geom& g, const __half* qs, const __half* ks,
                                const __half* vs, float scale, __half* os,
                                float* lse, cudaStream_t st) {
  return g.d == 64 ? fwd_d<64>(g, qs, ks, vs, scale, os, lse, st)
                   : fwd_d<128>(g, qs, ks, vs, scale, os, lse, st);
}

cudaError_t launch_attn_bwd_mma(const Geom& g, const __half* qs, const __half* ks,
                                const __half* vs, const __half* dos, const float* stats,
                                float scale, float* dqs, float* dks, float* dvs, cudaStream_t st) {
  return g.d == 64 ? bwd_d<64>(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, st)
                   : bwd_d<128>(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, st);
}

}  // namespace lh
