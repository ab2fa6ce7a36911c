// k_attn_tc.cu -- causal attention on the gathered sub-sequence with the
// 5th-generation tensor cores (tcgen05 MMA, accumulators in TMEM, operands
// staged by TMA in 128-byte-swizzled shared memory).
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.C: stock causal attention on the dense
// sub-sequence (row k sees k' <= k), scale 1/sqrt(d); §2.B: its backward is the
// only path from the layer output back to the selected Q, K and V.
//
// All three kernels use one CTA per SM (512 TMEM columns) and 10 warps:
//   warps 0-7  the row work: two threads per row of the 128-row tile (TMEM lane
//              = row; warp w reads lanes 32*(w%4).. and one half of the columns,
//              w/4), so 8 warps share the exponentials and the fp16 packing;
//   warp 8     TMA producer (one lane issues; in the dK/dV kernel all 32 lanes
//              also stage the per-query softmax statistics);
//   warp 9     MMA issuer (one lane) and owner of the TMEM allocation.
// Score tiles are read from TMEM into registers in one go and the buffer is
// released at once, so the next tile's products run while the row work goes on.
// Every mbarrier wait is bounded (two seconds); on expiry a status bit is set,
// the roles drain, loads and MMAs in flight are waited for, TMEM is freed.
// Rows past S are zero-filled by TMA (3-D tensor maps) and never stored; the
// TMEM loads, being warp-collective, are always executed by whole warps.
#include <type_traits>

#include "tc_common.cuh"

namespace lh {

cudaError_t device_status_read_clear(uint32_t* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
}

namespace tc {
namespace {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;

// Two tcgen05.ld of 32 columns each, then one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&a)[32], uint32_t (&b)[32]) {
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld_wait();
}

__device__ __forceinline__ void store_row_half(uint8_t* tile_half, int r, const uint32_t (&pk)[32]) {
  // one 64-column half of a row of a 128-byte-swizzled fp16 tile: 8 chunks of 16 B
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(tile_half + swz(r, c)) =
        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// ================================================================= forward
// Column groups: every 128-key tile is split into NG groups of CW = 128/NG
// keys; the 4 warps of group g (one per TMEM lane quarter) own the keys of
// group g in every tile, with their own running reference max, sum and TMEM
// accumulator O_g (D columns).  NG = 2: eight row-work warps, two per SM
// sub-partition (four groups, 16 warps, measured slower at d = 64: the
// per-thread register cap of 18 warps and four P handoffs per tile).
template <int D>
struct FwdCfg {
  static constexpr int NG = 2;
  static constexpr int CW = 128 / NG;        // keys per group and tile
  static constexpr int kRowWarps = 4 * NG;
  static constexpr int kTmaWarp = kRowWarps, kMmaWarp = kRowWarps + 1;
  static constexpr int kThreads = 32 * (kRowWarps + 2);
  static constexpr int OC = D / NG;          // output columns per thread
  static_assert(256 + NG * D <= (int)kTmemCols, "TMEM: two S buffers and NG accumulators");
  static_assert(CW % 64 == 0, "P of a group is stored as whole 32-column TMEM stores");
};

template <int NG>
struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[4], kv_empty[4];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[NG], pv_done[NG], mma_done;  // [column group]
  uint32_t tmem;
  int abort;
  float xm[NG][128], xl[NG][128];  // [group][row] final reference max and sum
};

template <int D>
struct FwdLayout {
  static constexpr int kKS = (D == 64) ? 4 : 2;  // K/V stages
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kKS * kTile;
  static constexpr int kBar = kV + kKS * kTile;  // (P lives in TMEM, over S)
  static constexpr int kBytes = kBar + (int)sizeof(FwdBars<FwdCfg<D>::NG>);
};

template <int NT>
__device__ __forceinline__ void named_bar() {  // the NT row-work threads only
  asm volatile("bar.sync 1, %0;\n" ::"n"(NT) : "memory");
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::kThreads, 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, __half* __restrict__ os,
                  float* __restrict__ lse, int S, int unit0, int nunits, float scale_log2,
                  int ntiles) {
  using Lt = FwdLayout<D>;
  using Cf = FwdCfg<D>;
  constexpr int NG = Cf::NG, CW = Cf::CW;
  constexpr int KS = Lt::kKS;
  static_assert(KS >= 2 && KS <= 4, "FwdBars holds at most 4 stages; the protocol needs 2");
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_status(kStatusAttnFwdTimeout | 1u);
    return;
  }
  auto* bars = reinterpret_cast<FwdBars<NG>*>(smem + Lt::kBar);
  uint8_t* sQ = smem + Lt::kQ;
  uint8_t* sK = smem + Lt::kK;
  uint8_t* sV = smem + Lt::kV;
  volatile int* abort = &bars->abort;
  constexpr uint32_t kStatus = kStatusAttnFwdTimeout;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 1-D grid ordered by work: all units' last (longest) query tiles first
  const int qt = ntiles - 1 - (int)(blockIdx.x / nunits);
  const int u = unit0 + (int)(blockIdx.x % nunits);
  const int n = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], Cf::kRowWarps);
    }
    for (int g = 0; g < NG; ++g) {
      mbar_init(&bars->p_full[g], 4);
      mbar_init(&bars->pv_done[g], 1);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == Cf::kMmaWarp) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  // S double buffer at tmem + 0 / + 128 (P_g of a tile is written over the first
  // CW/2 of its group's S columns); O_g at tmem + 256 + g * D
  const uint32_t tO = tmem + 256;

  if (warp == Cf::kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bars->q_full, Lt::kTile);
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(sQ + h * 16384, &tq, &bars->q_full, h * 64, qt * 128, u);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % KS;
        if (j >= KS && !mbar_wait(&bars->kv_empty[st], ((j - KS) / KS) & 1, abort, kStatus)) break;
        mbar_expect_tx(&bars->kv_full[st], 2 * Lt::kTile);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sK + st * Lt::kTile + h * 16384, &tk, &bars->kv_full[st], h * 64, j * 128, u);
          tma_load_3d(sV + st * Lt::kTile + h * 16384, &tv, &bars->kv_full[st], h * 64, j * 128, u);
        }
        issued = j + 1;
      }
      mbar_wait(&bars->q_full, 0, abort, kStatus, false);
      for (int j = (issued > KS ? issued - KS : 0); j < issued; ++j)
        mbar_wait(&bars->kv_full[j % KS], (j / KS) & 1, abort, kStatus, false);
    }
  } else if (warp == Cf::kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idPV = idesc_f16(128, D, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      // O_g += P[:, keys of group g] V[keys of group g, :], once group g has
      // written its P (TMEM, over S of tile i) -- issued before S of tile i + 2
      // overwrites that buffer
      auto issue_pv = [&](int i) {
        const int st = i % KS;
        const uint32_t tP = tmem + (i & 1) * 128;
        for (int g = 0; g < NG; ++g) {
          if (!mbar_wait(&bars->p_full[g], i & 1, abort, kStatus)) return false;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < CW / 16; ++k) {
            const int kk = g * (CW / 16) + k;  // 16-key step within the tile
            umma_f16_ta(tO + g * D, tP + g * CW + 8 * k,
                        desc_mnmajor(aV + st * Lt::kTile + kk * 2048, 16384), idPV, (i > 0 || k > 0));
          }
          umma_commit(&bars->pv_done[g]);
        }
        umma_commit(&bars->kv_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, kStatus);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % KS, b = j & 1;
        ok = mbar_wait(&bars->kv_full[st], (j / KS) & 1, abort, kStatus) &&
             (j < 2 || mbar_wait(&bars->s_free[b], ((j - 2) >> 1) & 1, abort, kStatus));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16(tmem + b * 128, desc_kmajor(aQ + off), desc_kmajor(aK + st * Lt::kTile + off),
                   idS, kk > 0);
        }
        umma_commit(&bars->s_full[b]);
        if (j >= 1 && !(ok = issue_pv(j - 1))) break;
      }
      if (ok) issue_pv(n - 1);
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, abort, kStatus, false);
    }
  } else {
    // ------------------------------------ row work: NG threads per row (one per group)
    // Thread (row r, group g) owns the CW keys of group g in every tile and the
    // partial softmax over them: its own running reference max m_ref, sum l and
    // accumulator O_g in TMEM.  Nothing is exchanged until the end, where the NG
    // partials of a row are merged (the usual split-softmax merge).  P is formed
    // against m_ref, and O_g is rescaled in TMEM only when a tile's max exceeds
    // m_ref by more than kRescale (exp2 domain), so P <= 2^kRescale fits fp16;
    // softmax is invariant to the reference, so the result is the same.
    constexpr float kRescale = 8.0f;
    const int qd = warp & 3, g = warp >> 2;
    const int r = qd * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    const uint32_t tOg = tO + g * D + lane_addr;
    float m_ref = -INFINITY, l = 0.0f;
    bool ok = true;
    // one key tile; kDiag: the last (diagonal) tile, keys past the row masked
    auto step = [&](int j, auto diag_tag) {
      constexpr bool kDiag = decltype(diag_tag)::value;
      const int b = j & 1;
      ok = warp_wait(&bars->s_full[b], (j >> 1) & 1, abort, kStatus);
      if (!ok) return;
      tc_fence_after();
      uint32_t v[CW];
#pragma unroll
      for (int c = 0; c < CW / 32; ++c)
        tmem_ld32(tmem + b * 128 + lane_addr + g * CW + 32 * c,
                  reinterpret_cast<uint32_t(&)[32]>(v[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free[b]);  // S is in registers now
      const int lim = r - g * CW;                     // keys i <= lim are visible
      // row max: four independent chains (max is exact in any order)
      float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < CW; i += 2) {
        const int c = (i >> 1) & 3;
        if (kDiag) {
          mc[c] = max3(mc[c], i <= lim ? __uint_as_float(v[i]) : -INFINITY,
                       i + 1 <= lim ? __uint_as_float(v[i + 1]) : -INFINITY);
        } else {
          mc[c] = max3(mc[c], __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
        }
      }
      float mx = fmaxf(max3(mc[0], mc[1], mc[2]), mc[3]);
      mx *= scale_log2;
      const bool grow = mx > m_ref + kRescale;
      const float m_new = grow ? mx : m_ref;
      // P first (against the new reference), so S is dead before O is touched;
      // a fully masked group (only in the diagonal tile) has m_new = -inf: its
      // exponent is NaN but every one of its elements is replaced by 0 below
      uint32_t pk[CW / 2];
      const float2 cc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_new, -m_new);
      // row sum: four independent paired accumulators
      float2 sacc[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                        make_float2(0.0f, 0.0f)};
#pragma unroll
      for (int i = 0; i < CW; i += 4) {
        const float2 x = ffma2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), cc, nm);
        const float2 y = ffma2(make_float2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])), cc, nm);
        float2 p = make_float2(ex2(x.x), ex2(x.y));
        // a quarter of the exponentials on the FMA pipe, the rest on MUFU
        float2 q = (i & 7) == 4 ? ex2_fma2(y) : make_float2(ex2(y.x), ex2(y.y));
        if (kDiag) {
          p.x = i <= lim ? p.x : 0.0f;
          p.y = i + 1 <= lim ? p.y : 0.0f;
          q.x = i + 2 <= lim ? q.x : 0.0f;
          q.y = i + 3 <= lim ? q.y : 0.0f;
        }
        const int c = (i >> 2) & 1;
        sacc[2 * c] = fadd2(sacc[2 * c], p);
        sacc[2 * c + 1] = fadd2(sacc[2 * c + 1], q);
        pk[i >> 1] = h2(p.x, p.y);
        pk[(i >> 1) + 1] = h2(q.x, q.y);
      }
      // every phase of pv_done[g] is waited for, in order (a parity wait must
      // never run two phases ahead of the barrier); the previous tile's product
      // is normally complete by now.  O_g must be complete before a rescale.
      if (j > 0) {
        ok = warp_wait(&bars->pv_done[g], (j - 1) & 1, abort, kStatus);
        if (!ok) return;
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        tc_fence_after();
        const float alpha = ex2(m_ref - m_new);  // 1 for rows that do not grow
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tOg + c * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(tOg + c * 32, ov);
        }
        l *= alpha;
      }
      m_ref = m_new;
      // P (CW keys = CW/2 packed columns) over this group's S columns of buffer b
#pragma unroll
      for (int c = 0; c < CW / 64; ++c)
        tmem_st32(tmem + b * 128 + lane_addr + g * CW + 32 * c,
                  reinterpret_cast<const uint32_t(&)[32]>(pk[32 * c]));
      tmem_st_wait();
      tc_fence_before();  // orders P and the O_g rescale (TMEM stores) before the product
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[g]);
      const float2 s01 = fadd2(sacc[0], sacc[1]), s23 = fadd2(sacc[2], sacc[3]);
      l += (s01.x + s01.y) + (s23.x + s23.y);
    };
    for (int j = 0; j < n - 1 && ok; ++j) step(j, std::false_type{});
    if (ok) step(n - 1, std::true_type{});
    if (ok) ok = warp_wait(&bars->pv_done[g], (n - 1) & 1, abort, kStatus);
    // merge the NG partials of each row:
    //   O = sum_q 2^(m_q - m) O_q / sum_q 2^(m_q - m) l_q,  m = max_q m_q
    bars->xm[g][r] = m_ref;
    bars->xl[g][r] = l;
    named_bar<32 * Cf::kRowWarps>();
    float m = bars->xm[0][r];  // finite: key 0 of group 0 is visible to every row
#pragma unroll
    for (int q = 1; q < NG; ++q) m = fmaxf(m, bars->xm[q][r]);
    float wq[NG];
    float lt = 0.0f;
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      wq[q] = ex2(bars->xm[q][r] - m);
      lt = __fmaf_rn(wq[q], bars->xl[q][r], lt);
    }
    const int row = qt * 128 + r;
    if (ok) {  // whole warps load TMEM; only rows inside the sequence are stored
      tc_fence_after();
      constexpr int OC = Cf::OC;  // output columns of this thread: [g*OC, (g+1)*OC)
      const float inv = 1.0f / lt;
#pragma unroll
      for (int q = 0; q < NG; ++q) wq[q] *= inv;
      __half* dst = os + ((int64_t)u * S + row) * D + g * OC;
#pragma unroll
      for (int c = 0; c < OC / 16; ++c) {
        float f[16];
#pragma unroll
        for (int q = 0; q < NG; ++q) {
          uint32_t ov[16];
          tmem_ld16(tO + q * D + lane_addr + g * OC + 16 * c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            f[i] = q == 0 ? __uint_as_float(ov[i]) * wq[0] : __fmaf_rn(__uint_as_float(ov[i]), wq[q], f[i]);
        }
        if (row < S) {
          uint4 w0, w1;
          w0.x = h2_sat(f[0], f[1]);   w0.y = h2_sat(f[2], f[3]);
          w0.z = h2_sat(f[4], f[5]);   w0.w = h2_sat(f[6], f[7]);
          w1.x = h2_sat(f[8], f[9]);   w1.y = h2_sat(f[10], f[11]);
          w1.z = h2_sat(f[12], f[13]); w1.w = h2_sat(f[14], f[15]);
          *reinterpret_cast<uint4*>(dst + 16 * c) = w0;
          *reinterpret_cast<uint4*>(dst + 16 * c + 8) = w1;
        }
      }
      if (g == 0 && row < S) lse[(int64_t)u * S + row] = (m + __log2f(lt)) * kLn2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cf::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ========================================================= backward: dK, dV
// One CTA per (unit, 128-key tile kt), walking the query tiles i >= kt:
// S^T = K Q_i^T and dP^T = V dO_i^T in TMEM; two threads per key row form
// P^T = 2^(S^T c - lse2) (zero where the query precedes the key) and
// dS^T = P^T (dP^T - D) in fp16 -- in TMEM at d = 64 (columns 384..511, read
// as the A operand), in shared memory at d = 128 (TMEM full); dV += P^T dO_i and
// dK += dS^T Q_i accumulate in TMEM over all query tiles (fixed order, no atomics).
struct DkvBars {
  uint64_t kv_full;
  uint64_t q_full[4], q_empty[4];  // [stage], at most 4 stages
  uint64_t s_full, st_free, p_full, pdone, mma_done;
  uint32_t tmem;
  int abort;
};

template <int D>
struct DkvLayout {
  static constexpr bool kTmemP = (D == 64);  // P^T, dS^T in TMEM (else shared memory)
  static constexpr int kStages = (D == 64) ? 4 : 1;  // DkvBars holds up to 4
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;
  static constexpr int kDO = kQ + kStages * kTile;
  static constexpr int kPT = kDO + kStages * kTile;
  static constexpr int kDST = kPT + (kTmemP ? 0 : 32768);
  static constexpr int kStat = kDST + (kTmemP ? 0 : 32768);  // per stage: -lse2[128], -D[128]
  static constexpr int kBar = kStat + kStages * 1024;
  static constexpr int kBytes = kBar + (int)sizeof(DkvBars);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const float* __restrict__ stats, float* __restrict__ dks,
                       float* __restrict__ dvs, int S, int unit0,
                       int nunits, float scale, float scale_log2, int ntiles) {
  using Lt = DkvLayout<D>;
  constexpr int STG = Lt::kStages;
  static_assert(STG >= 1 && STG <= 4, "DkvBars holds at most 4 stages");
  constexpr bool kTmemP = Lt::kTmemP;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_status(kStatusAttnBwdTimeout | 1u);
    return;
  }
  DkvBars* bars = reinterpret_cast<DkvBars*>(smem + Lt::kBar);
  uint8_t* sK = smem + Lt::kK;
  uint8_t* sV = smem + Lt::kV;
  uint8_t* sQ = smem + Lt::kQ;
  uint8_t* sDO = smem + Lt::kDO;
  uint8_t* sPT = smem + Lt::kPT;
  uint8_t* sDST = smem + Lt::kDST;
  float* sStat = reinterpret_cast<float*>(smem + Lt::kStat);
  volatile int* abort = &bars->abort;
  constexpr uint32_t kStatus = kStatusAttnBwdTimeout;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 1-D grid ordered by work: key tile 0 (the most query tiles) of every unit first
  const int kt = (int)(blockIdx.x / nunits);
  const int u = unit0 + (int)(blockIdx.x % nunits);
  const int n = ntiles - kt;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < STG; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->st_free, 8);
    mbar_init(&bars->p_full, 8);
    mbar_init(&bars->pdone, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 9) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tST = tmem, tDPT = tmem + 128, tDV = tmem + 256, tDK = tmem + 256 + D;
  const uint32_t tPT = tmem + 384, tDST = tmem + 448;  // P^T, dS^T packed fp16 (kTmemP)

  if (warp == 8) {
    // TMA producer: K, V once; per query tile Q, dO and the tile's statistics
    if (lane == 0) {
      mbar_expect_tx(&bars->kv_full, 2 * Lt::kTile);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sK + h * 16384, &tk, &bars->kv_full, h * 64, kt * 128, u);
        tma_load_3d(sV + h * 16384, &tv, &bars->kv_full, h * 64, kt * 128, u);
      }
      int issued = 0;
      for (int t = 0; t < n; ++t) {
        const int st = t % STG, i = kt + t;
        if (t >= STG && !mbar_wait(&bars->q_empty[st], ((t - STG) / STG) & 1, abort, kStatus)) break;
        mbar_expect_tx(&bars->q_full[st], 2 * Lt::kTile + 1024);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sQ + st * Lt::kTile + h * 16384, &tq, &bars->q_full[st], h * 64, i * 128, u);
          tma_load_3d(sDO + st * Lt::kTile + h * 16384, &tdo, &bars->q_full[st], h * 64, i * 128, u);
        }
        bulk_load(sStat + st * 256, stats + ((int64_t)u * ntiles + i) * 256, 1024, &bars->q_full[st]);
        issued = t + 1;
      }
      mbar_wait(&bars->kv_full, 0, abort, kStatus, false);
      for (int t = (issued > STG ? issued - STG : 0); t < issued; ++t)
        mbar_wait(&bars->q_full[t % STG], (t / STG) & 1, abort, kStatus, false);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idAcc = idesc_f16(128, D, true);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      const uint32_t aPT = smem_u32(sPT), aDST = smem_u32(sDST);
      auto issue_grads = [&](int t) {  // dV += P^T dO_t, dK += dS^T Q_t
        const int st = t % STG;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t b = st * Lt::kTile + kk * 2048;
          if constexpr (kTmemP) {
            umma_f16_ta(tDV, tPT + 8 * kk, desc_mnmajor(aDO + b, 16384), idAcc, (t > 0 || kk > 0));
            umma_f16_ta(tDK, tDST + 8 * kk, desc_mnmajor(aQ + b, 16384), idAcc, (t > 0 || kk > 0));
          } else {
            umma_f16(tDV, desc_kmajor(aPT + a), desc_mnmajor(aDO + b, 16384), idAcc, (t > 0 || kk > 0));
            umma_f16(tDK, desc_kmajor(aDST + a), desc_mnmajor(aQ + b, 16384), idAcc, (t > 0 || kk > 0));
          }
        }
        umma_commit(&bars->pdone);
        umma_commit(&bars->q_empty[st]);
      };
      bool ok = mbar_wait(&bars->kv_full, 0, abort, kStatus);
      for (int t = 0; ok && t < n; ++t) {
        const int st = t % STG;
        if (STG == 1 && t > 0) {  // one stage: free it before the next tile is loaded
          ok = mbar_wait(&bars->p_full, (t - 1) & 1, abort, kStatus);
          if (!ok) break;
          tc_fence_after();
          issue_grads(t - 1);
        }
        ok = mbar_wait(&bars->q_full[st], (t / STG) & 1, abort, kStatus) &&
             (t == 0 || mbar_wait(&bars->st_free, (t - 1) & 1, abort, kStatus));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16(tST, desc_kmajor(aK + off), desc_kmajor(aQ + st * Lt::kTile + off), idS, kk > 0);
          umma_f16(tDPT, desc_kmajor(aV + off), desc_kmajor(aDO + st * Lt::kTile + off), idS, kk > 0);
        }
        umma_commit(&bars->s_full);
        if (STG > 1 && t > 0) {
          ok = mbar_wait(&bars->p_full, (t - 1) & 1, abort, kStatus);
          if (!ok) break;
          tc_fence_after();
          issue_grads(t - 1);
        }
      }
      if (ok && mbar_wait(&bars->p_full, (n - 1) & 1, abort, kStatus)) {
        tc_fence_after();
        issue_grads(n - 1);
      }
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, abort, kStatus, false);
    }
  } else {
    // --------------------------------------- row work: two threads per key row
    const int qd = warp & 3, h = warp >> 2;
    const int r = qd * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    bool ok = true;
    // one query tile; kDiag: the first (diagonal) tile, queries before the key masked
    auto step = [&](int t, auto diag_tag) {
      constexpr bool kDiag = decltype(diag_tag)::value;
      const int st = t % STG;
      ok = warp_wait(&bars->q_full[st], (t / STG) & 1, abort, kStatus) &&
           warp_wait(&bars->s_full, t & 1, abort, kStatus);
      if (!ok) return;
      tc_fence_after();
      uint32_t a0[32], a1[32], b0[32], b1[32];
      tmem_ld32(tST + lane_addr + h * 64, a0);
      tmem_ld32(tST + lane_addr + h * 64 + 32, a1);
      tmem_ld32(tDPT + lane_addr + h * 64, b0);
      tmem_ld32(tDPT + lane_addr + h * 64 + 32, b1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->st_free);  // S^T, dP^T are in registers now
      const float4* cl = reinterpret_cast<const float4*>(sStat + st * 256 + h * 64);        // -lse2
      const float4* cd = reinterpret_cast<const float4*>(sStat + st * 256 + 128 + h * 64);  // -D
      const int lim = r - h * 64;  // query columns e < lim precede the key
      const float2 cc = make_float2(scale_log2, scale_log2);
      uint32_t pp[32], pd[32];
      auto quad = [&](int e, const uint32_t* sv, const uint32_t* gv) {
        const float4 nl = cl[e >> 2], nd = cd[e >> 2];
        const int k = e & 31;
        const float2 x0 = ffma2(make_float2(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])), cc,
                                make_float2(nl.x, nl.y));
        const float2 x1 = ffma2(make_float2(__uint_as_float(sv[k + 2]), __uint_as_float(sv[k + 3])), cc,
                                make_float2(nl.z, nl.w));
        float2 p0 = make_float2(ex2(x0.x), ex2(x0.y)), p1 = make_float2(ex2(x1.x), ex2(x1.y));
        if (kDiag) {
          p0.x = e < lim ? 0.0f : p0.x;
          p0.y = e + 1 < lim ? 0.0f : p0.y;
          p1.x = e + 2 < lim ? 0.0f : p1.x;
          p1.y = e + 3 < lim ? 0.0f : p1.y;
        }
        const float2 d0 = fmul2(p0, fadd2(make_float2(__uint_as_float(gv[k]), __uint_as_float(gv[k + 1])),
                                          make_float2(nd.x, nd.y)));
        const float2 d1 = fmul2(p1, fadd2(make_float2(__uint_as_float(gv[k + 2]), __uint_as_float(gv[k + 3])),
                                          make_float2(nd.z, nd.w)));
        pp[e >> 1] = h2(p0.x, p0.y);
        pp[(e >> 1) + 1] = h2(p1.x, p1.y);
        pd[e >> 1] = h2_sat(d0.x, d0.y);
        pd[(e >> 1) + 1] = h2_sat(d1.x, d1.y);
      };
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        quad(e, a0, b0);
        quad(e + 32, a1, b1);
      }
      if (t > 0 && !(ok = warp_wait(&bars->pdone, (t - 1) & 1, abort, kStatus))) return;
      if constexpr (kTmemP) {  // this row's 64 query columns = 32 packed columns
        tmem_st32(tPT + lane_addr + h * 32, pp);
        tmem_st32(tDST + lane_addr + h * 32, pd);
        tmem_st_wait();
        tc_fence_before();
      } else {
        store_row_half(sPT + h * 16384, r, pp);
        store_row_half(sDST + h * 16384, r, pd);
        fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    };
    step(0, std::true_type{});
    for (int t = 1; t < n && ok; ++t) step(t, std::false_type{});
    if (ok) ok = warp_wait(&bars->pdone, (n - 1) & 1, abort, kStatus);
    const int row = kt * 128 + r;
    if (ok) {
      tc_fence_after();
      const bool in = row < S;
      constexpr int DH = D / 2;
      float* gv = dvs + ((int64_t)u * S + row) * D + h * DH;
      float* gk = dks + ((int64_t)u * S + row) * D + h * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tDV + lane_addr + h * DH + c * 32, v);
        tmem_ld_wait();
        if (in) {
#pragma unroll
          for (int x = 0; x < 8; ++x)
            *reinterpret_cast<float4*>(gv + c * 32 + 4 * x) =
                make_float4(__uint_as_float(v[4 * x]), __uint_as_float(v[4 * x + 1]),
                            __uint_as_float(v[4 * x + 2]), __uint_as_float(v[4 * x + 3]));
        }
        tmem_ld32(tDK + lane_addr + h * DH + c * 32, v);
        tmem_ld_wait();
        if (in) {
#pragma unroll
          for (int x = 0; x < 8; ++x)
            *reinterpret_cast<float4*>(gk + c * 32 + 4 * x) =
                make_float4(__uint_as_float(v[4 * x]) * scale, __uint_as_float(v[4 * x + 1]) * scale,
                            __uint_as_float(v[4 * x + 2]) * scale, __uint_as_float(v[4 * x + 3]) * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================= backward: dQ
// One CTA per (unit, 128-query tile qt), walking the key tiles j <= qt:
// S = Q K_j^T, dP = dO V_j^T in TMEM; two threads per query row form
// dS = P (dP - D) in fp16, double-buffered in TMEM (read as the A operand);
// dQ += dS K_j in TMEM.
struct DqBars {
  uint64_t q_full;
  uint64_t kv_full[4], kv_empty[4];  // [stage], at most 4 stages
  uint64_t s_full, s_free, mma_done;
  uint64_t ds_full[2], dsdone[2];
  uint32_t tmem;
  int abort;
};

template <int D>
struct DqLayout {
  static constexpr int kStages = (D == 64) ? 4 : 2;  // DqBars holds up to 4
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTile;
  static constexpr int kK = kDO + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;  // (dS lives in TMEM)
  static constexpr int kBytes = kBar + (int)sizeof(DqBars);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                     const float* __restrict__ stats, float* __restrict__ dqs, int S,
                     int unit0, int nunits, float scale,
                     float scale_log2, int ntiles) {
  using Lt = DqLayout<D>;
  constexpr int STG = Lt::kStages;
  static_assert(STG >= 1 && STG <= 4, "DqBars holds at most 4 stages");
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_status(kStatusAttnBwdTimeout | 2u);
    return;
  }
  DqBars* bars = reinterpret_cast<DqBars*>(smem + Lt::kBar);
  uint8_t* sQ = smem + Lt::kQ;
  uint8_t* sDO = smem + Lt::kDO;
  uint8_t* sK = smem + Lt::kK;
  uint8_t* sV = smem + Lt::kV;
  volatile int* abort = &bars->abort;
  constexpr uint32_t kStatus = kStatusAttnBwdTimeout;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = ntiles - 1 - (int)(blockIdx.x / nunits);  // most key tiles first
  const int u = unit0 + (int)(blockIdx.x % nunits);
  const int n = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < STG; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->ds_full[i], 8);
      mbar_init(&bars->dsdone[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 8);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 9) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256;
  const uint32_t tDS = tmem + 256 + D;  // 2 buffers of 64 packed fp16 columns (dS of a tile)

  if (warp == 8) {
    if (lane == 0) {
      mbar_expect_tx(&bars->q_full, 2 * Lt::kTile);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sQ + h * 16384, &tq, &bars->q_full, h * 64, qt * 128, u);
        tma_load_3d(sDO + h * 16384, &tdo, &bars->q_full, h * 64, qt * 128, u);
      }
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % STG;
        if (j >= STG && !mbar_wait(&bars->kv_empty[st], ((j - STG) / STG) & 1, abort, kStatus)) break;
        mbar_expect_tx(&bars->kv_full[st], 2 * Lt::kTile);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sK + st * Lt::kTile + h * 16384, &tk, &bars->kv_full[st], h * 64, j * 128, u);
          tma_load_3d(sV + st * Lt::kTile + h * 16384, &tv, &bars->kv_full[st], h * 64, j * 128, u);
        }
        issued = j + 1;
      }
      mbar_wait(&bars->q_full, 0, abort, kStatus, false);
      for (int j = (issued > STG ? issued - STG : 0); j < issued; ++j)
        mbar_wait(&bars->kv_full[j % STG], (j / STG) & 1, abort, kStatus, false);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idAcc = idesc_f16(128, D, true);
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
      auto issue_dq = [&](int j) {  // dQ += dS_j K_j, dS_j from TMEM
        const int st = j % STG, b = j & 1;
        if (!mbar_wait(&bars->ds_full[b], (j >> 1) & 1, abort, kStatus)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_ta(tDQ, tDS + b * 64 + 8 * kk,
                      desc_mnmajor(aK + st * Lt::kTile + kk * 2048, 16384), idAcc, (j > 0 || kk > 0));
        umma_commit(&bars->dsdone[b]);
        umma_commit(&bars->kv_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, kStatus);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % STG;
        if (STG == 1 && j > 0 && !(ok = issue_dq(j - 1))) break;
        ok = mbar_wait(&bars->kv_full[st], (j / STG) & 1, abort, kStatus) &&
             (j == 0 || mbar_wait(&bars->s_free, (j - 1) & 1, abort, kStatus));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16(tS, desc_kmajor(aQ + off), desc_kmajor(aK + st * Lt::kTile + off), idS, kk > 0);
          umma_f16(tDP, desc_kmajor(aDO + off), desc_kmajor(aV + st * Lt::kTile + off), idS, kk > 0);
        }
        umma_commit(&bars->s_full);
        if (STG > 1 && j > 0 && !(ok = issue_dq(j - 1))) break;
      }
      if (ok) issue_dq(n - 1);
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, abort, kStatus, false);
    }
  } else {
    // ------------------------------------- row work: two threads per query row
    const int qd = warp & 3, h = warp >> 2;
    const int r = qd * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    const int row = qt * 128 + r;
    const bool in = row < S;
    // -lse*log2(e) and -D of this row (padded rows: -inf and 0, so P = 0)
    const float* srow = stats + ((int64_t)u * ntiles + qt) * 256 + r;
    const float nlse2 = __ldg(srow), nD = __ldg(srow + 128);
    bool ok = true;
    // one key tile; kDiag: the last (diagonal) tile, keys past the query masked
    auto step = [&](int j, auto diag_tag) {
      constexpr bool kDiag = decltype(diag_tag)::value;
      ok = warp_wait(&bars->s_full, j & 1, abort, kStatus);
      if (!ok) return;
      tc_fence_after();
      uint32_t a0[32], a1[32], b0[32], b1[32];
      tmem_ld32(tS + lane_addr + h * 64, a0);
      tmem_ld32(tS + lane_addr + h * 64 + 32, a1);
      tmem_ld32(tDP + lane_addr + h * 64, b0);
      tmem_ld32(tDP + lane_addr + h * 64 + 32, b1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);
      const float2 cc = make_float2(scale_log2, scale_log2), nl = make_float2(nlse2, nlse2);
      const float2 nd = make_float2(nD, nD);
      const int lim = r - h * 64;  // key columns e > lim follow the query
      uint32_t pd[32];
      auto pair = [&](int e, uint32_t s0, uint32_t s1, uint32_t g0, uint32_t g1) {
        const float2 x = ffma2(make_float2(__uint_as_float(s0), __uint_as_float(s1)), cc, nl);
        float2 p = make_float2(ex2(x.x), ex2(x.y));
        if (kDiag) {
          p.x = e > lim ? 0.0f : p.x;
          p.y = e + 1 > lim ? 0.0f : p.y;
        }
        const float2 ds = fmul2(p, fadd2(make_float2(__uint_as_float(g0), __uint_as_float(g1)), nd));
        pd[e >> 1] = h2_sat(ds.x, ds.y);
      };
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        pair(e, a0[e], a0[e + 1], b0[e], b0[e + 1]);
        pair(e + 32, a1[e], a1[e + 1], b1[e], b1[e + 1]);
      }
      const int b = j & 1;
      if (j >= 2 && !(ok = warp_wait(&bars->dsdone[b], ((j - 2) >> 1) & 1, abort, kStatus))) return;
      tmem_st32(tDS + b * 64 + lane_addr + h * 32, pd);  // 64 key columns, packed
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full[b]);
    };
    for (int j = 0; j < n - 1 && ok; ++j) step(j, std::false_type{});
    if (ok) step(n - 1, std::true_type{});
    if (ok) ok = warp_wait(&bars->dsdone[(n - 1) & 1], ((n - 1) >> 1) & 1, abort, kStatus);
    if (ok) {
      tc_fence_after();
      constexpr int DH = D / 2;
      float* gq = dqs + ((int64_t)u * S + row) * D + h * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tDQ + lane_addr + h * DH + c * 32, v);
        tmem_ld_wait();
        if (in) {
#pragma unroll
          for (int x = 0; x < 8; ++x)
            *reinterpret_cast<float4*>(gq + c * 32 + 4 * x) =
                make_float4(__uint_as_float(v[4 * x]) * scale, __uint_as_float(v[4 * x + 1]) * scale,
                            __uint_as_float(v[4 * x + 2]) * scale, __uint_as_float(v[4 * x + 3]) * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [U, S, d] fp16 viewed as (x = column, y = row, z = unit); boxes of 64 x 128 x 1,
// 128-byte swizzle; rows past S read as zeros.
bool make_map(CUtensorMap* map, const void* base, int d, int64_t S, int64_t U) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)S, (cuuint64_t)U};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)S * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t fwd_d(const Geom& g, const __half* qs, const __half* ks, const __half* vs,
                  float scale, __half* os, float* lse, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qs, D, g.S, g.U) || !make_map(&mk, ks, D, g.S, g.U) ||
      !make_map(&mv, vs, D, g.S, g.U))
    return cudaErrorNotSupported;
  constexpr int smem = FwdLayout<D>::kBytes;
  cudaError_t e =
      cudaFuncSetAttribute(k_attn_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((g.S + 127) / 128);
  const int64_t per = 0x7fffffff / ntiles;  // units per launch (grid.x limit)
  for (int64_t u0 = 0; u0 < g.U; u0 += per) {
    const int64_t nu = g.U - u0 < per ? g.U - u0 : per;
    k_attn_fwd_tc<D><<<(unsigned)(nu * ntiles), FwdCfg<D>::kThreads, smem, st>>>(
        mq, mk, mv, os, lse, (int)g.S, (int)u0, (int)nu, scale * kLog2e, ntiles);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t bwd_d(const Geom& g, const __half* qs, const __half* ks, const __half* vs,
                  const __half* dos, const float* stats, float scale, float* dqs, float* dks,
                  float* dvs, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, qs, D, g.S, g.U) || !make_map(&mk, ks, D, g.S, g.U) ||
      !make_map(&mv, vs, D, g.S, g.U) || !make_map(&mdo, dos, D, g.S, g.U))
    return cudaErrorNotSupported;
  constexpr int smem_a = DkvLayout<D>::kBytes, smem_b = DqLayout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k_attn_bwd_dkdv_tc<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem_a);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attn_bwd_dq_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_b);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((g.S + 127) / 128);
  const int64_t per = 0x7fffffff / ntiles;
  for (int64_t u0 = 0; u0 < g.U; u0 += per) {
    const int64_t nu = g.U - u0 < per ? g.U - u0 : per;
    k_attn_bwd_dkdv_tc<D><<<(unsigned)(nu * ntiles), kThreads, smem_a, st>>>(
        mq, mk, mv, mdo, stats, dks, dvs, (int)g.S, (int)u0, (int)nu, scale, scale * kLog2e,
        ntiles);
    k_attn_bwd_dq_tc<D><<<(unsigned)(nu * ntiles), kThreads, smem_b, st>>>(
        mq, mk, mv, mdo, stats, dqs, (int)g.S, (int)u0, (int)nu, scale, scale * kLog2e, ntiles);
  }
  return cudaGetLastError();
}

}  // namespace
}  // namespace tc

bool attn_tc_available() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return false;
  return major == 10 && minor == 0 && tc::encode_fn() != nullptr;
}
bool attn_tc_bwd_available() { return attn_tc_available(); }
int attn_tc_fwd_launches(const Geom& g) {
  const int64_t ntiles = (g.S + 127) / 128, per = 0x7fffffff / ntiles;
  return (int)((g.U + per - 1) / per);
}
int attn_tc_bwd_launches(const Geom& g) { return 2 * attn_tc_fwd_launches(g); }

cudaError_t launch_attn_fwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, float scale, __half* os, float* lse,
                               cudaStream_t st) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::fwd_d<64>(g, qs, ks, vs, scale, os, lse, st)
                   : tc::fwd_d<128>(g, qs, ks, vs, scale, os, lse, st);
}

cudaError_t launch_attn_bwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, const __half* dos, const float* stats,
                               float scale, float* dqs, float* dks, float* dvs, cudaStream_t st) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::bwd_d<64>(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, st)
                   : tc::bwd_d<128>(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, st);
}

}  // namespace lh
