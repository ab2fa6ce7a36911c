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

__device__ __forceinline__ void rows_bar() {  // the 8 row-work warps only
  asm volatile("bar.sync 1, 256;\n" ::: "memory");
}

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
struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[3], kv_empty[3];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2], mma_done;  // [column half]
  uint32_t tmem;
  int abort;
  float xm[2][128], xl[2][128];  // [half][row] final max and sum
};

template <int D>
struct FwdLayout {
  static constexpr int kKS = (D == 64) ? 3 : 2;  // K/V stages
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kKS * kTile;
  static constexpr int kP = kV + kKS * kTile;  // 128 x 128 fp16
  static constexpr int kBar = kP + 32768;
  static constexpr int kBytes = kBar + (int)sizeof(FwdBars);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, __half* __restrict__ os,
                  float* __restrict__ lse, int S, int unit0, int nunits, float scale_log2,
                  int ntiles) {
  using Lt = FwdLayout<D>;
  constexpr int KS = Lt::kKS;
  static_assert(KS >= 2 && KS <= 3, "FwdBars holds at most 3 stages; the protocol needs 2");
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_status(kStatusAttnFwdTimeout | 1u);
    return;
  }
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + Lt::kBar);
  uint8_t* sQ = smem + Lt::kQ;
  uint8_t* sK = smem + Lt::kK;
  uint8_t* sV = smem + Lt::kV;
  uint8_t* sP = smem + Lt::kP;
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
      mbar_init(&bars->s_free[b], 8);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars->p_full[h], 4);
      mbar_init(&bars->pv_done[h], 1);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 9) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  // O_h (h = key half of every tile) accumulates at tmem + 256 + h * D
  const uint32_t tO = tmem + 256;

  if (warp == 8) {
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
  } else if (warp == 9) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idPV = idesc_f16(128, D, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      // O_h += P[:, keys of half h] V[keys of half h, :], once the row work
      // of half h has stored its P
      auto issue_pv = [&](int i) {
        const int st = i % KS;
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(&bars->p_full[h], i & 1, abort, kStatus)) return false;
          tc_fence_after();
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = h * 4 + k4;
            umma_f16(tO + h * D, desc_kmajor(aP + h * 16384 + k4 * 32),
                     desc_mnmajor(aV + st * Lt::kTile + kk * 2048, 16384), idPV, (i > 0 || k4 > 0));
          }
          umma_commit(&bars->pv_done[h]);
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
    // ------------------------------------------- row work: two threads per row
    // Thread (row r, half h) owns the 64 keys of half h in every tile and the
    // partial softmax over them: its own running reference max m_ref, sum l
    // and accumulator O_h in TMEM.  No exchange is needed until the end, where
    // the two partials of a row are combined (the usual split-softmax merge).
    // P is formed against m_ref, and O_h is rescaled in TMEM only when a tile's
    // max exceeds m_ref by more than kRescale (exp2 domain), so P <= 2^kRescale
    // fits fp16; softmax is invariant to the reference, so the result is the same.
    constexpr float kRescale = 8.0f;
    const int qd = warp & 3, h = warp >> 2;
    const int r = qd * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    const uint32_t tOh = tO + h * D + lane_addr;
    float m_ref = -INFINITY, l = 0.0f;
    bool ok = true;
    // one key tile; kDiag: the last (diagonal) tile, keys past the row masked
    auto step = [&](int j, auto diag_tag) {
      constexpr bool kDiag = decltype(diag_tag)::value;
      const int b = j & 1;
      ok = warp_wait(&bars->s_full[b], (j >> 1) & 1, abort, kStatus);
      if (!ok) return;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld64(tmem + b * 128 + lane_addr + h * 64, v0, v1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free[b]);  // S is in registers now
      const int lim = r - h * 64;                     // keys i <= lim are visible
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (kDiag) {
          mx = max3(mx, i <= lim ? __uint_as_float(v0[i]) : -INFINITY,
                    i + 32 <= lim ? __uint_as_float(v1[i]) : -INFINITY);
        } else {
          mx = max3(mx, __uint_as_float(v0[i]), __uint_as_float(v1[i]));
        }
      }
      mx *= scale_log2;
      const bool grow = mx > m_ref + kRescale;
      const float m_new = grow ? mx : m_ref;
      if (j > 0) {
        // P_h of the previous tile must be consumed before this one is stored,
        // and O_h must be complete before it is rescaled
        ok = warp_wait(&bars->pv_done[h], (j - 1) & 1, abort, kStatus);
        if (!ok) return;
        if (__any_sync(0xffffffffu, grow)) {
          tc_fence_after();
          const float alpha = ex2(m_ref - m_new);  // 1 for rows that do not grow
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tOh + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(tOh + c * 32, ov);
          }
          tmem_st_wait();
          l *= alpha;
        }
      }
      m_ref = m_new;
      // a fully masked half (only in the diagonal tile) has m_ref = -inf: its
      // exponent is NaN but every one of its elements is replaced by 0 below
      uint32_t pk[32];
      const float2 cc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_ref, -m_ref);
      float2 sa = make_float2(0.0f, 0.0f), sb = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 x = ffma2(make_float2(__uint_as_float(v0[i]), __uint_as_float(v0[i + 1])), cc, nm);
        const float2 y = ffma2(make_float2(__uint_as_float(v1[i]), __uint_as_float(v1[i + 1])), cc, nm);
        float2 p = make_float2(ex2(x.x), ex2(x.y));
        float2 q = make_float2(ex2(y.x), ex2(y.y));
        if (kDiag) {
          p.x = i <= lim ? p.x : 0.0f;
          p.y = i + 1 <= lim ? p.y : 0.0f;
          q.x = i + 32 <= lim ? q.x : 0.0f;
          q.y = i + 33 <= lim ? q.y : 0.0f;
        }
        sa = fadd2(sa, p);
        sb = fadd2(sb, q);
        pk[i >> 1] = h2(p.x, p.y);
        pk[16 + (i >> 1)] = h2(q.x, q.y);
      }
      store_row_half(sP + h * 16384, r, pk);
      tc_fence_before();  // orders the O_h rescale (TMEM stores) before the next product
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[h]);
      l += (sa.x + sa.y) + (sb.x + sb.y);
    };
    for (int j = 0; j < n - 1 && ok; ++j) step(j, std::false_type{});
    if (ok) step(n - 1, std::true_type{});
    if (ok) ok = warp_wait(&bars->pv_done[h], (n - 1) & 1, abort, kStatus);
    // merge the two halves of each row: O = sum_h 2^(m_h - m) O_h / sum_h 2^(m_h - m) l_h
    bars->xm[h][r] = m_ref;
    bars->xl[h][r] = l;
    rows_bar();
    const float m0 = bars->xm[0][r], m1 = bars->xm[1][r];
    const float m = fmaxf(m0, m1);  // finite: key 0 of half 0 is visible to every row
    const float w0 = ex2(m0 - m), w1 = ex2(m1 - m);
    const float lt = w0 * bars->xl[0][r] + w1 * bars->xl[1][r];
    const int row = qt * 128 + r;
    if (ok) {  // whole warps load TMEM; only rows inside the sequence are stored
      tc_fence_after();
      constexpr int DH = D / 2;  // output columns of this thread
      const float inv = 1.0f / lt;
      const float2 c0 = make_float2(w0 * inv, w0 * inv), c1 = make_float2(w1 * inv, w1 * inv);
      __half* dst = os + ((int64_t)u * S + row) * D + h * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o0[32], o1[32];
        tmem_ld32(tO + lane_addr + h * DH + c * 32, o0);
        tmem_ld32(tO + D + lane_addr + h * DH + c * 32, o1);
        tmem_ld_wait();
        if (row < S) {
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            uint32_t w[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const int e = 8 * x + 2 * y;
              const float2 f = ffma2(make_float2(__uint_as_float(o1[e]), __uint_as_float(o1[e + 1])), c1,
                                     fmul2(make_float2(__uint_as_float(o0[e]), __uint_as_float(o0[e + 1])), c0));
              w[y] = h2_sat(f.x, f.y);
            }
            *reinterpret_cast<uint4*>(dst + c * 32 + 8 * x) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (h == 0 && row < S) lse[(int64_t)u * S + row] = (m + __log2f(lt)) * kLn2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ========================================================= backward: dK, dV
// One CTA per (unit, 128-key tile kt), walking the query tiles i >= kt:
// S^T = K Q_i^T and dP^T = V dO_i^T in TMEM; two threads per key row form
// P^T = 2^(S^T c - lse2) (zero where the query precedes the key) and
// dS^T = P^T (dP^T - D) in fp16 shared memory; dV += P^T dO_i and dK += dS^T Q_i
// accumulate in TMEM over all query tiles (fixed order, no atomics).
struct DkvBars {
  uint64_t kv_full;
  uint64_t q_full[3], q_empty[3];  // [stage], at most 3 stages
  uint64_t s_full, st_free, p_full, pdone, mma_done;
  uint32_t tmem;
  int abort;
};

template <int D>
struct DkvLayout {
  static constexpr int kStages = (D == 64) ? 3 : 1;  // DkvBars holds up to 3
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;
  static constexpr int kDO = kQ + kStages * kTile;
  static constexpr int kPT = kDO + kStages * kTile;
  static constexpr int kDST = kPT + 32768;
  static constexpr int kStat = kDST + 32768;  // per stage: -lse2[128], -D[128]
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
  static_assert(STG >= 1 && STG <= 3, "DkvBars holds at most 3 stages");
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
          umma_f16(tDV, desc_kmajor(aPT + a), desc_mnmajor(aDO + b, 16384), idAcc, (t > 0 || kk > 0));
          umma_f16(tDK, desc_kmajor(aDST + a), desc_mnmajor(aQ + b, 16384), idAcc, (t > 0 || kk > 0));
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
      store_row_half(sPT + h * 16384, r, pp);
      store_row_half(sDST + h * 16384, r, pd);
      fence_async_smem();
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
// dS = P (dP - D) in fp16 shared memory (double-buffered); dQ += dS K_j in TMEM.
struct DqBars {
  uint64_t q_full;
  uint64_t kv_full[3], kv_empty[3];  // [stage], at most 3 stages
  uint64_t s_full, s_free, mma_done;
  uint64_t ds_full[2], dsdone[2];
  uint32_t tmem;
  int abort;
};

template <int D>
struct DqLayout {
  static constexpr int kStages = (D == 64) ? 3 : 1;  // DqBars holds up to 3
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTile;
  static constexpr int kK = kDO + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kDS = kV + kStages * kTile;  // 2 buffers of 128 x 128 fp16
  static constexpr int kBar = kDS + 2 * 32768;
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
  static_assert(STG >= 1 && STG <= 3, "DqBars holds at most 3 stages");
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
  uint8_t* sDS = smem + Lt::kDS;
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
      const uint32_t aDS = smem_u32(sDS);
      auto issue_dq = [&](int j) {  // dQ += dS_j K_j
        const int st = j % STG, b = j & 1;
        if (!mbar_wait(&bars->ds_full[b], (j >> 1) & 1, abort, kStatus)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = aDS + b * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16(tDQ, desc_kmajor(a), desc_mnmajor(aK + st * Lt::kTile + kk * 2048, 16384), idAcc,
                   (j > 0 || kk > 0));
        }
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
      store_row_half(sDS + b * 32768 + h * 16384, r, pd);
      fence_async_smem();
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
    k_attn_fwd_tc<D><<<(unsigned)(nu * ntiles), kThreads, smem, st>>>(
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
