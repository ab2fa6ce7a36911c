// k_attn_tc.cu -- causal attention on the gathered sub-sequence with the
// 5th-generation tensor cores (tcgen05 MMA, accumulators in TMEM, operands
// staged by TMA in 128-byte-swizzled shared memory).
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.C: stock causal attention on the dense
// sub-sequence (row k sees k' <= k), scale 1/sqrt(d); §2.B: its backward is the
// only path from the layer output back to the selected Q, K and V.
//
// Forward, one CTA per (unit, 128-query tile), 6 warps:
//   warp 4 (one lane)  TMA producer: Q once, then K/V tiles of 128 keys into a
//                      2-stage ring;
//   warp 5 (one lane)  MMA issuer: S = Q K^T into TMEM (128 columns), then
//                      PV = P V into TMEM (d columns) once P is in shared memory;
//                      warp 5 also owns the TMEM allocation;
//   warps 0-3          one thread per query row (= TMEM lane): row max over S,
//                      P = 2^(s*scale*log2e - m) rounded to fp16 into swizzled
//                      shared memory, running sum, and O kept in registers:
//                      O <- alpha * O + PV each tile (online softmax).
// S for tile j+1 is computed while the softmax threads finish tile j, and P V
// for tile j while they find the max of tile j+1.  Every wait is bounded
// (two seconds); on expiry the kernel records a status code, lets the other
// roles drain, waits for its own TMA loads and MMAs, frees TMEM and returns.
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
constexpr int kFwdThreads = 192;
constexpr uint32_t kTmemCols = 256;

struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full, s_free, p_full, pv_done, mma_done;
  uint32_t tmem;
  int abort;
};

template <int D>
struct FwdLayout {
  static constexpr int kTile = 128 * D * 2;  // one 128-row fp16 tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;      // 2 stages
  static constexpr int kV = kK + 2 * kTile;  // 2 stages
  static constexpr int kP = kV + 2 * kTile;  // 128 x 128 fp16, two 64-column halves
  static constexpr int kBar = kP + 128 * 128 * 2;
  static constexpr int kBytes = kBar + (int)sizeof(FwdBars);
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, (D == 64) ? 2 : 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, __half* __restrict__ os,
                  float* __restrict__ lse, int S, int unit0, float scale_log2, int ntiles) {
  using Lt = FwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) report_status(kStatusAttnFwdTimeout | 1u);
    return;
  }
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + Lt::kBar);
  uint8_t* sQ = smem + Lt::kQ;
  uint8_t* sK = smem + Lt::kK;
  uint8_t* sV = smem + Lt::kV;
  uint8_t* sP = smem + Lt::kP;
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = ntiles - 1 - (int)blockIdx.x;  // longest rows first
  const int u = unit0 + (int)blockIdx.y;
  const int nkv = qt + 1;
  constexpr uint32_t kStatus = kStatusAttnFwdTimeout;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 5) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tS = tmem, tPV = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bars->q_full, Lt::kTile);
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(sQ + h * 16384, &tq, &bars->q_full, h * 64, qt * 128, u);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&bars->kv_empty[st], ((j - 2) >> 1) & 1, abort, kStatus)) break;
        mbar_expect_tx(&bars->kv_full[st], 2 * Lt::kTile);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sK + st * Lt::kTile + h * 16384, &tk, &bars->kv_full[st], h * 64, j * 128, u);
          tma_load_3d(sV + st * Lt::kTile + h * 16384, &tv, &bars->kv_full[st], h * 64, j * 128, u);
        }
        issued = j + 1;
      }
      // every load this thread issued lands before the CTA may exit
      mbar_wait(&bars->q_full, 0, abort, kStatus, false);
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
        mbar_wait(&bars->kv_full[j & 1], (j >> 1) & 1, abort, kStatus, false);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idPV = idesc_f16(128, D, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      auto issue_s = [&](int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16(tS, desc_kmajor(aQ + off), desc_kmajor(aK + st * Lt::kTile + off), idS,
                   kk > 0);
        }
        umma_commit(&bars->s_full);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, kStatus) &&
                mbar_wait(&bars->kv_full[0], 0, abort, kStatus);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv) {
          const int st1 = (j + 1) & 1;
          ok = mbar_wait(&bars->kv_full[st1], ((j + 1) >> 1) & 1, abort, kStatus) &&
               mbar_wait(&bars->s_free, j & 1, abort, kStatus);
          if (!ok) break;
          tc_fence_after();
          issue_s(st1);
        }
        ok = mbar_wait(&bars->p_full, j & 1, abort, kStatus);
        if (!ok) break;
        tc_fence_after();
        const int st = j & 1;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = aP + (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t b = aV + st * Lt::kTile + kk * 2048;
          umma_f16(tPV, desc_kmajor(a), desc_mnmajor(b, 16384), idPV, kk > 0);
        }
        umma_commit(&bars->pv_done);
        umma_commit(&bars->kv_empty[st]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, abort, kStatus, false);
    }
  } else {
    // ------------------------------------------------------- softmax, 1 row/thread
    const int r = threadIdx.x;  // query row in the tile = TMEM lane
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    float o[D];
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] = 0.0f;
    float m = -INFINITY, l = 0.0f, alpha_prev = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = warp_wait(&bars->s_full, j & 1, abort, kStatus);
      if (!ok) break;
      tc_fence_after();
      const bool diag = (j == qt);
      // pass 1: row max of the raw scores
      float mx = -INFINITY;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        tmem_ld32(tS + lane_addr + ch * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = __uint_as_float(v[i]);
          if (!diag || ch * 32 + i <= r) mx = fmaxf(mx, x);
        }
      }
      const float m_new = fmaxf(m, mx * scale_log2);
      const float alpha = ex2(m - m_new);
      // fold P V of the previous tile into O (also frees the P buffer)
      if (j > 0) {
        ok = warp_wait(&bars->pv_done, (j - 1) & 1, abort, kStatus);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < D / 32; ++h) {
          uint32_t v[32];
          tmem_ld32(tPV + lane_addr + h * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[h * 32 + i] = fmaf(o[h * 32 + i], alpha_prev, __uint_as_float(v[i]));
        }
      }
      // pass 2: P = 2^(s * scale_log2 - m_new) -> fp16 -> swizzled shared memory
      float rs = 0.0f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        tmem_ld32(tS + lane_addr + ch * 32, v);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float p0 = ex2(fmaf(__uint_as_float(v[i]), scale_log2, -m_new));
          float p1 = ex2(fmaf(__uint_as_float(v[i + 1]), scale_log2, -m_new));
          if (diag && ch * 32 + i > r) p0 = 0.0f;
          if (diag && ch * 32 + i + 1 > r) p1 = 0.0f;
          rs += p0 + p1;
          pk[i >> 1] = pack_h2(p0, p1);
        }
        uint8_t* base = sP + (ch >> 1) * 16384;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const uint32_t c = (ch & 1) * 4 + qd;
          *reinterpret_cast<uint4*>(base + swz(r, c)) =
              make_uint4(pk[qd * 4], pk[qd * 4 + 1], pk[qd * 4 + 2], pk[qd * 4 + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
      l = fmaf(l, alpha, rs);
      m = m_new;
      alpha_prev = alpha;
    }
    if (ok) ok = warp_wait(&bars->pv_done, (nkv - 1) & 1, abort, kStatus);
    if (ok) {  // whole warps: the TMEM loads below are warp-collective
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < D / 32; ++h) {
        uint32_t v[32];
        tmem_ld32(tPV + lane_addr + h * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[h * 32 + i] = fmaf(o[h * 32 + i], alpha_prev, __uint_as_float(v[i]));
      }
      const int row = qt * 128 + r;
      if (row < S) {
        const float inv = 1.0f / l;
        __half* dst = os + ((int64_t)u * S + row) * D;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 w;
          w.x = pack_h2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
          w.y = pack_h2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
          w.z = pack_h2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
          w.w = pack_h2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
          *reinterpret_cast<uint4*>(dst + 8 * c) = w;
        }
        lse[(int64_t)u * S + row] = (m + __log2f(l)) * kLn2;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ========================================================= backward: dK, dV
// One CTA per (unit, 128-key tile kt); it walks the query tiles i >= kt.
//   warp 4: TMA for K, V once and a ring of (Q_i, dO_i) tiles; its 32 lanes also
//           stage lse_i * log2(e) and D_i of the 128 queries in shared memory;
//   warp 5: MMA issuer: S^T = K Q_i^T and dP^T = V dO_i^T (TMEM, 128 columns
//           each), then dV += P^T dO_i and dK += dS^T Q_i (TMEM, d columns each);
//   warps 0-3: one key row each: P^T = 2^(S^T c - lse2) (zero where the query
//           precedes the key), dS^T = P^T (dP^T - D), both to fp16 in swizzled
//           shared memory as the A operands of the two accumulating products.
// dK and dV never leave TMEM until the last tile: no atomics, fixed order.
struct DkvBars {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, st_free, p_full, pdone, mma_done;
  uint32_t tmem;
  int abort;
};

template <int D>
struct DkvLayout {
  static constexpr int kStages = (D == 64) ? 2 : 1;
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;                 // kStages
  static constexpr int kDO = kQ + kStages * kTile;      // kStages
  static constexpr int kPT = kDO + kStages * kTile;     // 128 x 128 fp16
  static constexpr int kDST = kPT + 32768;              // 128 x 128 fp16
  static constexpr int kLse = kDST + 32768;             // kStages x 128 fp32
  static constexpr int kDv = kLse + kStages * 512;      // kStages x 128 fp32
  static constexpr int kBar = kDv + kStages * 512;
  static constexpr int kBytes = kBar + (int)sizeof(DkvBars);
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    k_attn_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const float* __restrict__ lse, const float* __restrict__ Dv,
                       float* __restrict__ dks, float* __restrict__ dvs, int S, int unit0,
                       float scale, float scale_log2, int ntiles) {
  using Lt = DkvLayout<D>;
  constexpr int STG = Lt::kStages;
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
  float* sLse = reinterpret_cast<float*>(smem + Lt::kLse);
  float* sDv = reinterpret_cast<float*>(smem + Lt::kDv);
  volatile int* abort = &bars->abort;
  constexpr uint32_t kStatus = kStatusAttnBwdTimeout;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = (int)blockIdx.x;  // kt = 0 has the most query tiles: it starts first
  const int u = unit0 + (int)blockIdx.y;
  const int n = ntiles - kt;       // query tiles kt .. ntiles-1

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 33);
      mbar_init(&bars->q_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->st_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pdone, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 5) tmem_alloc(&bars->tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tST = tmem, tDPT = tmem + 128, tDV = tmem + 256, tDK = tmem + 256 + D;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(&bars->kv_full, 2 * Lt::kTile);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sK + h * 16384, &tk, &bars->kv_full, h * 64, kt * 128, u);
        tma_load_3d(sV + h * 16384, &tv, &bars->kv_full, h * 64, kt * 128, u);
      }
    }
    int issued = 0;
    for (int t = 0; t < n; ++t) {
      const int st = t % STG, i = kt + t;
      if (t >= STG && !warp_wait(&bars->q_empty[st], ((t - STG) / STG) & 1, abort, kStatus)) break;
      if (lane == 0) {
        mbar_expect_tx(&bars->q_full[st], 2 * Lt::kTile);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sQ + st * Lt::kTile + h * 16384, &tq, &bars->q_full[st], h * 64, i * 128, u);
          tma_load_3d(sDO + st * Lt::kTile + h * 16384, &tdo, &bars->q_full[st], h * 64, i * 128, u);
        }
      }
      for (int c = lane; c < 128; c += 32) {
        const int q = i * 128 + c;
        const bool in = q < S;
        // padded queries: lse2 = +inf makes their P^T (and dS^T) exactly zero
        sLse[st * 128 + c] = in ? __ldg(lse + (int64_t)u * S + q) * kLog2e : INFINITY;
        sDv[st * 128 + c] = in ? __ldg(Dv + (int64_t)u * S + q) : 0.0f;
      }
      mbar_arrive(&bars->q_full[st]);
      issued = t + 1;
    }
    if (lane == 0) {
      mbar_wait(&bars->kv_full, 0, abort, kStatus, false);
      for (int t = (issued > STG ? issued - STG : 0); t < issued; ++t)
        mbar_wait(&bars->q_full[t % STG], (t / STG) & 1, abort, kStatus, false);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
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
        // with one (Q, dO) stage the previous tile's products must finish before
        // the producer can bring the next tile into it
        if (STG == 1 && t > 0) {
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
    // ------------------------------------------------------- one key row per thread
    const int r = threadIdx.x;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      const int st = t % STG;
      ok = warp_wait(&bars->q_full[st], (t / STG) & 1, abort, kStatus) &&
           warp_wait(&bars->s_full, t & 1, abort, kStatus);
      if (!ok) break;
      tc_fence_after();
      const bool diag = (t == 0);
      const float* cl = sLse + st * 128;
      const float* cd = sDv + st * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t a[32], b[32];
        tmem_ld32(tST + lane_addr + ch * 32, a);
        tmem_ld32(tDPT + lane_addr + ch * 32, b);
        tmem_ld_wait();
        if (ch == 3) {  // S^T and dP^T of this tile are in registers: TMEM may be overwritten
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->st_free);
        }
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int q = ch * 32 + e;
          const float2 l2 = *reinterpret_cast<const float2*>(cl + q);
          const float2 dd = *reinterpret_cast<const float2*>(cd + q);
          float p0 = ex2(fmaf(__uint_as_float(a[e]), scale_log2, -l2.x));
          float p1 = ex2(fmaf(__uint_as_float(a[e + 1]), scale_log2, -l2.y));
          if (diag && q < r) p0 = 0.0f;
          if (diag && q + 1 < r) p1 = 0.0f;
          const float d0 = p0 * (__uint_as_float(b[e]) - dd.x);
          const float d1 = p1 * (__uint_as_float(b[e + 1]) - dd.y);
          pp[e >> 1] = pack_h2(p0, p1);
          pd[e >> 1] = pack_h2_sat(d0, d1);
        }
        // the previous tile's products must be done reading the P^T / dS^T buffers
        if (ch == 0 && t > 0 && !(ok = warp_wait(&bars->pdone, (t - 1) & 1, abort, kStatus))) break;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int c = ch * 4 + qd;  // 16-byte chunk of the 128-column row
          const uint32_t off = (c >> 3) * 16384 + swz(r, c & 7);
          *reinterpret_cast<uint4*>(sPT + off) =
              make_uint4(pp[4 * qd], pp[4 * qd + 1], pp[4 * qd + 2], pp[4 * qd + 3]);
          *reinterpret_cast<uint4*>(sDST + off) =
              make_uint4(pd[4 * qd], pd[4 * qd + 1], pd[4 * qd + 2], pd[4 * qd + 3]);
        }
      }
      if (!ok) break;
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok) ok = warp_wait(&bars->pdone, (n - 1) & 1, abort, kStatus);
    const int row = kt * 128 + r;
    if (ok) {  // whole warps load TMEM; only rows inside the sequence are stored
      tc_fence_after();
      float* gv = dvs + ((int64_t)u * S + row) * D;
      float* gk = dks + ((int64_t)u * S + row) * D;
      const bool in = row < S;
#pragma unroll
      for (int h = 0; h < D / 32; ++h) {
        uint32_t v[32];
        tmem_ld32(tDV + lane_addr + h * 32, v);
        tmem_ld_wait();
        if (in) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(gv + h * 32 + 4 * c) =
                make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                            __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
        }
        tmem_ld32(tDK + lane_addr + h * 32, v);
        tmem_ld_wait();
        if (in) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(gk + h * 32 + 4 * c) =
                make_float4(__uint_as_float(v[4 * c]) * scale, __uint_as_float(v[4 * c + 1]) * scale,
                            __uint_as_float(v[4 * c + 2]) * scale, __uint_as_float(v[4 * c + 3]) * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================= backward: dQ
// One CTA per (unit, 128-query tile qt); it walks the key tiles j <= qt.
//   S = Q K_j^T, dP = dO V_j^T in TMEM; one query row per softmax thread:
//   dS = P (dP - D) to fp16 in shared memory; dQ += dS K_j accumulates in TMEM.
struct DqBars {
  uint64_t q_full;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t s_full, s_free, ds_full, dsdone, mma_done;
  uint32_t tmem;
  int abort;
};

template <int D>
struct DqLayout {
  static constexpr int kStages = (D == 64) ? 2 : 1;
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTile;
  static constexpr int kK = kDO + kTile;             // kStages
  static constexpr int kV = kK + kStages * kTile;    // kStages
  static constexpr int kDS = kV + kStages * kTile;   // 128 x 128 fp16
  static constexpr int kBar = kDS + 32768;
  static constexpr int kBytes = kBar + (int)sizeof(DqBars);
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    k_attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                     const float* __restrict__ lse, const float* __restrict__ Dv,
                     float* __restrict__ dqs, int S, int unit0, float scale, float scale_log2,
                     int ntiles) {
  using Lt = DqLayout<D>;
  constexpr int STG = Lt::kStages;
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
  const int qt = ntiles - 1 - (int)blockIdx.x;  // most key tiles first
  const int u = unit0 + (int)blockIdx.y;
  const int n = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->ds_full, 4);
    mbar_init(&bars->dsdone, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 5) tmem_alloc(&bars->tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256;

  if (warp == 4) {
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
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idAcc = idesc_f16(128, D, true);
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
      const uint32_t aDS = smem_u32(sDS);
      auto issue_dq = [&](int j) {  // dQ += dS_j K_j
        const int st = j % STG;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = aDS + (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t b = aK + st * Lt::kTile + kk * 2048;
          umma_f16(tDQ, desc_kmajor(a), desc_mnmajor(b, 16384), idAcc, (j > 0 || kk > 0));
        }
        umma_commit(&bars->dsdone);
        umma_commit(&bars->kv_empty[st]);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, kStatus);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % STG;
        if (STG == 1 && j > 0) {  // one K/V stage: free it before the next tile loads
          ok = mbar_wait(&bars->ds_full, (j - 1) & 1, abort, kStatus);
          if (!ok) break;
          tc_fence_after();
          issue_dq(j - 1);
        }
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
        if (STG > 1 && j > 0) {
          ok = mbar_wait(&bars->ds_full, (j - 1) & 1, abort, kStatus);
          if (!ok) break;
          tc_fence_after();
          issue_dq(j - 1);
        }
      }
      if (ok && mbar_wait(&bars->ds_full, (n - 1) & 1, abort, kStatus)) {
        tc_fence_after();
        issue_dq(n - 1);
      }
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, abort, kStatus, false);
    }
  } else {
    const int r = threadIdx.x;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const int row = qt * 128 + r;
    const bool in = row < S;
    const float lse2 = in ? __ldg(lse + (int64_t)u * S + row) * kLog2e : 0.0f;
    const float Dr = in ? __ldg(Dv + (int64_t)u * S + row) : 0.0f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = warp_wait(&bars->s_full, j & 1, abort, kStatus);
      if (!ok) break;
      tc_fence_after();
      const bool diag = (j == qt);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t a[32], b[32];
        tmem_ld32(tS + lane_addr + ch * 32, a);
        tmem_ld32(tDP + lane_addr + ch * 32, b);
        tmem_ld_wait();
        if (ch == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->s_free);
        }
        uint32_t pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int k = ch * 32 + e;
          float p0 = ex2(fmaf(__uint_as_float(a[e]), scale_log2, -lse2));
          float p1 = ex2(fmaf(__uint_as_float(a[e + 1]), scale_log2, -lse2));
          if (diag && k > r) p0 = 0.0f;
          if (diag && k + 1 > r) p1 = 0.0f;
          pd[e >> 1] = pack_h2_sat(p0 * (__uint_as_float(b[e]) - Dr),
                                   p1 * (__uint_as_float(b[e + 1]) - Dr));
        }
        if (ch == 0 && j > 0 && !(ok = warp_wait(&bars->dsdone, (j - 1) & 1, abort, kStatus))) break;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int c = ch * 4 + qd;
          const uint32_t off = (c >> 3) * 16384 + swz(r, c & 7);
          *reinterpret_cast<uint4*>(sDS + off) =
              make_uint4(pd[4 * qd], pd[4 * qd + 1], pd[4 * qd + 2], pd[4 * qd + 3]);
        }
      }
      if (!ok) break;
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full);
    }
    if (ok) ok = warp_wait(&bars->dsdone, (n - 1) & 1, abort, kStatus);
    if (ok) {  // whole warps load TMEM; only rows inside the sequence are stored
      tc_fence_after();
      float* gq = dqs + ((int64_t)u * S + row) * D;
#pragma unroll
      for (int h = 0; h < D / 32; ++h) {
        uint32_t v[32];
        tmem_ld32(tDQ + lane_addr + h * 32, v);
        tmem_ld_wait();
        if (in) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(gq + h * 32 + 4 * c) =
                make_float4(__uint_as_float(v[4 * c]) * scale, __uint_as_float(v[4 * c + 1]) * scale,
                            __uint_as_float(v[4 * c + 2]) * scale, __uint_as_float(v[4 * c + 3]) * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
    const int64_t nu = g.U - u0 < 65535 ? g.U - u0 : 65535;
    k_attn_fwd_tc<D><<<dim3(ntiles, (unsigned)nu), kFwdThreads, smem, st>>>(
        mq, mk, mv, os, lse, (int)g.S, (int)u0, scale * kLog2e, ntiles);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t bwd_d(const Geom& g, const __half* qs, const __half* ks, const __half* vs,
                  const __half* dos, const float* lse, const float* Dv, float scale, float* dqs,
                  float* dks, float* dvs, cudaStream_t st) {
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
  for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
    const int64_t nu = g.U - u0 < 65535 ? g.U - u0 : 65535;
    k_attn_bwd_dkdv_tc<D><<<dim3(ntiles, (unsigned)nu), kFwdThreads, smem_a, st>>>(
        mq, mk, mv, mdo, lse, Dv, dks, dvs, (int)g.S, (int)u0, scale, scale * kLog2e, ntiles);
    k_attn_bwd_dq_tc<D><<<dim3(ntiles, (unsigned)nu), kFwdThreads, smem_b, st>>>(
        mq, mk, mv, mdo, lse, Dv, dqs, (int)g.S, (int)u0, scale, scale * kLog2e, ntiles);
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
int attn_tc_fwd_launches(const Geom& g) { return (int)((g.U + 65534) / 65535); }
int attn_tc_bwd_launches(const Geom& g) { return 2 * (int)((g.U + 65534) / 65535); }

cudaError_t launch_attn_fwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, float scale, __half* os, float* lse,
                               cudaStream_t st) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::fwd_d<64>(g, qs, ks, vs, scale, os, lse, st)
                   : tc::fwd_d<128>(g, qs, ks, vs, scale, os, lse, st);
}

cudaError_t launch_attn_bwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, const __half* dos, const float* lse,
                               const float* Dv, float scale, float* dqs, float* dks, float* dvs,
                               cudaStream_t st) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::bwd_d<64>(g, qs, ks, vs, dos, lse, Dv, scale, dqs, dks, dvs, st)
                   : tc::bwd_d<128>(g, qs, ks, vs, dos, lse, Dv, scale, dqs, dks, dvs, st);
}

}  // namespace lh
