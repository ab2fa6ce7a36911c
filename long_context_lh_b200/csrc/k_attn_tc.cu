// k_attn_tc.cu -- causal attention on the gathered sub-sequence with the
// 5th-generation tensor cores (tcgen05 MMA, accumulators in TMEM, operands
// staged by TMA in 128-byte-swizzled shared memory).
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.C: stock causal attention on the dense
// sub-sequence (row k sees k' <= k), scale 1/sqrt(d); §2.B: its backward is the
// only path from the layer output back to the selected Q, K and V.
//
// All three kernels use one CTA per SM (512 TMEM columns) and 11 warps:
//   warps 0-7  the row work (TMEM lane = row; warp w reads lanes 32*(w%4)..):
//              in the forward, one thread per row of one of two query tiles
//              (warps 0-3 tile A, 4-7 tile B, ping-pong); in the two backward
//              kernels, two threads per row of the one 128-row tile, warp w
//              taking the column half w/4;
//   warp 8     TMA producer (one lane issues);
//   warps 9-10 MMA issuers, on two SM sub-partitions: each waits as a whole
//              converged warp and one elected lane issues.  Warp 9 issues the
//              score products (S, or S^T and dP^T, or S and dP), warp 10 the
//              products that consume them (P V, or dV and dK, or dQ); at d = 128
//              the forward issues from warp 9 alone.  Warp 9 owns the TMEM
//              allocation.
// The backward kernels read a score tile from TMEM into registers in one go
// and release the buffer at once, so the next tile's products run while the
// row work goes on; the forward releases it after its second read.
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
constexpr int kThreads = 352;  // 8 row-work warps, TMA warp 8, MMA warps 9 and 10
constexpr uint32_t kTmemCols = 512;

// The dQ kernel reads nothing the dK/dV kernel writes, so it is launched as a
// programmatic dependent of it: the dK/dV kernel releases it once all its CTAs
// run (pdl_release), and dQ CTAs fill the SMs its last wave frees.  Each dQ CTA
// waits, before it exits, for the dK/dV kernel to have completed (pdl_join), so
// that whatever follows the dQ kernel in the stream sees both kernels' results.
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
__device__ __forceinline__ void pdl_join() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

__device__ __forceinline__ void store_row_half(uint8_t* tile_half, int r, const uint32_t (&pk)[32]) {
  // one 64-column half of a row of a 128-byte-swizzled fp16 tile: 8 chunks of 16 B
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(tile_half + swz(r, c)) =
        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// ================================================================= forward
// Ping-pong: one CTA per (unit, pair of query tiles) -- tiles A = 2i+1 and
// B = 2i (A alone when it is the last, odd one).  Both walk the same key tiles
// (B one fewer), so each K/V tile is loaded once for both.  Row-work warps 0-3
// own tile A, warps 4-7 tile B, one thread per row and all 128 keys of a tile:
// every SM sub-partition holds one warp of each tile, and the two alternate
// (while one computes its exponentials, the tensor core serves the other).
// TMEM: S_A, S_B (128 columns each), O_A, O_B (D columns each) and, at d = 64,
// P_A, P_B (64 columns each, packed fp16).  At d = 64 a tile's row work releases
// S_T as soon as it has read it (before its exponentials are done), and the MMA
// warp issues S_T(j+1) then, so the next scores are computed under the current
// tile's exponentials and O_T += P_T(j) V(j) runs under the next tile's row max.
// At d = 128 TMEM is full: P is written over the S columns already read, and
// S_T(j+1) follows O_T += P_T(j) V(j).
template <int D>
struct FwdLayout {
  static constexpr int kKS = (D == 64) ? 4 : 2;  // K/V stages
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQ = 0;                   // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kTile;
  static constexpr int kV = kK + kKS * kTile;
  static constexpr int kBar = kV + kKS * kTile;
};

struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[4], kv_empty[4];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], mma_done;  // [tile A, B]
  uint32_t tmem;
  int abort;
};

template <int D>
constexpr int fwd_smem_bytes() {
  return FwdLayout<D>::kBar + (int)sizeof(FwdBars);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, __half* __restrict__ os,
                  float* __restrict__ lse, int S, int unit0, int nunits, float scale_log2,
                  int ntiles, int full) {
  pdl_enter();
  using Lt = FwdLayout<D>;
  constexpr int KS = Lt::kKS;
  static_assert(KS >= 1 && KS <= 4, "FwdBars holds at most 4 stages");
  static_assert(256 + 2 * D <= (int)kTmemCols, "TMEM: S_A, S_B, O_A, O_B");
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_status(kStatusAttnFwdTimeout | 1u);
    return;
  }
  constexpr bool kSepP = (D == 64);
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + Lt::kBar);
  uint8_t* sQ = smem + Lt::kQ;
  uint8_t* sK = smem + Lt::kK;
  uint8_t* sV = smem + Lt::kV;
  volatile int* abort = &bars->abort;
  constexpr uint32_t kStatus = kStatusAttnFwdTimeout;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 1-D grid ordered by work: all units' last (longest) pairs first
  const int npairs = (ntiles + 1) / 2;
  const int pi = npairs - 1 - (int)(blockIdx.x / nunits);
  const int u = unit0 + (int)(blockIdx.x % nunits);
  const bool hasB = 2 * pi + 1 < ntiles;
  const int qtA = hasB ? 2 * pi + 1 : 2 * pi;  // the longer tile
  const int qtB = hasB ? 2 * pi : -1;
  // key tiles of each (nB = 0: no tile B): causal, the tiles up to the diagonal;
  // full (a query block against an earlier key block), all of them
  const int nA = full ? ntiles : qtA + 1, nB = qtB < 0 ? 0 : (full ? ntiles : qtB + 1);
  // debug build: the CTA's unit and query tiles lie inside the problem (checked
  // before any barrier or TMEM is set up, so a bad CTA leaves as a whole)
  if (!LH_CHECK(pi >= 0 && u < unit0 + nunits && (int64_t)qtA * 128 < S && qtB < qtA, kBoundsAttnFwd))
    return;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->s_free[t], 4);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->pv_done[t], 1);
    }
    mbar_init(&bars->mma_done, kSepP ? 2 : 1);  // one commit from each MMA issuer
    bars->abort = 0;
    mbar_init_fence();
  }
  if (warp == 9) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t tO = tmem + 256;  // O_A at +256, O_B at +256+D; S_T at +128*T
  // d = 64: P_A, P_B in their own columns (+384, +448), so S_T(j+1) need not
  // wait for O_T += P_T(j) V_j (kSepP, defined above)
  static_assert(!kSepP || 256 + 2 * D + 128 <= (int)kTmemCols, "TMEM: S_A, S_B, O_A, O_B, P_A, P_B");
  const uint32_t tP = tmem + 256 + 2 * D;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bars->q_full, (hasB ? 2 : 1) * Lt::kTile);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sQ + h * 16384, &tq, &bars->q_full, h * 64, qtA * 128, u);
        if (hasB) tma_load_3d(sQ + Lt::kTile + h * 16384, &tq, &bars->q_full, h * 64, qtB * 128, u);
      }
      int issued = 0;
      for (int j = 0; j < nA; ++j) {
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
  } else if (warp == 9 || (kSepP && warp == 10)) {
    // ------------------------------------------------------------- MMA issuers
    // The whole warp runs the loop (its waits are warp-uniform) and computes the
    // descriptors, so they stay warp-uniform values; one elected lane issues
    // each group of MMAs and its commit.  (Issuing from lane 0 inside a
    // lane-0-only branch measured ~1.4x slower per MMA when row-work warps share
    // the issuer's SM sub-partition.)  At d = 64 two warps on two sub-partitions
    // issue: warp 9 the S products, warp 10 the P V products (an issuing warp
    // competes with the row-work warps of its sub-partition; splitting halves
    // that load).  At d = 128 P lives over S, so S_T(j+1) must follow
    // O_T += P_T(j) V_j in one in-order stream: warp 9 issues everything.
    // A descriptor for base + off is the base descriptor plus off / 16 (the
    // 14-bit address field never overflows inside shared memory).  At d = 64
    // the two issuers sleep 16 ns between polls of a barrier (spinning, each
    // slowed the row-work warps of its sub-partition: forward 190 -> 184 us at
    // the pretraining shape with the sleep); the backward's issuers sit on the
    // critical handoffs and poll without sleeping (the same sleep there: 509 ->
    // 541 us).
    constexpr uint32_t kIssuerSleepNs = 16;
    {
      constexpr uint32_t idS = idesc_f16(128, 128, false);
      constexpr uint32_t idPV = idesc_f16(128, D, true);
      const uint64_t dQ = desc_kmajor(smem_u32(sQ)), dK = desc_kmajor(smem_u32(sK));
      const uint64_t dV = desc_mnmajor(smem_u32(sV), 16384);
      auto issue_s = [&](int t, int j) {  // S_t = Q_t K_j^T
        const uint64_t q = dQ + (uint64_t)((t * Lt::kTile) >> 4);
        const uint64_t k = dK + (uint64_t)(((j % KS) * Lt::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)((((kk >> 2) * 16384) + ((kk & 3) * 32)) >> 4);
            umma_f16(tmem + t * 128, q + off, k + off, idS, kk > 0);
          }
          umma_commit(&bars->s_full[t]);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int j) {  // O_t += P_t(j) V_j, P_t from TMEM
        const uint64_t v = dV + (uint64_t)(((j % KS) * Lt::kTile) >> 4);
        const uint32_t pt = kSepP ? tP + t * 64 : tmem + t * 128;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ta(tO + t * D, pt + 8 * kk, v + (uint64_t)((kk * 2048) >> 4), idPV,
                        (j > 0 || kk > 0));
          umma_commit(&bars->pv_done[t]);
        }
        __syncwarp();
      };
      bool ok = true;
      if (warp == 9) {
        ok = warp_wait(&bars->q_full, 0, abort, kStatus) &&
             warp_wait(&bars->kv_full[0], 0, abort, kStatus);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          if (nB > 0) issue_s(1, 0);
        }
      }
      if constexpr (kSepP) {
        if (warp == 9) {
          // S_T(j+1) once S_T(j) is read (and K_{j+1} is in place), tile A then B
          for (int j = 0; ok && j + 1 < nA; ++j) {
            if (!(ok = warp_wait_sleep(&bars->s_free[0], j & 1, abort, kStatus, kIssuerSleepNs))) break;
            if (!(ok = warp_wait_sleep(&bars->kv_full[(j + 1) % KS], ((j + 1) / KS) & 1, abort, kStatus, kIssuerSleepNs))) break;
            tc_fence_after();
            issue_s(0, j + 1);
            if (j + 1 < nB) {  // K_{j+1} is in place (waited for above: j + 1 < nB <= nA)
              if (!(ok = warp_wait_sleep(&bars->s_free[1], j & 1, abort, kStatus, kIssuerSleepNs))) break;
              tc_fence_after();
              issue_s(1, j + 1);
            }
          }
        } else {
          // O_T += P_T(j) V_j once P_T(j) is written, tile A then B; then K_j, V_j
          // are free (S_A(j), S_B(j) completed before the row work wrote P)
          for (int j = 0; ok && j < nA; ++j) {
            const int st = j % KS;
            if (!(ok = warp_wait_sleep(&bars->p_full[0], j & 1, abort, kStatus, kIssuerSleepNs))) break;
            tc_fence_after();
            issue_pv(0, j);
            if (j < nB) {
              if (!(ok = warp_wait_sleep(&bars->p_full[1], j & 1, abort, kStatus, kIssuerSleepNs))) break;
              tc_fence_after();
              issue_pv(1, j);
            }
            if (elect_one()) umma_commit(&bars->kv_empty[st]);
            __syncwarp();
          }
        }
      }
      for (int j = 0; !kSepP && ok && j < nA; ++j) {
        const int st = j % KS;
        const bool next = j + 1 < nA;
        // tile A: its product with V_j, then (S_A buffer free again) its next scores
        if (!(ok = warp_wait(&bars->p_full[0], j & 1, abort, kStatus))) break;
        tc_fence_after();
        issue_pv(0, j);
        if (next) {
          if (!(ok = warp_wait(&bars->kv_full[(j + 1) % KS], ((j + 1) / KS) & 1, abort, kStatus))) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        // tile B likewise
        if (j < nB) {
          if (!(ok = warp_wait(&bars->p_full[1], j & 1, abort, kStatus))) break;
          tc_fence_after();
          issue_pv(1, j);
          if (j + 1 < nB) issue_s(1, j + 1);
        }
        if (elect_one()) umma_commit(&bars->kv_empty[st]);  // K_j, V_j no longer needed
        __syncwarp();
      }
      if (elect_one()) umma_commit(&bars->mma_done);  // from each issuer
      __syncwarp();
      // every MMA issued has completed before TMEM is freed, aborted or not
      warp_wait(&bars->mma_done, 0, abort, kStatus, false);
    }
  } else if (warp < 8) {
    // -------------------- row work: one thread per row of its tile, all 128 keys
    // P is formed against a running reference max m_ref, and O_t is rescaled in
    // TMEM only when a tile's max exceeds m_ref by more than kRescale (exp2
    // domain), so P <= 2^kRescale fits fp16; softmax is invariant to the
    // reference, so the result is the same.
    constexpr float kRescale = 8.0f;
    const int t = warp >> 2;  // 0: tile A, 1: tile B
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const int n = t == 0 ? nA : nB;
    const int qt = t == 0 ? qtA : qtB;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_addr;
    const uint32_t tOt = tO + t * D + lane_addr;
    float m_ref = -INFINITY, l = 0.0f;
    bool ok = true;
    // the masked (last) key tile keeps keys 0..lim: causal, the keys up to the
    // row (the diagonal tile); full, the keys inside the block (a ragged tail)
    const int lim = full ? ((S - 1) & 127) : r;
    const bool mask_last = !full || (S & 127) != 0;
    // one key tile; kDiag: the last tile with the mask above
    auto step = [&](int j, auto diag_tag) {
      constexpr bool kDiag = decltype(diag_tag)::value;
      ok = warp_wait(&bars->s_full[t], j & 1, abort, kStatus);
      if (!ok) return;
      tc_fence_after();
      // the row max over the whole row of S (128 columns): four loads, one wait,
      // four independent chains
      float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      {
        uint32_t v[128];
        tmem_ld32_at<0>(tS, v);
        tmem_ld32_at<32>(tS + 32, v);
        tmem_ld32_at<64>(tS + 64, v);
        tmem_ld32_at<96>(tS + 96, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 128; i += 2) {
          const int k = (i >> 1) & 3;
          if (kDiag) {
            mc[k] = max3(mc[k], i <= lim ? __uint_as_float(v[i]) : -INFINITY,
                         i + 1 <= lim ? __uint_as_float(v[i + 1]) : -INFINITY);
          } else {
            mc[k] = max3(mc[k], __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
          }
        }
      }
      const float mx = fmaxf(max3(mc[0], mc[1], mc[2]), mc[3]) * scale_log2;  // finite: key 0
      const bool grow = mx > m_ref + kRescale;
      const float m_new = grow ? mx : m_ref;
      // every phase of pv_done[t] is waited for, in order; O_t (and the P of the
      // previous tile) must be done with before O_t is rescaled or P rewritten
      auto pv_wait_rescale = [&]() -> bool {
        if (j > 0 && !warp_wait(&bars->pv_done[t], (j - 1) & 1, abort, kStatus)) return false;
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          tc_fence_after();
          const float alpha = ex2(m_ref - m_new);  // 1 for rows that do not grow
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tOt + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(tOt + c * 32, ov);
          }
          l *= alpha;
        }
        m_ref = m_new;
        return true;
      };
      // at d = 64 the wait is deferred to the first P store (after the first
      // 32 exponentials), so the previous P V runs under the row max
      if constexpr (!kSepP) {
        ok = pv_wait_rescale();
        if (!ok) return;
      }
      // P = 2^(S c - m_ref): S read again in two 64-column halves (two loads, one
      // wait each), packed fp16 written over S columns already read (chunk c of
      // 32 columns writes columns 16c..16c+15)
      const float2 cc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_new, -m_new);
      float2 sacc[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                        make_float2(0.0f, 0.0f)};
      uint32_t v[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if ((c & 1) == 0) {
          tmem_ld32_at<0>(tS + 32 * c, v);
          tmem_ld32_at<32>(tS + 32 * c + 32, v);
          tmem_ld_wait();
          if (kSepP && c == 2) {  // S_t(j) fully read: the MMA warp may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->s_free[t]);
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int a = 32 * (c & 1) + i;
          const float2 x = ffma2(make_float2(__uint_as_float(v[a]), __uint_as_float(v[a + 1])), cc, nm);
          const float2 y = ffma2(make_float2(__uint_as_float(v[a + 2]), __uint_as_float(v[a + 3])), cc, nm);
          float2 p = make_float2(ex2(x.x), ex2(x.y));
          // a quarter of the exponentials on the FMA pipe, the rest on MUFU (half
          // on the FMA pipe measured slower: the row work is then issue-bound;
          // three eighths the same as a quarter)
          float2 q = (i & 7) == 4 ? ex2_fma2(y) : make_float2(ex2(y.x), ex2(y.y));
          if (kDiag) {
            const int k0 = 32 * c + i;
            p.x = k0 <= lim ? p.x : 0.0f;
            p.y = k0 + 1 <= lim ? p.y : 0.0f;
            q.x = k0 + 2 <= lim ? q.x : 0.0f;
            q.y = k0 + 3 <= lim ? q.y : 0.0f;
          }
          const int k = (i >> 2) & 1;
          sacc[2 * k] = fadd2(sacc[2 * k], p);
          sacc[2 * k + 1] = fadd2(sacc[2 * k + 1], q);
          pk[i >> 1] = h2(p.x, p.y);
          pk[(i >> 1) + 1] = h2(q.x, q.y);
        }
        if constexpr (kSepP) {
          if (c == 0) {
            ok = pv_wait_rescale();
            if (!ok) return;
          }
          tmem_st16(tP + t * 64 + lane_addr + 16 * c, pk);
        } else {
          tmem_st16(tS + 16 * c, pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();  // orders P and the O_t rescale (TMEM stores) before the product
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t]);
      const float2 s01 = fadd2(sacc[0], sacc[1]), s23 = fadd2(sacc[2], sacc[3]);
      l += (s01.x + s01.y) + (s23.x + s23.y);
    };
    if (n > 0) {
      for (int j = 0; j < n - 1 && ok; ++j) step(j, std::false_type{});
      if (ok) {
        if (mask_last)
          step(n - 1, std::true_type{});
        else
          step(n - 1, std::false_type{});
      }
      if (ok) ok = warp_wait(&bars->pv_done[t], (n - 1) & 1, abort, kStatus);
      const int row = qt * 128 + r;
      if (ok) {  // whole warps load TMEM; only rows inside the sequence are stored
        tc_fence_after();
        const float inv = 1.0f / l;
        __half* dst = os + ((int64_t)u * S + row) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tOt + c * 32, ov);
          tmem_ld_wait();
          if (row < S) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              uint4 w;
              w.x = h2_sat(__uint_as_float(ov[8 * x + 0]) * inv, __uint_as_float(ov[8 * x + 1]) * inv);
              w.y = h2_sat(__uint_as_float(ov[8 * x + 2]) * inv, __uint_as_float(ov[8 * x + 3]) * inv);
              w.z = h2_sat(__uint_as_float(ov[8 * x + 4]) * inv, __uint_as_float(ov[8 * x + 5]) * inv);
              w.w = h2_sat(__uint_as_float(ov[8 * x + 6]) * inv, __uint_as_float(ov[8 * x + 7]) * inv);
              *reinterpret_cast<uint4*>(dst + c * 32 + 8 * x) = w;
            }
          }
        }
        if (row < S) lse[(int64_t)u * S + row] = (m_ref + __log2f(l)) * kLn2;
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
                       int nunits, float scale, float scale_log2, int ntiles, int full) {
  pdl_enter();
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
  // query tiles i0.. of this key tile: causal, from the diagonal on; full (an
  // earlier key block), all of them, none masked (padded query rows have P = 0)
  const int i0 = full ? 0 : kt;
  const int n = ntiles - i0;
  if (!LH_CHECK(kt < ntiles && (int64_t)kt * 128 < S, kBoundsAttnBwd)) return;  // whole CTA

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
    mbar_init(&bars->mma_done, 2);  // one commit from each MMA issuer
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
        const int st = t % STG, i = i0 + t;
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
  } else if (warp == 9 || warp == 10) {
    // Two MMA issuers on two SM sub-partitions: warp 9 the S^T and dP^T products
    // of every query tile, warp 10 the dV and dK products.  (An issuing warp
    // competes for issue slots with the row-work warps of its sub-partition,
    // and those set the pace of every handoff; splitting the products halves
    // that load.)  Each whole warp waits and computes the descriptors, so they
    // stay warp-uniform; one elected lane issues each group and its commits.
    // A descriptor for base + off is the base descriptor plus off / 16 (the
    // 14-bit address field never overflows inside shared memory).
    constexpr uint32_t idS = idesc_f16(128, 128, false);
    constexpr uint32_t idAcc = idesc_f16(128, D, true);
    bool ok = true;
    if (warp == 9) {
      const uint64_t dK = desc_kmajor(smem_u32(sK)), dV = desc_kmajor(smem_u32(sV));
      const uint64_t dQk = desc_kmajor(smem_u32(sQ)), dDOk = desc_kmajor(smem_u32(sDO));
      ok = warp_wait(&bars->kv_full, 0, abort, kStatus);
      for (int t = 0; ok && t < n; ++t) {
        const int st = t % STG;
        // Q_t, dO_t in place; S^T, dP^T of the previous tile read by the row work
        ok = warp_wait(&bars->q_full[st], (t / STG) & 1, abort, kStatus) &&
             (t == 0 || warp_wait(&bars->st_free, (t - 1) & 1, abort, kStatus));
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * Lt::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)((((kk >> 2) * 16384) + ((kk & 3) * 32)) >> 4);
            umma_f16(tST, dK + off, dQk + so + off, idS, kk > 0);
            umma_f16(tDPT, dV + off, dDOk + so + off, idS, kk > 0);
          }
          umma_commit(&bars->s_full);
        }
        __syncwarp();
      }
    } else {
      const uint64_t dQm = desc_mnmajor(smem_u32(sQ), 16384), dDOm = desc_mnmajor(smem_u32(sDO), 16384);
      const uint64_t dPT = desc_kmajor(smem_u32(sPT)), dDST = desc_kmajor(smem_u32(sDST));
      for (int t = 0; ok && t < n; ++t) {  // dV += P^T dO_t, dK += dS^T Q_t
        ok = warp_wait(&bars->p_full, t & 1, abort, kStatus);  // P^T, dS^T of tile t written
        if (!ok) break;
        tc_fence_after();
        const int st = t % STG;
        const uint64_t so = (uint64_t)((st * Lt::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = (uint64_t)((((kk >> 2) * 16384) + ((kk & 3) * 32)) >> 4);
            const uint64_t b = so + (uint64_t)((kk * 2048) >> 4);
            if constexpr (kTmemP) {
              umma_f16_ta(tDV, tPT + 8 * kk, dDOm + b, idAcc, (t > 0 || kk > 0));
              umma_f16_ta(tDK, tDST + 8 * kk, dQm + b, idAcc, (t > 0 || kk > 0));
            } else {
              umma_f16(tDV, dPT + a, dDOm + b, idAcc, (t > 0 || kk > 0));
              umma_f16(tDK, dDST + a, dQm + b, idAcc, (t > 0 || kk > 0));
            }
          }
          umma_commit(&bars->pdone);
          umma_commit(&bars->q_empty[st]);  // stage st free for tile t + STG
        }
        __syncwarp();
      }
    }
    // both issuers commit: every MMA issued has completed before TMEM is freed
    if (elect_one()) umma_commit(&bars->mma_done);
    __syncwarp();
    warp_wait(&bars->mma_done, 0, abort, kStatus, false);
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
      // this row's 64 query columns of S^T and dP^T in two 32-column halves (the
      // second loaded once the first is consumed: the registers they free let a
      // quarter of the exponentials run on the FMA pipe without spilling)
      uint32_t a[32], b[32];
      tmem_ld32(tST + lane_addr + h * 64, a);
      tmem_ld32(tDPT + lane_addr + h * 64, b);
      tmem_ld_wait();
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
        // a quarter of the exponentials on the FMA pipe (this row work is MUFU-bound)
        float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
        float2 p1 = (e & 4) ? ex2_fma2(x1) : make_float2(ex2(x1.x), ex2(x1.y));
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
      for (int e = 0; e < 32; e += 4) quad(e, a, b);
      tmem_ld32(tST + lane_addr + h * 64 + 32, a);
      tmem_ld32(tDPT + lane_addr + h * 64 + 32, b);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->st_free);  // S^T, dP^T are in registers now
#pragma unroll
      for (int e = 32; e < 64; e += 4) quad(e, a, b);
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
    if (full)
      step(0, std::false_type{});
    else
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
                     float scale_log2, int ntiles, int full) {
  using Lt = DqLayout<D>;
  constexpr int STG = Lt::kStages;
  static_assert(STG >= 1 && STG <= 4, "DqBars holds at most 4 stages");
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_status(kStatusAttnBwdTimeout | 2u);
    pdl_join();
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
  const int n = full ? ntiles : qt + 1;  // key tiles: up to the diagonal, or all of the block
  if (!LH_CHECK(qt >= 0 && (int64_t)qt * 128 < S, kBoundsAttnBwd)) {  // whole CTA
    pdl_join();
    return;
  }

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
    mbar_init(&bars->mma_done, 2);  // one commit from each MMA issuer
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
  } else if (warp == 9 || warp == 10) {
    // Two MMA issuers, as in the dK/dV kernel: warp 9 the S and dP products of
    // every key tile, warp 10 the dQ products; descriptors are base descriptors
    // plus offset / 16
    constexpr uint32_t idS = idesc_f16(128, 128, false);
    constexpr uint32_t idAcc = idesc_f16(128, D, true);
    bool ok = true;
    if (warp == 9) {
      const uint64_t dQ = desc_kmajor(smem_u32(sQ)), dDO = desc_kmajor(smem_u32(sDO));
      const uint64_t dK = desc_kmajor(smem_u32(sK)), dV = desc_kmajor(smem_u32(sV));
      ok = warp_wait(&bars->q_full, 0, abort, kStatus);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % STG;
        // K_j, V_j in place; S, dP of the previous key tile read by the row work
        ok = warp_wait(&bars->kv_full[st], (j / STG) & 1, abort, kStatus) &&
             (j == 0 || warp_wait(&bars->s_free, (j - 1) & 1, abort, kStatus));
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * Lt::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)((((kk >> 2) * 16384) + ((kk & 3) * 32)) >> 4);
            umma_f16(tS, dQ + off, dK + so + off, idS, kk > 0);
            umma_f16(tDP, dDO + off, dV + so + off, idS, kk > 0);
          }
          umma_commit(&bars->s_full);
        }
        __syncwarp();
      }
    } else {
      const uint64_t dKm = desc_mnmajor(smem_u32(sK), 16384);
      for (int j = 0; ok && j < n; ++j) {  // dQ += dS_j K_j, dS_j from TMEM
        const int st = j % STG, b = j & 1;
        ok = warp_wait(&bars->ds_full[b], (j >> 1) & 1, abort, kStatus);
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * Lt::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ta(tDQ, tDS + b * 64 + 8 * kk, dKm + so + (uint64_t)((kk * 2048) >> 4), idAcc,
                        (j > 0 || kk > 0));
          umma_commit(&bars->dsdone[b]);
          umma_commit(&bars->kv_empty[st]);  // K_j, V_j no longer needed (S, dP done before dS)
        }
        __syncwarp();
      }
    }
    // both issuers commit: every MMA issued has completed before TMEM is freed
    if (elect_one()) umma_commit(&bars->mma_done);
    __syncwarp();
    warp_wait(&bars->mma_done, 0, abort, kStatus, false);
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
      // key columns e > lim are masked in the last tile: those after the query
      // (causal), those past the block's end (full, ragged tail)
      const int lim = (full ? ((S - 1) & 127) : r) - h * 64;
      uint32_t pd[32];
      auto pair = [&](int e, uint32_t s0, uint32_t s1, uint32_t g0, uint32_t g1) {
        const float2 x = ffma2(make_float2(__uint_as_float(s0), __uint_as_float(s1)), cc, nl);
        // a quarter of the exponentials on the FMA pipe (this row work is MUFU-bound;
        // measured: none 571 us, a quarter 530, half 546 for the whole backward)
        float2 p = (e & 6) == 6 ? ex2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
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
    if (ok) {
      if (!full || (S & 127) != 0)
        step(n - 1, std::true_type{});
      else
        step(n - 1, std::false_type{});
    }
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
  pdl_join();
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
                  float scale, __half* os, float* lse, int full, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qs, D, g.S, g.U) || !make_map(&mk, ks, D, g.S, g.U) ||
      !make_map(&mv, vs, D, g.S, g.U))
    return cudaErrorNotSupported;
  constexpr int smem = fwd_smem_bytes<D>();
  cudaError_t e =
      cudaFuncSetAttribute(k_attn_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((g.S + 127) / 128);
  const int npairs = (ntiles + 1) / 2;
  const int64_t per = 0x7fffffff / npairs;  // units per launch (grid.x limit)
  for (int64_t u0 = 0; u0 < g.U; u0 += per) {
    const int64_t nu = g.U - u0 < per ? g.U - u0 : per;
    (void)launch_pdl(k_attn_fwd_tc<D>, (unsigned)(nu * npairs), kThreads, smem, st, 
        mq, mk, mv, os, lse, (int)g.S, (int)u0, (int)nu, scale * kLog2e, ntiles, full);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t bwd_d(const Geom& g, const __half* qs, const __half* ks, const __half* vs,
                  const __half* dos, const float* stats, float scale, float* dqs, float* dks,
                  float* dvs, int full, cudaStream_t st) {
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
    (void)launch_pdl(k_attn_bwd_dkdv_tc<D>, (unsigned)(nu * ntiles), kThreads, smem_a, st, 
        mq, mk, mv, mdo, stats, dks, dvs, (int)g.S, (int)u0, (int)nu, scale, scale * kLog2e,
        ntiles, full);
    // a programmatic dependent of the dK/dV kernel (see pdl_release / pdl_join)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nu * ntiles), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_b;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_attn_bwd_dq_tc<D>, mq, mk, mv, mdo, stats, dqs, (int)g.S, (int)u0,
                           (int)nu, scale, scale * kLog2e, ntiles, full);
    if (e != cudaSuccess) return e;
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
  const int64_t npairs = ((g.S + 127) / 128 + 1) / 2, per = 0x7fffffff / npairs;
  return (int)((g.U + per - 1) / per);
}
int attn_tc_bwd_launches(const Geom& g) {
  const int64_t ntiles = (g.S + 127) / 128, per = 0x7fffffff / ntiles;
  return 2 * (int)((g.U + per - 1) / per);
}

cudaError_t launch_attn_fwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, float scale, __half* os, float* lse,
                               cudaStream_t st, int full) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::fwd_d<64>(g, qs, ks, vs, scale, os, lse, full, st)
                   : tc::fwd_d<128>(g, qs, ks, vs, scale, os, lse, full, st);
}

cudaError_t launch_attn_bwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, const __half* dos, const float* stats,
                               float scale, float* dqs, float* dks, float* dvs, cudaStream_t st,
                               int full) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::bwd_d<64>(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, full, st)
                   : tc::bwd_d<128>(g, qs, ks, vs, dos, stats, scale, dqs, dks, dvs, full, st);
}

}  // namespace lh
