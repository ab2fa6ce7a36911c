// k_topk.cu -- joint top-S over all pyramid levels and the gather order.
//
// Method: [ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
// Largo mediante Atención Lighthouse" §2.B (one top-K across all levels) and
// §2.C (the selected triplets are sorted topologically into one dense,
// hole-free sequence; phase 3 of bitsgeniais.com.br "Adeus Custo Quadrático!").
//
// Selection rule: the S entries with the largest (score, -gid); the ranking is
// a strict total order, so the set is unique.  Because it is a threshold rule,
// no sort of the keys is needed, only the S-th largest key:
//   1. radix select on the 32 score bits (scores are >= 0, so their bits order
//      like their values) in digits of 11/11/10 bits, giving the threshold score
//      T and how many entries scoring exactly T are still needed;
//   2. if only some of the entries at T fit, radix select (ascending) on their
//      gids gives the largest gid that still fits.
//   Entry g is selected iff score > T, or score == T and gid <= that gid.
// Gather order (pos ascending, then level ascending) is a fixed enumeration of
// all entries: token t = 0..N-1, and at each t the levels l whose span ends at
// t ((t+1) % p^l == 0).  One ordered stream compaction over that enumeration
// gives slots directly, with no sort.
//
// B200 mapping: one thread-block cluster of CL CTAs per unit.  Each CTA
// histograms its share of the unit's scores in shared memory; the cluster sums
// the histograms through distributed shared memory, and every CTA picks the
// digit redundantly (same integers, same result), so a pass costs one cluster
// barrier.  The compaction uses per-warp ballots/scans, per-CTA totals through
// DSMEM, and writes idx/pos/slot once.  Integer work only: bit-exact.
#include <cooperative_groups.h>

#include <atomic>
#include <type_traits>

#include "lh_internal.cuh"

namespace cg = cooperative_groups;

namespace lh {

// Status word of the selection kernel (bounds checks of the debug build).
__device__ uint32_t g_topk_status = 0;
#define LH_STATUS_WORD g_topk_status

cudaError_t topk_status_read_clear(uint32_t* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_topk_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_topk_status, &zero, sizeof(zero));
}

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
// Shared memory for a CTA's cached keys (the static part holds the histograms).
constexpr int64_t kKeyCacheBytes = 180 * 1024;
// Key bits of a kept coarsest entry: +inf, above every finite score; ties among
// kept entries go to the lower gid like any other tie.
constexpr uint32_t kTopBits = 0x7F800000u;
// At most this many entries tied at the threshold are resolved from a list;
// more take the radix passes over the gids.
constexpr int kTieCap = 256;

struct TopkParams {
  int32_t N, M;  // within-unit sizes fit 32 bits (M < 2^31 is a checked limit)
  int p, L, S, log2p;
  int keep_top;  // level L-1 ranks as +inf (keep-coarsest-level variant)
  int64_t unit0;
  int32_t off[kMaxLevels + 1];
  int32_t pw[kMaxLevels + 1];
};

// Does the span of a level-l entry end at token t, i.e. p^l divides t + 1?
__device__ __forceinline__ bool ends_at(const TopkParams& prm, uint32_t t1, int l) {
  return prm.log2p >= 0 ? (t1 & ((uint32_t)prm.pw[l] - 1u)) == 0u : (t1 % (uint32_t)prm.pw[l]) == 0u;
}
// gid of the level-l entry whose span ends at token t (requires ends_at)
__device__ __forceinline__ int32_t gid_at(const TopkParams& prm, uint32_t t1, int l) {
  const uint32_t j1 = prm.log2p >= 0 ? (t1 >> (l * prm.log2p)) : t1 / (uint32_t)prm.pw[l];
  return prm.off[l] + (int32_t)j1 - 1;
}

// Histogram increment.  Warp-aggregated (lanes with the same bin add once) when
// the keys crowd a few bins (the first digit); plain otherwise.
__device__ __forceinline__ void hist_add_plain(uint32_t* hist, bool active, uint32_t bin) {
  if (active) atomicAdd(&hist[bin], 1u);
}
__device__ __forceinline__ void hist_add(uint32_t* hist, bool active, uint32_t bin) {
  const unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const unsigned same = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == (unsigned)(__ffs(same) - 1)) atomicAdd(&hist[bin], (uint32_t)__popc(same));
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Block-wide exclusive scan of one value per thread; returns the exclusive
// prefix and writes the block total to *total (all threads see it).
__device__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_buf, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = warp_incl_scan(v);
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_buf[lane];
    uint32_t wi = warp_incl_scan(w);
    warp_buf[lane] = wi - w;  // exclusive
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  uint32_t res = warp_buf[warp] + incl - v;
  __syncthreads();  // warp_buf may be reused right after
  return res;
}

struct Pick {
  uint32_t bin;    // selected digit value
  uint32_t before; // count of candidates ranked before that digit
  uint32_t inbin;  // candidates with that digit
};

// Cluster-summed histogram -> digit where the need-th candidate falls.
// descending: rank digits from the largest value down (scores), else up (gids).
template <int CL>
__device__ Pick pick_digit(cg::cluster_group& cluster, uint32_t* hist, int nbins, bool descending,
                           uint32_t need, uint32_t* warp_buf, uint32_t* sh) {
  const int per = nbins / kThreads;  // 2 or 1 ordinals per thread
  uint32_t tot[2] = {0, 0};
  if (per == 2) {
    // the thread's two ordinals are adjacent bins: one 8-byte load per rank,
    // every rank's load in flight at once
    const int lo = descending ? nbins - 2 - 2 * (int)threadIdx.x : 2 * (int)threadIdx.x;
    uint2 v[CL];
#pragma unroll
    for (int r = 0; r < CL; ++r) v[r] = *reinterpret_cast<const uint2*>(cluster.map_shared_rank(hist, r) + lo);
    uint32_t a = 0, b = 0;
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      a += v[r].x;
      b += v[r].y;
    }
    tot[0] = descending ? b : a;  // ordinal 2t first
    tot[1] = descending ? a : b;
  } else {
    const int bin = descending ? (nbins - 1 - (int)threadIdx.x) : (int)threadIdx.x;
    uint32_t v[CL];
#pragma unroll
    for (int r = 0; r < CL; ++r) v[r] = cluster.map_shared_rank(hist, r)[bin];
#pragma unroll
    for (int r = 0; r < CL; ++r) tot[0] += v[r];
  }
  const uint32_t local = tot[0] + tot[1];
  uint32_t all;
  uint32_t before = block_excl_scan(local, warp_buf, &all);
  for (int i = 0; i < per; ++i) {
    const int ord = threadIdx.x * per + i;
    if (before < need && need <= before + tot[i]) {
      sh[0] = descending ? (uint32_t)(nbins - 1 - ord) : (uint32_t)ord;
      sh[1] = before;
      sh[2] = tot[i];
    }
    before += tot[i];
  }
  __syncthreads();
  Pick pk{sh[0], sh[1], sh[2]};
  __syncthreads();
  return pk;
}

// CTA r of the cluster owns the tokens [t_b, t_e) (whole coarsest spans) and
// every entry whose span lies in them: at level l the contiguous gids
// off[l] + [t_b / p^l, t_e / p^l).  Its keys are copied to shared memory once
// (cached != 0; else read from L2 in each pass); the histograms, the tie pass
// and the compaction then only touch the CTA's own keys.
template <int CL>
__global__ void __launch_bounds__(kThreads, 1)
    k_topk(const float* __restrict__ score, int32_t* __restrict__ idx, int32_t* __restrict__ pos,
           int32_t* __restrict__ slot, const TopkParams prm, int cached, int kcap, int masks) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int64_t u = prm.unit0 + blockIdx.y;

  __shared__ uint32_t hist[2][kBins];
  __shared__ uint32_t warp_buf[32];
  __shared__ uint32_t sh[4];
  __shared__ uint32_t warp_tot[kWarps];
  __shared__ uint32_t cta_total;
  __shared__ uint32_t tie_n;                 // this CTA's keys equal to the threshold T
  __shared__ uint32_t tie_gid[kTieCap];      // ... their gids
  __shared__ uint32_t all_tie[kTieCap];      // the cluster's, gathered
  extern __shared__ __align__(16) uint32_t skey[];  // the CTA's keys, level by level (cached), kcap words
  // then per token of the CTA: bits 0-7 the selected levels ending at it,
  // bits 8-15 all levels ending at it (written by the counting pass)
  uint16_t* smask = reinterpret_cast<uint16_t*>(skey + kcap);

  const uint32_t* key = reinterpret_cast<const uint32_t*>(score + u * prm.M);
  const int32_t Ptop = prm.pw[prm.L - 1];
  const int32_t spans = prm.N / Ptop;
  const int32_t sper = (spans + CL - 1) / CL;
  const int32_t t_b = (int32_t)imin64(prm.N, (int64_t)rank * sper * Ptop);
  const int32_t t_e = (int32_t)imin64(prm.N, (int64_t)t_b + (int64_t)sper * Ptop);
  // level l: entries jb[l] .. jb[l] + nl[l] - 1, cached at skey[kb[l] ..]
  int32_t jb[kMaxLevels], nl[kMaxLevels], kb[kMaxLevels];
  int32_t nk = 0;
#pragma unroll
  for (int l = 0; l < kMaxLevels; ++l) {
    jb[l] = l < prm.L ? t_b / prm.pw[l] : 0;
    nl[l] = l < prm.L ? (t_e - t_b) / prm.pw[l] : 0;
    kb[l] = nk;
    nk += nl[l];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the CTA's key range fits the cache it was sized for, and its entries lie in the unit
  const bool range_ok = LH_CHECK(!cached || nk <= (int32_t)kcap, kBoundsTopk) &&
                        LH_CHECK(dbg::rows_ok(prm.off[0] + jb[0], nl[0], prm.M), kBoundsTopk);
  if (cached && range_ok) {
#pragma unroll
    for (int l = 0; l < kMaxLevels; ++l) {
      const uint32_t* src = key + prm.off[l] + jb[l];
      const bool top = prm.keep_top && l == prm.L - 1;
#pragma unroll 4
      for (int32_t j = threadIdx.x; j < nl[l]; j += kThreads)
        skey[kb[l] + j] = top ? kTopBits : __ldg(src + j);
    }
  }
  auto key_of = [&](int l, int32_t j) -> uint32_t {  // j: index within the CTA's level-l range
    if (cached) return skey[kb[l] + j];
    return (prm.keep_top && l == prm.L - 1) ? kTopBits : __ldg(key + prm.off[l] + jb[l] + j);
  };

  cluster.sync();  // every CTA is running (DSMEM) and its keys are in place

  // ---- 1. threshold score by radix select on the key bits (descending)
  uint32_t prefix = 0, pmask = 0, need = (uint32_t)prm.S, ties = 0;
  int buf = 0;
  // digits of the 32 key bits, high to low: [21,32), [10,21), [0,10)
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < kBins; i += kThreads) hist[buf][i] = 0;
    __syncthreads();
    if (cached) {
      // the level does not matter here: one flat pass over the CTA's keys, four
      // per 16-byte shared-memory load (the tail, nk % 4 keys, one by one)
      const int32_t nq = nk >> 2;
      for (int32_t i0 = warp * 32; i0 < nq; i0 += kThreads) {  // warp-uniform trip count
        const int32_t i = i0 + lane;
        const uint4 k4 = i < nq ? reinterpret_cast<const uint4*>(skey)[i] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool act = i < nq && (kk[e] & pmask) == prefix;
          if (pass == 0)
            hist_add(hist[buf], act, (kk[e] >> shift) & dmask);
          else
            hist_add_plain(hist[buf], act, (kk[e] >> shift) & dmask);
        }
      }
      for (int32_t i = 4 * nq + (int32_t)threadIdx.x; i < nk; i += kThreads) {
        const uint32_t kv = skey[i];
        if ((kv & pmask) == prefix) atomicAdd(&hist[buf][(kv >> shift) & dmask], 1u);
      }
    } else {
#pragma unroll
      for (int l = 0; l < kMaxLevels; ++l) {
        for (int32_t j0 = warp * 32; j0 < nl[l]; j0 += kThreads) {  // warp-uniform trip count
          const int32_t j = j0 + lane;
          const uint32_t kv = j < nl[l] ? key_of(l, j) : 0u;
          const bool act = j < nl[l] && (kv & pmask) == prefix;
          if (pass == 0)
            hist_add(hist[buf], act, (kv >> shift) & dmask);
          else
            hist_add_plain(hist[buf], act, (kv >> shift) & dmask);
        }
      }
    }
    cluster.sync();
    Pick pk = pick_digit<CL>(cluster, hist[buf], nb, true, need, warp_buf, sh);
    prefix |= pk.bin << shift;
    pmask |= dmask << shift;
    need -= pk.before;
    ties = pk.inbin;
    buf ^= 1;
  }
  const uint32_t T = prefix;

  // ---- 2. among entries scoring exactly T, the need smallest gids
  int64_t gid_thr = INT64_MAX;
  if (need < ties && ties <= (uint32_t)kTieCap) {
    // Few ties (the usual case: one max-inheritance chain, at most L entries):
    // each CTA lists the gids of its keys equal to T, every CTA reads the
    // cluster's lists through DSMEM and takes the need-th smallest directly.
    if (threadIdx.x == 0) tie_n = 0;
    __syncthreads();
    auto add_tie = [&](uint32_t gid) {
      const uint32_t k = atomicAdd(&tie_n, 1u);
      if (k < (uint32_t)kTieCap) tie_gid[k] = gid;
    };
    if (cached) {
      for (int32_t i = (int32_t)threadIdx.x; i < nk; i += kThreads) {
        if (skey[i] != T) continue;
        int32_t gb = prm.off[0] + jb[0] - kb[0];
#pragma unroll
        for (int l = 1; l < kMaxLevels; ++l)
          if (l < prm.L && i >= kb[l]) gb = prm.off[l] + jb[l] - kb[l];
        add_tie((uint32_t)(gb + i));
      }
    } else {
#pragma unroll
      for (int l = 0; l < kMaxLevels; ++l)
        for (int32_t j = (int32_t)threadIdx.x; j < nl[l]; j += kThreads)
          if (key_of(l, j) == T) add_tie((uint32_t)(prm.off[l] + jb[l] + j));
    }
    cluster.sync();  // every CTA's list is complete
    // the cluster's ties, CTA by CTA (their total is `ties`, at most kTieCap)
    if (threadIdx.x < (unsigned)ties) {
      uint32_t i = threadIdx.x;
      int r = 0;
      for (; r < CL; ++r) {
        const uint32_t nr = *cluster.map_shared_rank(&tie_n, r);
        if (i < nr) break;
        i -= nr;
      }
      all_tie[threadIdx.x] = r < CL ? cluster.map_shared_rank(tie_gid, r)[i] : 0xffffffffu;
    }
    __syncthreads();
    if (threadIdx.x < (unsigned)ties) {  // gids are distinct: exactly one has rank need - 1
      const uint32_t gme = all_tie[threadIdx.x];
      uint32_t rank = 0;
      for (uint32_t j = 0; j < ties; ++j) rank += all_tie[j] < gme ? 1u : 0u;
      if (rank == need - 1) sh[3] = gme;
    }
    __syncthreads();
    gid_thr = (int64_t)sh[3];
    need = 0;
  } else if (need < ties) {
    int nbits = 1;
    while (nbits < 31 && ((int64_t)1 << nbits) < prm.M) ++nbits;
    uint32_t gprefix = 0, gmask = 0;
    for (int hi = nbits; hi > 0;) {
      const int w = hi >= 11 ? 11 : hi;
      const int shift = hi - w;
      const int nb = 1 << w;
      const uint32_t dmask = (uint32_t)nb - 1u;
      for (int i = threadIdx.x; i < kBins; i += kThreads) hist[buf][i] = 0;
      __syncthreads();
      if (cached) {
        // flat over the cached keys; a key at position i of level l has gid
        // off[l] + jb[l] + (i - kb[l]), the level found by comparing i with kb[]
        for (int32_t i = (int32_t)threadIdx.x; i < nk; i += kThreads) {
          if (skey[i] != T) continue;
          int32_t gb = prm.off[0] + jb[0] - kb[0];
#pragma unroll
          for (int l = 1; l < kMaxLevels; ++l)
            if (l < prm.L && i >= kb[l]) gb = prm.off[l] + jb[l] - kb[l];
          const uint32_t gid = (uint32_t)(gb + i);
          if ((gid & gmask) == gprefix) atomicAdd(&hist[buf][(gid >> shift) & dmask], 1u);
        }
      } else {
#pragma unroll
        for (int l = 0; l < kMaxLevels; ++l) {
          for (int32_t j0 = warp * 32; j0 < nl[l]; j0 += kThreads) {
            const int32_t j = j0 + lane;
            const uint32_t gid = (uint32_t)(prm.off[l] + jb[l] + j);
            const bool in = j < nl[l] && key_of(l, j < nl[l] ? j : 0) == T && (gid & gmask) == gprefix;
            hist_add_plain(hist[buf], in, (gid >> shift) & dmask);
          }
        }
      }
      cluster.sync();
      // pick_digit needs nbins to be a multiple of the thread count or equal to
      // 1024/2048; smaller digit widths are padded with empty bins.
      const int nbp = nb < kThreads ? kThreads : nb;
      Pick pk = pick_digit<CL>(cluster, hist[buf], nbp, false, need, warp_buf, sh);
      gprefix |= pk.bin << shift;
      gmask |= dmask << shift;
      need -= pk.before;
      buf ^= 1;
      hi = shift;
    }
    gid_thr = (int64_t)gprefix;
  }

  // ---- 3. ordered compaction over (token, level) of the CTA's tokens
  const int32_t wper = ((t_e - t_b + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int32_t w_begin = (int32_t)imin64(t_e, (int64_t)t_b + (int64_t)warp * wper);
  const int32_t w_end = (int32_t)imin64(t_e, (int64_t)w_begin + wper);
  // level-l entry whose span ends at token t (t1 = t + 1, requires ends_at)
  auto selected = [&](int l, uint32_t t1) -> bool {
    const int32_t g = gid_at(prm, t1, l);
    const uint32_t kv = key_of(l, g - prm.off[l] - jb[l]);
    return kv > T || (kv == T && (int64_t)g <= gid_thr);
  };
  // pass A: per token, which levels end at it and which of those are selected
  // (kept for pass B); counts per warp
  uint32_t wcount = 0;
  for (int32_t tb = w_begin; tb < w_end; tb += 32) {
    const int32_t t = tb + lane;
    uint32_t c = 0;
    if (t < w_end) {
      const uint32_t t1 = (uint32_t)t + 1u;
      uint32_t mask = 0;
#pragma unroll
      for (int l = 0; l < kMaxLevels; ++l) {  // unrolled: jb[l], kb[l] stay in registers
        if (l >= prm.L || !ends_at(prm, t1, l)) break;  // spans end at t up to some level
        mask |= (selected(l, t1) ? 1u : 0u) << l | 1u << (8 + l);
      }
      if (masks) smask[t - t_b] = (uint16_t)mask;
      c = __popc(mask & 0xffu);
    }
    wcount += __reduce_add_sync(0xffffffffu, c);
  }
  if (lane == 0) warp_tot[warp] = wcount;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_tot[lane];
    uint32_t wi = warp_incl_scan(w);
    warp_tot[lane] = wi - w;
    if (lane == 31) cta_total = wi;
  }
  cluster.sync();
  uint32_t base = 0;
  for (int r = 0; r < rank; ++r) base += *cluster.map_shared_rank(&cta_total, r);
  base += warp_tot[warp];
  // pass B: write idx, pos and the slot map from the masks
  int32_t* idx_u = idx + u * prm.S;
  int32_t* pos_u = pos + u * prm.S;
  int32_t* slot_u = slot + u * prm.M;
  for (int32_t tb = w_begin; tb < w_end; tb += 32) {
    const int32_t t = tb + lane;
    uint32_t mask = 0;
    if (t < w_end) {
      if (masks) {
        mask = smask[t - t_b];
      } else {  // masks did not fit in shared memory: recompute them
        const uint32_t t1 = (uint32_t)t + 1u;
#pragma unroll
        for (int l = 0; l < kMaxLevels; ++l) {
          if (l >= prm.L || !ends_at(prm, t1, l)) break;
          mask |= (selected(l, t1) ? 1u : 0u) << l | 1u << (8 + l);
        }
      }
    }
    const uint32_t c = __popc(mask & 0xffu);
    const uint32_t incl = warp_incl_scan(c);
    uint32_t k = base + incl - c;
    const uint32_t t1 = (uint32_t)t + 1u;
#pragma unroll
    for (int l = 0; l < kMaxLevels; ++l) {
      if (!((mask >> (8 + l)) & 1u)) break;
      const int32_t g = gid_at(prm, t1, l);
      if (!LH_CHECK(dbg::in_range(g, prm.M), kBoundsTopk)) break;
      if ((mask >> l) & 1u) {
        if (LH_CHECK(dbg::in_range(k, prm.S), kBoundsTopk)) {
          idx_u[k] = (int32_t)g;
          pos_u[k] = (int32_t)t;
          slot_u[g] = (int32_t)k;
        }
        ++k;
      } else {
        slot_u[g] = -1;
      }
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  cluster.sync();  // keep shared memory alive until every remote read is done
}

}  // namespace

struct SmemPlan {
  int cached, masks, kcap;
  size_t dyn;
};

// How many clusters of C CTAs (dyn bytes of dynamic shared memory each) this
// device runs at once; 0 when the query fails.
template <int C>
int max_active_clusters(size_t dyn) {
  auto* kf = k_topk<C>;
  if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t q = {};
  q.gridDim = dim3((unsigned)C, 1, 1);
  q.blockDim = dim3(kThreads, 1, 1);
  q.dynamicSmemBytes = dyn;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeClusterDimension;
  a[0].val.clusterDim.x = (unsigned)C;
  a[0].val.clusterDim.y = 1;
  a[0].val.clusterDim.z = 1;
  q.attrs = a;
  q.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kf, &q) != cudaSuccess) n = 0;
  (void)cudaGetLastError();
  return n;
}

cudaError_t launch_topk(const Geom& g, const float* score, int32_t* idx, int32_t* pos,
                        int32_t* slot, cudaStream_t st) {
  TopkParams prm;
  prm.N = (int32_t)g.N;
  prm.M = (int32_t)g.M;
  prm.p = g.p;
  prm.L = g.L;
  prm.S = g.S;
  prm.log2p = ((g.p & (g.p - 1)) == 0) ? __builtin_ctz((unsigned)g.p) : -1;
  prm.keep_top = g.keep_top;
  for (int l = 0; l <= kMaxLevels; ++l) {
    prm.off[l] = (int32_t)g.off[l];
    prm.pw[l] = (int32_t)(g.pw[l] > 0x7fffffff ? 0x7fffffff : g.pw[l]);
  }
  // Larger clusters for larger units: more SMs per unit, same barrier count.
  // A 16-CTA cluster is a non-portable size; it is used only when this device
  // can hold one (checked once per device).
  int CL = 8;
  if (g.M > ((int64_t)1 << 19)) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    static std::atomic<int> ok16[64];  // 0 unknown, 1 yes, 2 no
    int state = dev < 64 ? ok16[dev].load() : 2;
    if (state == 0) {
      state = 2;
      if (cudaFuncSetAttribute(k_topk<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(16, 1, 1);
        q.blockDim = dim3(kThreads, 1, 1);
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeClusterDimension;
        a[0].val.clusterDim.x = 16;
        a[0].val.clusterDim.y = 1;
        a[0].val.clusterDim.z = 1;
        q.attrs = a;
        q.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, k_topk<16>, &q) == cudaSuccess &&
            nclusters > 0)
          state = 1;
      }
      (void)cudaGetLastError();
      ok16[dev].store(state);
    }
    if (state == 1) CL = 16;
  }
  // keys of one CTA: whole coarsest spans, every level.  Shared memory holds
  // the CTA's keys if they fit (every pass reads them), and the per-token masks
  // of the compaction only if both fit (else pass B recomputes them, cheaply,
  // from the cached keys).
  const int64_t Ptop = g.pw[g.L - 1];
  const int64_t spans = g.N / Ptop;
  int64_t per_span = 0;
  for (int l = 0; l < g.L; ++l) per_span += Ptop / g.pw[l];
  const auto plan = [&](int cl) -> SmemPlan {
    const int64_t sper = (spans + cl - 1) / cl;
    const int64_t key_bytes = sper * per_span * 4;
    int64_t mask_bytes = (sper * Ptop * 2 + 15) / 16 * 16;  // 16 bits per token
    SmemPlan sp;
    sp.cached = key_bytes <= kKeyCacheBytes ? 1 : 0;
    sp.masks = (sp.cached ? key_bytes : 0) + mask_bytes <= kKeyCacheBytes ? 1 : 0;
    if (!sp.masks) mask_bytes = 0;
    sp.kcap = sp.cached ? (int)(key_bytes / 4) : 0;
    sp.dyn = (size_t)sp.kcap * 4 + (size_t)mask_bytes;
    return sp;
  };
  if (CL == 8) {
    // A unit is one cluster, and a cluster runs on one GPC: when the device
    // holds fewer clusters of 8 at once than there are units, a second wave of
    // clusters doubles the time.  Smaller clusters fit more at once, each CTA
    // with proportionally more keys: take the size with the fewest waves per
    // CTA of work, ceil(units / clusters at once) / CL, among those that keep
    // the keys in shared memory when 8 does (ties to the larger cluster).
    const int64_t units = g.U < 65535 ? g.U : 65535;
    const SmemPlan p8 = plan(8);
    double best = -1.0;
    int best_cl = 8;
    const int cands[3] = {8, 6, 4};
    for (int c : cands) {
      const SmemPlan pc = plan(c);
      if (p8.cached && !pc.cached) continue;
      const int fit = c == 8 ? max_active_clusters<8>(pc.dyn)
                             : (c == 6 ? max_active_clusters<6>(pc.dyn) : max_active_clusters<4>(pc.dyn));
      if (fit <= 0) continue;
      const double cost = (double)((units + fit - 1) / fit) / (double)c;
      if (best < 0.0 || cost < best) {
        best = cost;
        best_cl = c;
      }
    }
    CL = best_cl;
  }
  const SmemPlan sp = plan(CL);
  const int cached = sp.cached, masks = sp.masks, kcap = sp.kcap;
  const size_t dyn = sp.dyn;
  auto launch = [&](auto clc) -> cudaError_t {
    constexpr int C = decltype(clc)::value;
    auto* kf = k_topk<C>;
    cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return e;
    if (C > 8 && (e = cudaFuncSetAttribute(kf, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) !=
                     cudaSuccess)
      return e;
    for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
      prm.unit0 = u0;
      const int64_t nu = g.U - u0 < 65535 ? g.U - u0 : 65535;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)C, (unsigned)nu, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = dyn;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)C;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, kf, score, idx, pos, slot, prm, cached, kcap, masks);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  };
  switch (CL) {
    case 16: return launch(std::integral_constant<int, 16>{});
    case 6: return launch(std::integral_constant<int, 6>{});
    case 4: return launch(std::integral_constant<int, 4>{});
    default: return launch(std::integral_constant<int, 8>{});
  }
}


// ================================================== device-wide pass selection
// The same selection and slots as k_topk, as a sequence of short kernels over
// all SMs instead of one thread-block cluster per unit (a unit's passes then run
// on every SM, not on one GPC's; large units need no second wave of clusters).
// State between the kernels lives in a per-unit workspace (zeroed first):
//   hist[3][2048]  the three digit histograms of the key bits (high to low),
//   st[16]         the radix state after each digit and the threshold (kSt*),
//   tie_n, tie[kSelTies]  gids of the keys equal to the threshold, if needed,
//   cnt[nbt]       selected entries per token block (for the slot offsets).
// Every kernel takes a warp-uniform view of the same integers, so the result is
// the cluster kernel's, bit for bit.
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelKeys = 16384;    // keys per CTA of a histogram pass
constexpr int kSelTokens = 8192;   // tokens per CTA of the count / write passes
constexpr int kSelTies = 4096;     // ties at the threshold resolved from a list
// state words: after digit 0 (written by pass 1), after digit 1 (pass 2), the
// threshold (tie pass) and the largest tie gid that fits (resolve)
enum : int {
  kSt1Prefix = 0, kSt1Mask, kSt1Need, kSt2Prefix, kSt2Mask, kSt2Need, kStT, kStNeed, kStTies, kStGid,
  kStCount = 16
};
constexpr int kWsHist = 0, kWsSt = 3 * kBins, kWsTieN = kWsSt + kStCount, kWsTie = kWsTieN + 8,
              kWsCnt = kWsTie + kSelTies;

struct SelPrm {
  TopkParams t;
  int32_t stride;  // workspace words per unit
  int32_t nbk;     // CTAs per unit of a histogram pass
  int32_t nbt;     // CTAs per unit of the count / write passes
  int32_t top;     // first gid of the coarsest level (ranked +inf when kept)
};

// Programmatic dependent launch: each pass is launched while the one before it
// drains; it waits here until that pass has completed (its writes visible), then
// lets the next pass be launched.  Both are no-ops for an ordinary launch.
__device__ __forceinline__ void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t sel_key(const SelPrm& sp, const uint32_t* key, int32_t g) {
  return (sp.t.keep_top && g >= sp.top) ? kTopBits : __ldg(key + g);
}

// Block-wide exclusive scan (kSelThreads threads) of one value per thread.
__device__ uint32_t sel_excl_scan(uint32_t v, uint32_t* warp_buf, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t incl = warp_incl_scan(v);
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = warp_buf[lane];
    const uint32_t wi = warp_incl_scan(w);
    warp_buf[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const uint32_t r = warp_buf[warp] + incl - v;
  __syncthreads();
  return r;
}

// The digit of a (global) histogram of nb bins where the need-th key falls,
// counting from the largest digit (descending) or the smallest.
__device__ Pick sel_pick(const uint32_t* hist, int nb, bool descending, uint32_t need,
                         uint32_t* warp_buf, uint32_t* sh) {
  const int per = nb / kSelThreads;  // 2 or 1
  uint32_t c[2] = {0, 0};
  for (int i = 0; i < per; ++i) {
    const int ord = (int)threadIdx.x * per + i;
    c[i] = __ldcg(hist + (descending ? nb - 1 - ord : ord));
  }
  uint32_t all;
  uint32_t before = sel_excl_scan(c[0] + c[1], warp_buf, &all);
  for (int i = 0; i < per; ++i) {
    const int ord = (int)threadIdx.x * per + i;
    if (before < need && need <= before + c[i]) {
      sh[0] = (uint32_t)(descending ? nb - 1 - ord : ord);
      sh[1] = before;
      sh[2] = c[i];
    }
    before += c[i];
  }
  __syncthreads();
  const Pick pk{sh[0], sh[1], sh[2]};
  __syncthreads();
  return pk;
}

// Histogram pass PASS (0, 1, 2: key bits [21,32), [10,21), [0,10)) over keys
// [b kSelKeys, (b+1) kSelKeys) of unit u, among the keys matching the digits
// chosen so far.  PASS 1 picks digit 0 from hist[0] (CTA 0 records the state);
// PASS 2 reads that state and picks digit 1 from hist[1].
template <int PASS>
__global__ void __launch_bounds__(kSelThreads) k_sel_hist(const float* __restrict__ score,
                                                          uint32_t* __restrict__ ws, const SelPrm sp) {
  pdl_wait_then_release();
  __shared__ uint32_t h[kBins];
  __shared__ uint32_t warp_buf[32], sh[4];
  const int64_t u = sp.t.unit0 + blockIdx.y;
  uint32_t* w = ws + (int64_t)blockIdx.y * sp.stride;
  const uint32_t* key = reinterpret_cast<const uint32_t*>(score + u * sp.t.M);
  constexpr int shift = PASS == 0 ? 21 : (PASS == 1 ? 10 : 0);
  constexpr uint32_t dmask = PASS == 2 ? 1023u : 2047u;
  uint32_t prefix = 0, pmask = 0, need = (uint32_t)sp.t.S;
  if (PASS == 1) {
    const Pick pk = sel_pick(w + kWsHist, 2048, true, need, warp_buf, sh);
    prefix = pk.bin << 21;
    pmask = 2047u << 21;
    need -= pk.before;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      w[kWsSt + kSt1Prefix] = prefix;
      w[kWsSt + kSt1Mask] = pmask;
      w[kWsSt + kSt1Need] = need;
    }
  } else if (PASS == 2) {
    prefix = __ldcg(w + kWsSt + kSt1Prefix);
    pmask = __ldcg(w + kWsSt + kSt1Mask);
    need = __ldcg(w + kWsSt + kSt1Need);
    const Pick pk = sel_pick(w + kWsHist + kBins, 2048, true, need, warp_buf, sh);
    prefix |= pk.bin << 10;
    pmask |= 2047u << 10;
    need -= pk.before;
    if (blockIdx.x == 0 && threadIdx.x == 0) {  // the state after two digits (read by the tie pass)
      w[kWsSt + kSt2Prefix] = prefix;
      w[kWsSt + kSt2Mask] = pmask;
      w[kWsSt + kSt2Need] = need;
    }
  }
  for (int i = threadIdx.x; i < kBins; i += kSelThreads) h[i] = 0;
  __syncthreads();
  const int32_t i0 = (int32_t)blockIdx.x * kSelKeys;
  const int32_t i1 = (int32_t)imin64(sp.t.M, (int64_t)i0 + kSelKeys);
  // keys up to the first 16-byte boundary one by one, then four per load (all of
  // a thread's loads in flight at once), then the tail
  const int32_t head = (int32_t)((4 - ((u * sp.t.M + i0) & 3)) & 3);
  const int32_t q0 = (int32_t)imin64(i1, (int64_t)i0 + head);
  const int32_t nq = (i1 - q0) >> 2;
  auto one = [&](int32_t j) {
    const uint32_t kv = sel_key(sp, key, j);
    if ((kv & pmask) == prefix) atomicAdd(&h[(kv >> shift) & dmask], 1u);
  };
  for (int32_t j = i0 + (int32_t)threadIdx.x; j < q0; j += kSelThreads) one(j);
  for (int32_t j = q0 + 4 * nq + (int32_t)threadIdx.x; j < i1; j += kSelThreads) one(j);
  const uint4* kq = reinterpret_cast<const uint4*>(key + q0);
#pragma unroll 4
  for (int32_t b0 = (int32_t)(threadIdx.x & ~31u); b0 < nq; b0 += kSelThreads) {  // warp-uniform
    const int32_t qi = b0 + (int32_t)(threadIdx.x & 31);
    const uint4 v4 = qi < nq ? __ldg(kq + qi) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t kk[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int32_t g = q0 + 4 * qi + e;
      const uint32_t kv = (sp.t.keep_top && g >= sp.top) ? kTopBits : kk[e];
      const bool act = qi < nq && (kv & pmask) == prefix;
      if (PASS == 0)
        hist_add(h, act, (kv >> shift) & dmask);
      else
        hist_add_plain(h, act, (kv >> shift) & dmask);
    }
  }
  __syncthreads();
  uint32_t* gh = w + kWsHist + PASS * kBins;
  for (int i = threadIdx.x; i < kBins; i += kSelThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
}

// The threshold T (digit 2 from hist[2]), how many keys equal to T are still
// needed and how many there are; CTA 0 records them.  When only some of the ties
// fit, every CTA lists the gids of its keys equal to T (up to kSelTies).
__global__ void __launch_bounds__(kSelThreads) k_sel_ties(const float* __restrict__ score,
                                                          uint32_t* __restrict__ ws, const SelPrm sp) {
  pdl_wait_then_release();
  __shared__ uint32_t warp_buf[32], sh[4];
  const int64_t u = sp.t.unit0 + blockIdx.y;
  uint32_t* w = ws + (int64_t)blockIdx.y * sp.stride;
  const uint32_t* key = reinterpret_cast<const uint32_t*>(score + u * sp.t.M);
  const uint32_t prefix = __ldcg(w + kWsSt + kSt2Prefix);
  uint32_t need = __ldcg(w + kWsSt + kSt2Need);
  const Pick pk = sel_pick(w + kWsHist + 2 * kBins, 1024, true, need, warp_buf, sh);
  const uint32_t T = prefix | pk.bin;
  need -= pk.before;
  const uint32_t ties = pk.inbin;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    w[kWsSt + kStT] = T;
    w[kWsSt + kStNeed] = need;
    w[kWsSt + kStTies] = ties;
  }
  if (!(need < ties)) return;
  const int32_t i0 = (int32_t)blockIdx.x * kSelKeys;
  const int32_t i1 = (int32_t)imin64(sp.t.M, (int64_t)i0 + kSelKeys);
  for (int32_t j = i0 + (int32_t)threadIdx.x; j < i1; j += kSelThreads) {
    if (sel_key(sp, key, j) != T) continue;
    const uint32_t k = atomicAdd(w + kWsTieN, 1u);
    if (k < (uint32_t)kSelTies) w[kWsTie + k] = (uint32_t)j;
  }
}

// One CTA per unit: the largest gid among the ties that still fit (the need-th
// smallest gid equal to T), or all of them.  From the list when it holds every
// tie; else radix passes on the gids over all the unit's keys (only when more
// than kSelTies entries share the threshold score).
__global__ void __launch_bounds__(kSelThreads) k_sel_resolve(const float* __restrict__ score,
                                                             uint32_t* __restrict__ ws, const SelPrm sp) {
  pdl_wait_then_release();
  __shared__ uint32_t h[kBins];
  __shared__ uint32_t warp_buf[32], sh[4];
  __shared__ uint32_t list[kSelTies];
  const int64_t u = sp.t.unit0 + blockIdx.x;
  uint32_t* w = ws + (int64_t)blockIdx.x * sp.stride;
  const uint32_t* key = reinterpret_cast<const uint32_t*>(score + u * sp.t.M);
  const uint32_t T = __ldcg(w + kWsSt + kStT);
  uint32_t need = __ldcg(w + kWsSt + kStNeed);
  const uint32_t ties = __ldcg(w + kWsSt + kStTies);
  if (!(need < ties)) {
    if (threadIdx.x == 0) w[kWsSt + kStGid] = 0x7fffffffu;  // every key equal to T fits
    return;
  }
  const bool listed = ties <= (uint32_t)kSelTies;
  if (listed)
    for (uint32_t i = threadIdx.x; i < ties; i += kSelThreads) list[i] = __ldcg(w + kWsTie + i);
  int nbits = 1;
  while (nbits < 31 && ((int64_t)1 << nbits) < sp.t.M) ++nbits;
  uint32_t gprefix = 0, gmask = 0;
  for (int hi = nbits; hi > 0;) {
    const int wd = hi >= 11 ? 11 : hi;
    const int shift = hi - wd;
    const uint32_t dmask = (1u << wd) - 1u;
    for (int i = threadIdx.x; i < kBins; i += kSelThreads) h[i] = 0;
    __syncthreads();
    if (listed) {
      for (uint32_t i = threadIdx.x; i < ties; i += kSelThreads) {
        const uint32_t gid = list[i];
        if ((gid & gmask) == gprefix) atomicAdd(&h[(gid >> shift) & dmask], 1u);
      }
    } else {
      for (int32_t j = (int32_t)threadIdx.x; j < sp.t.M; j += kSelThreads)
        if (sel_key(sp, key, j) == T && ((uint32_t)j & gmask) == gprefix)
          atomicAdd(&h[((uint32_t)j >> shift) & dmask], 1u);
    }
    __syncthreads();
    // ascending over the 2048 shared bins (digits of fewer bits leave the top empty)
    uint32_t c[2] = {h[2 * threadIdx.x], h[2 * threadIdx.x + 1]};
    uint32_t all;
    uint32_t before = sel_excl_scan(c[0] + c[1], warp_buf, &all);
    for (int i = 0; i < 2; ++i) {
      if (before < need && need <= before + c[i]) {
        sh[0] = 2 * threadIdx.x + i;
        sh[1] = before;
      }
      before += c[i];
    }
    __syncthreads();
    gprefix |= sh[0] << shift;
    gmask |= dmask << shift;
    need -= sh[1];
    __syncthreads();
    hi = shift;
  }
  if (threadIdx.x == 0) w[kWsSt + kStGid] = gprefix;
}

// Is the level-l entry g (span ending at token t) selected?
__device__ __forceinline__ bool sel_in(const SelPrm& sp, const uint32_t* key, int32_t g, uint32_t T,
                                       uint32_t gthr) {
  const uint32_t kv = sel_key(sp, key, g);
  return kv > T || (kv == T && (uint32_t)g <= gthr);
}

// Entries of level l whose span ends inside tokens [t0, t1): the level-l entry j
// spans tokens [j p^l, (j+1) p^l) and is enumerated at its last token.
__device__ __forceinline__ void level_range(const SelPrm& sp, int l, int32_t t0, int32_t t1,
                                            int32_t& j0, int32_t& j1) {
  const int32_t pw = sp.t.pw[l];
  j0 = (t0 + pw) / pw - 1;  // ceil((t0 + 1) / pw) - 1
  j1 = t1 / pw;
}

// Selected entries per block of kSelTokens tokens, level by level (every load
// independent of the others, so many are in flight at once).
__global__ void __launch_bounds__(kSelThreads) k_sel_count(const float* __restrict__ score,
                                                           uint32_t* __restrict__ ws, const SelPrm sp) {
  pdl_wait_then_release();
  __shared__ uint32_t warp_buf[32], tot;
  const int64_t u = sp.t.unit0 + blockIdx.y;
  uint32_t* w = ws + (int64_t)blockIdx.y * sp.stride;
  const uint32_t* key = reinterpret_cast<const uint32_t*>(score + u * sp.t.M);
  const uint32_t T = __ldcg(w + kWsSt + kStT), gthr = __ldcg(w + kWsSt + kStGid);
  const int32_t t0 = (int32_t)blockIdx.x * kSelTokens;
  const int32_t t1 = (int32_t)imin64(sp.t.N, (int64_t)t0 + kSelTokens);
  uint32_t c = 0;
#pragma unroll
  for (int l = 0; l < kMaxLevels; ++l) {
    if (l >= sp.t.L) break;
    int32_t j0, j1;
    level_range(sp, l, t0, t1, j0, j1);
    const int32_t gb = sp.t.off[l];
#pragma unroll 4
    for (int32_t j = j0 + (int32_t)threadIdx.x; j < j1; j += kSelThreads)
      c += sel_in(sp, key, gb + j, T, gthr) ? 1u : 0u;
  }
  sel_excl_scan(c, warp_buf, &tot);
  if (threadIdx.x == 0) w[kWsCnt + blockIdx.x] = tot;
}

// idx, pos and the slot map of a block of tokens: per token a mask of its
// selected levels (level by level into shared memory), a block scan of the
// per-token counts from the blocks before it on, then slots level by level:
// entry (t, l) takes tok_off[t] + the selected levels of t below l.
__global__ void __launch_bounds__(kSelThreads) k_sel_write(const float* __restrict__ score,
                                                           uint32_t* __restrict__ ws, int32_t* __restrict__ idx,
                                                           int32_t* __restrict__ pos, int32_t* __restrict__ slot,
                                                           const SelPrm sp) {
  pdl_wait_then_release();
  __shared__ uint32_t warp_buf[32], tot;
  __shared__ uint8_t mask[kSelTokens];
  __shared__ uint32_t tok_off[kSelTokens];
  constexpr int kPer = kSelTokens / kSelThreads;  // consecutive tokens per thread in the scan
  const int64_t u = sp.t.unit0 + blockIdx.y;
  const uint32_t* w = ws + (int64_t)blockIdx.y * sp.stride;
  const uint32_t* key = reinterpret_cast<const uint32_t*>(score + u * sp.t.M);
  const uint32_t T = __ldcg(w + kWsSt + kStT), gthr = __ldcg(w + kWsSt + kStGid);
  const int32_t t0 = (int32_t)blockIdx.x * kSelTokens;
  const int32_t t1 = (int32_t)imin64(sp.t.N, (int64_t)t0 + kSelTokens);
  // slots before this block: the counts of blocks 0..b-1
  uint32_t part = 0;
  for (int i = threadIdx.x; i < (int)blockIdx.x; i += kSelThreads) part += __ldcg(w + kWsCnt + i);
  sel_excl_scan(part, warp_buf, &tot);
  const uint32_t base = tot;
  // per-token masks, one level at a time (level l + 1 ORs into bytes level l wrote)
#pragma unroll
  for (int l = 0; l < kMaxLevels; ++l) {
    if (l >= sp.t.L) break;
    int32_t j0, j1;
    level_range(sp, l, t0, t1, j0, j1);
    const int32_t gb = sp.t.off[l], pw = sp.t.pw[l];
#pragma unroll 4
    for (int32_t j = j0 + (int32_t)threadIdx.x; j < j1; j += kSelThreads) {
      const int32_t t = (j + 1) * pw - 1 - t0;
      const uint8_t bit = sel_in(sp, key, gb + j, T, gthr) ? (uint8_t)(1u << l) : (uint8_t)0;
      if (l == 0)
        mask[t] = bit;
      else
        mask[t] |= bit;
    }
    __syncthreads();
  }
  // token offsets: kPer consecutive tokens per thread, then a block scan
  const int32_t nt = t1 - t0;
  uint32_t loc[kPer], sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int32_t t = (int32_t)threadIdx.x * kPer + i;
    loc[i] = sum;
    sum += t < nt ? (uint32_t)__popc(mask[t]) : 0u;
  }
  const uint32_t toff = base + sel_excl_scan(sum, warp_buf, &tot);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int32_t t = (int32_t)threadIdx.x * kPer + i;
    if (t < nt) tok_off[t] = toff + loc[i];
  }
  __syncthreads();
  int32_t* idx_u = idx + u * sp.t.S;
  int32_t* pos_u = pos + u * sp.t.S;
  int32_t* slot_u = slot + u * sp.t.M;
#pragma unroll
  for (int l = 0; l < kMaxLevels; ++l) {
    if (l >= sp.t.L) break;
    int32_t j0, j1;
    level_range(sp, l, t0, t1, j0, j1);
    const int32_t gb = sp.t.off[l], pw = sp.t.pw[l];
    for (int32_t j = j0 + (int32_t)threadIdx.x; j < j1; j += kSelThreads) {
      const int32_t t = (j + 1) * pw - 1 - t0;
      const uint32_t m = mask[t];
      const int32_t g = gb + j;
      if (!LH_CHECK(dbg::in_range(g, sp.t.M), kBoundsTopk)) continue;
      if ((m >> l) & 1u) {
        const uint32_t k = tok_off[t] + (uint32_t)__popc(m & ((1u << l) - 1u));
        // exactly S entries are selected, so k < S; the test is kept in every build
        if (LH_CHECK(dbg::in_range(k, sp.t.S), kBoundsTopk) && k < (uint32_t)sp.t.S) {
          idx_u[k] = g;
          pos_u[k] = t0 + t;
          slot_u[g] = (int32_t)k;
        }
      } else {
        slot_u[g] = -1;
      }
    }
  }
}

SelPrm sel_prm(const Geom& g) {
  SelPrm sp;
  TopkParams& prm = sp.t;
  prm.N = (int32_t)g.N;
  prm.M = (int32_t)g.M;
  prm.p = g.p;
  prm.L = g.L;
  prm.S = g.S;
  prm.log2p = ((g.p & (g.p - 1)) == 0) ? __builtin_ctz((unsigned)g.p) : -1;
  prm.keep_top = g.keep_top;
  prm.unit0 = 0;
  for (int l = 0; l <= kMaxLevels; ++l) {
    prm.off[l] = (int32_t)g.off[l];
    prm.pw[l] = (int32_t)(g.pw[l] > 0x7fffffff ? 0x7fffffff : g.pw[l]);
  }
  sp.top = (int32_t)g.off[g.L - 1];
  sp.nbk = (int32_t)((g.M + kSelKeys - 1) / kSelKeys);
  sp.nbt = (int32_t)((g.N + kSelTokens - 1) / kSelTokens);
  sp.stride = (kWsCnt + sp.nbt + 63) / 64 * 64;
  return sp;
}

}  // namespace

size_t topk_passes_workspace_bytes(const Geom& g) {
  return (size_t)g.U * sel_prm(g).stride * sizeof(uint32_t);
}

cudaError_t launch_topk_passes(const Geom& g, const float* score, int32_t* idx, int32_t* pos,
                               int32_t* slot, void* ws, cudaStream_t st) {
  SelPrm sp = sel_prm(g);
  uint32_t* w = static_cast<uint32_t*>(ws);
  cudaError_t e = cudaMemsetAsync(w, 0, topk_passes_workspace_bytes(g), st);
  if (e != cudaSuccess) return e;
  for (int64_t u0 = 0; u0 < g.U; u0 += 65535) {
    const unsigned nu = (unsigned)(g.U - u0 < 65535 ? g.U - u0 : 65535);
    sp.t.unit0 = u0;
    uint32_t* wu = w + u0 * sp.stride;
    const dim3 gk((unsigned)sp.nbk, nu), gt((unsigned)sp.nbt, nu);
    k_sel_hist<0><<<gk, kSelThreads, 0, st>>>(score, wu, sp);  // after the memset: ordinary launch
    // the later passes: programmatic dependent launches (see pdl_wait_then_release)
    auto pdl = [&](dim3 grid, auto kern, auto... a) -> cudaError_t {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = grid;
      cfg.blockDim = dim3(kSelThreads, 1, 1);
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, kern, a...);
    };
    if ((e = pdl(gk, k_sel_hist<1>, score, wu, sp)) != cudaSuccess) return e;
    if ((e = pdl(gk, k_sel_hist<2>, score, wu, sp)) != cudaSuccess) return e;
    if ((e = pdl(gk, k_sel_ties, score, wu, sp)) != cudaSuccess) return e;
    if ((e = pdl(dim3(nu, 1, 1), k_sel_resolve, score, wu, sp)) != cudaSuccess) return e;
    if ((e = pdl(gt, k_sel_count, score, wu, sp)) != cudaSuccess) return e;
    if ((e = pdl(gt, k_sel_write, score, wu, idx, pos, slot, sp)) != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

int topk_passes_launches(const Geom& g) { return 7 * (int)((g.U + 65534) / 65535); }

}  // namespace lh
