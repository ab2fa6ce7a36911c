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
      ok = mbar_wait(&bars->s_full, j & 1, abort, kStatus);
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
        ok = mbar_wait(&bars->pv_done, (j - 1) & 1, abort, kStatus);
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
    if (ok) ok = mbar_wait(&bars->pv_done, (nkv - 1) & 1, abort, kStatus);
    if (ok) {
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
bool attn_tc_bwd_available() { return false; }
int attn_tc_fwd_launches(const Geom& g) { return (int)((g.U + 65534) / 65535); }
int attn_tc_bwd_launches(const Geom&) { return 0; }

cudaError_t launch_attn_fwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, float scale, __half* os, float* lse,
                               cudaStream_t st) {
  if (g.S > 0x7fffffff || g.U > 0x7fffffff) return cudaErrorInvalidValue;
  return g.d == 64 ? tc::fwd_d<64>(g, qs, ks, vs, scale, os, lse, st)
                   : tc::fwd_d<128>(g, qs, ks, vs, scale, os, lse, st);
}

cudaError_t launch_attn_bwd_tc(const Geom&, const __half*, const __half*, const __half*,
                               const __half*, const float*, const float*, float, float*, float*,
                               float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lh
