// lh_internal.cuh -- shared definitions of the CUDA library (not part of the ABI).
#pragma once

#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/lighthouse.h"

namespace lh {

constexpr int kMaxLevels = 8;

// Per-unit geometry derived from an lh_shape (host and device).
struct Geom {
  int64_t U;      // B * H independent units
  int64_t N;      // tokens
  int64_t M;      // pyramid entries per unit
  int d, p, L, S;
  int64_t pw[kMaxLevels + 1];   // p^l
  int64_t off[kMaxLevels + 1];  // first gid of level l; off[L] = M
  int score_mode = 0;           // lh_score_mode
  int keep_top = 0;             // keep every level-(L-1) entry (lh_options.keep_coarsest)
  int scatter_mode = 0;         // lh_scatter_mode
};

Geom make_geom(const lh_shape& s);

// ---------------------------------------------------------------- device status
// One word per device, set by kernels whose bounded waits give up and read and
// cleared by lh_read_device_status.  It lives in the translation unit of the
// kernels that wait (k_attn_tc.cu); this reads and clears it (synchronous).
cudaError_t device_status_read_clear(uint32_t* value);
// The word of the kernels that write the fp16 sub-sequence from caller data
// (gather, scatter-back adjoint; k_gather_scatter.cu), read and cleared alike.
cudaError_t subseq_status_read_clear(uint32_t* value);

// Bits of the status words (LH_STATUS_* in lighthouse.h).
enum : uint32_t {
  kStatusAttnFwdTimeout = 0x100,
  kStatusAttnBwdTimeout = 0x200,
  kStatusFp16Saturated = 0x400,
  kStatusBounds = 0x800,  // a bounds check of the debug build failed (kernel bit below)
  kBoundsPyramid = 1u << 16,
  kBoundsTopk = 1u << 17,
  kBoundsGather = 1u << 18,
  kBoundsScatter = 1u << 19,
  kBoundsScatterBwd = 1u << 20,
  kBoundsGatherBwd = 1u << 21,
  kBoundsAttnFwd = 1u << 22,
  kBoundsAttnBwd = 1u << 23,
  kBoundsAttnStats = 1u << 24,
};
// Status words of the other kernel files (each file's kernels report into a
// word of their own; lh_read_device_status reads and clears all of them).
cudaError_t pyramid_status_read_clear(uint32_t* value);
cudaError_t topk_status_read_clear(uint32_t* value);
cudaError_t mma_status_read_clear(uint32_t* value);

// ---------------------------------------------------------------- debug build
// Compiled with -DLH_DEBUG=1 (liblighthouse_debug.so), every global or shared
// memory access whose index comes from data (idx, pos, slot) or from unit, tile
// and level coordinates is preceded by a check; a failed check ORs
// kStatusBounds and the kernel's bit into the status word of its file and the
// access is skipped (no trap, no assert).  In the normal build LH_CHECK is the
// constant true and the checks compile to nothing.
#ifndef LH_DEBUG
#define LH_DEBUG 0
#endif

namespace dbg {
// 0 <= v < n
__host__ __device__ constexpr bool in_range(int64_t v, int64_t n) { return v >= 0 && v < n; }
// a slot-map entry: -1 (not selected) or a row of the sub-sequence, 0 <= s < S
__host__ __device__ constexpr bool slot_ok(int64_t s, int64_t S) { return s >= -1 && s < S; }
// rows [first, first + count) inside [0, n)
__host__ __device__ constexpr bool rows_ok(int64_t first, int64_t count, int64_t n) {
  return first >= 0 && count >= 0 && first <= n && count <= n - first;
}
// entry j of level l of a unit: off[l] <= off[l] + j < off[l + 1]
__host__ __device__ constexpr bool entry_ok(int64_t j, int64_t off_l, int64_t off_next) {
  return j >= 0 && off_l + j < off_next;
}
}  // namespace dbg

__device__ __forceinline__ bool dbg_report(bool ok, uint32_t bits, uint32_t* word) {
  if (!ok) atomicOr(word, kStatusBounds | bits);
  return ok;
}
// LH_CHECK(ok, bits) with LH_STATUS_WORD naming the file's status word.
#if LH_DEBUG
#define LH_CHECK(ok, bits) (::lh::dbg_report((ok), (bits), &LH_STATUS_WORD))
#else
#define LH_CHECK(ok, bits) true
#endif

__device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// Programmatic dependent launch.  The stage kernels are launched with
// launch_pdl, which lets the GPU start a grid while the one before it in the
// stream drains; each such kernel first waits (pdl_enter) until the grid before
// it has completed and its writes are visible -- the order of an ordinary launch
// -- and then releases the grid after it.  For an ordinary launch both
// instructions are no-ops.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// f(std::integral_constant<int, i>) for i = I .. N-1: a loop whose index is a
// compile-time constant in the body (register arrays stay in registers, powers
// and divisions by them fold), whether or not the compiler would unroll it.
template <int I, int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (I < N) {
    f(std::integral_constant<int, I>{});
    static_for<I + 1, N>(f);
  }
}

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Largest finite fp16; the sub-sequence saturates there instead of overflowing.
constexpr float kHalfMax = 65504.0f;

__device__ __forceinline__ float h_lo(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
}
__device__ __forceinline__ float h_hi(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_h2_sat(float lo, float hi) {
  return pack_h2(fminf(fmaxf(lo, -kHalfMax), kHalfMax), fminf(fmaxf(hi, -kHalfMax), kHalfMax));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&h);
}

// Load 8 consecutive elements of a row as fp32 (bf16 widening is exact).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
  uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// Streaming variant for data read exactly once (keeps L2 for reused data).
__device__ __forceinline__ void load8_stream(const __nv_bfloat16* p, float (&x)[8]) {
  uint4 w = __ldcs(reinterpret_cast<const uint4*>(p));
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void load8_stream(const float* p, float (&x)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void load8(const __half* p, float (&x)[8]) {
  uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
  x[0] = h_lo(w.x); x[1] = h_hi(w.x);
  x[2] = h_lo(w.y); x[3] = h_hi(w.y);
  x[4] = h_lo(w.z); x[5] = h_hi(w.z);
  x[6] = h_lo(w.w); x[7] = h_hi(w.w);
}
// fp16 store that saturates at +-65504 (never writes inf).  `sat` gets 1 when
// a finite value beyond that range was clipped (non-finite values are not
// counted: results from non-finite inputs are unspecified anyway).
__device__ __forceinline__ void store8_h(__half* p, const float (&x)[8], uint32_t& sat) {
  uint4 w;
  w.x = pack_h2_sat(x[0], x[1]);
  w.y = pack_h2_sat(x[2], x[3]);
  w.z = pack_h2_sat(x[4], x[5]);
  w.w = pack_h2_sat(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = w;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = fabsf(x[i]);
    sat |= (a > kHalfMax && a < INFINITY) ? 1u : 0u;
  }
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&x)[8]) {
  uint4 w;
  w.x = pack_bf16(x[0], x[1]);
  w.y = pack_bf16(x[2], x[3]);
  w.z = pack_bf16(x[4], x[5]);
  w.w = pack_bf16(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = w;
}
__device__ __forceinline__ void store8(float* p, const float (&x)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void store8_stream(__nv_bfloat16* p, const float (&x)[8]) {
  uint4 w;
  w.x = pack_bf16(x[0], x[1]);
  w.y = pack_bf16(x[2], x[3]);
  w.z = pack_bf16(x[4], x[5]);
  w.w = pack_bf16(x[6], x[7]);
  __stcs(reinterpret_cast<uint4*>(p), w);
}
__device__ __forceinline__ void store8_stream(float* p, const float (&x)[8]) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
}

// x / c rounded to nearest fp32, for an integer 1 <= c < 2^20, as one fp64
// product with inv_c = 1/c (rounded to fp64) rounded once to fp32.  It is the
// correctly rounded quotient: with c = 2^a c' (c' odd) and the quotient
// measured in half-ulps, x / c' = N / c' for an even integer N, so it is never
// a rounding midpoint and lies at least 1/c' > 2^-20 half-ulps from one, while
// the fp64 product is within 2^-52 relative (< 2^-28 ulp) of the quotient.
__device__ __forceinline__ float div_exact(float x, double inv_c) {
  return __double2float_rn((double)x * inv_c);
}

// x / c rounded to nearest fp32 for a small integer c, in fp32 FMAs only (no
// fp64 conversions, which run on the narrow conversion pipe): q = x*y with
// y = 1/c rounded to fp32, the residual r = q*c - x is exact under FMA, and
// q - r*y is the correctly rounded quotient -- Markstein's correction step
// (P. W. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Develop. 34(1), 1990).  Checked
// exhaustively against IEEE division for c = 1..8 and every finite fp32 x
// with |x| >= 2^-123 (below that, c = 6 can miss by an ulp of a subnormal);
// a zero quotient may differ in its sign.
__device__ __forceinline__ float div_small(float x, float c, float y) {
  const float q = x * y;
  const float r = fmaf(q, c, -x);
  return fmaf(-r, y, q);
}

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; arguments are already checked.
cudaError_t launch_pyramid_score(const Geom& g, lh_dtype dt, const void* q, const void* k,
                                 const void* v, float* pq, float* pk, float* pv, float* score,
                                 cudaStream_t st);
int pyramid_launches(const Geom& g, lh_dtype dt);  // kernel launches of one launch_pyramid_score
cudaError_t launch_topk(const Geom& g, const float* score, int32_t* idx, int32_t* pos,
                        int32_t* slot, cudaStream_t st);
// The same selection as device-wide passes over a workspace of
// topk_passes_workspace_bytes(g) (zeroed here, on the stream).
size_t topk_passes_workspace_bytes(const Geom& g);
cudaError_t launch_topk_passes(const Geom& g, const float* score, int32_t* idx, int32_t* pos,
                               int32_t* slot, void* ws, cudaStream_t st);
int topk_passes_launches(const Geom& g);
cudaError_t launch_gather(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                          const float* pq, const float* pk, const float* pv, const int32_t* idx,
                          __half* qs, __half* ks, __half* vs, cudaStream_t st);
cudaError_t launch_scatter(const Geom& g, lh_dtype dt, const __half* os,
                           const int32_t* slot, void* o, float* inv_count, cudaStream_t st);
cudaError_t launch_scatter_bwd(const Geom& g, lh_dtype dt, const void* dO, const int32_t* slot,
                               const float* inv_count, __half* dos, cudaStream_t st);
cudaError_t launch_gather_bwd(const Geom& g, lh_dtype dt, const float* dqs, const float* dks,
                              const float* dvs, const int32_t* slot, void* dq, void* dk, void* dv,
                              cudaStream_t st);
cudaError_t launch_gather_pooled(const Geom& g, lh_dtype dt, const void* q, const void* k,
                                 const void* v, const int32_t* idx, __half* qs, __half* ks,
                                 __half* vs, cudaStream_t st);
// Backward softmax statistics in the tile-padded layout both backward
// implementations read: per unit and 128-row tile, 128 values of -lse*log2(e)
// then 128 of -rowsum(dos*os); padded rows -inf and 0.
inline size_t attn_stats_floats(const Geom& g) { return (size_t)g.U * ((g.S + 127) / 128) * 256; }
cudaError_t launch_attn_stats(const Geom& g, const __half* os, const __half* dos,
                              const float* lse, float* stats, cudaStream_t st);

// Attention: two implementations with the same contract.
cudaError_t launch_attn_fwd_mma(const Geom& g, const __half* qs, const __half* ks,
                                const __half* vs, float scale, __half* os,
                                float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_mma(const Geom& g, const __half* qs, const __half* ks,
                                const __half* vs, const __half* dos, const float* stats,
                                float scale, float* dqs, float* dks, float* dvs, cudaStream_t st);
// full = 1: a query block against a whole earlier key block of the same length
// (no causal mask; the keys past the block's end masked) -- the off-diagonal
// steps of ring attention; full = 0: causal attention within one sequence.
cudaError_t launch_attn_fwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, float scale, __half* os,
                               float* lse, cudaStream_t st, int full = 0);
cudaError_t launch_attn_bwd_tc(const Geom& g, const __half* qs, const __half* ks,
                               const __half* vs, const __half* dos, const float* stats,
                               float scale, float* dqs, float* dks, float* dvs, cudaStream_t st,
                               int full = 0);
bool attn_tc_available();      // tcgen05 forward can run on this device
bool attn_tc_bwd_available();  // tcgen05 backward can run on this device
bool attn_fwd_uses_tc();       // dispatch decisions (lh_set_attention_impl + availability)
bool attn_bwd_uses_tc();
int attn_tc_fwd_launches(const Geom& g);
int attn_tc_bwd_launches(const Geom& g);

// The whole sub-sequence attention backward (softmax statistics into `stats`,
// attn_stats_floats(g) floats, then the gradient kernels); scale already resolved.
lh_status attn_bwd(const Geom& g, const __half* qs, const __half* ks, const __half* vs,
                   const __half* os, const float* lse, const __half* dos, float scale,
                   float* dqs, float* dks, float* dvs, float* stats, cudaStream_t st,
                   int full = 0);

}  // namespace lh
