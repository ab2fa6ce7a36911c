// lh_cp.cu -- the per-GPU pieces of context parallelism: attention of a query
// block against one key block (causal on the diagonal, full for an earlier
// block), the online merge of block results, and the accumulation of the
// block gradients that ring attention passes around.
//
// Method: [PT] bitsgeniais.com.br "Adeus Custo Quadrático! ...", section
// "Escalando para o Céu (ou 1 Milhão de Tokens!): Paralelismo de Contexto":
// each GPU builds its shard's pyramid, scores and selection locally, and the
// dense sub-sequence (the shards' sub-sequences in shard order) is attended
// with standard ring attention.  The ring itself (the order of the steps and
// the NCCL sends) lives in long_context_lh_b200/cp.py.
#include "lh_internal.cuh"

namespace lh {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// One thread per row: o_acc, lse_acc <- the softmax-weighted merge of
// (o_acc, lse_acc) and (o_part, lse_part); first: a plain copy.  A row whose two
// log-sum-exps are both -inf (no key seen yet) stays as it is.
template <int D>
__global__ void __launch_bounds__(256) k_merge(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                               const __half* __restrict__ o_part,
                                               const float* __restrict__ lse_part, int64_t rows,
                                               int first) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  float* oa = o_acc + row * D;
  const __half* op = o_part + row * D;
  const float lb = lse_part[row];
  if (first) {
#pragma unroll 4
    for (int c = 0; c < D; c += 8) {
      float x[8];
      load8(op + c, x);
      store8(oa + c, x);
    }
    lse_acc[row] = lb;
    return;
  }
  const float la = lse_acc[row];
  const float m = fmaxf(la, lb);
  if (m == -INFINITY) return;
  // weights 2^((lse - m) log2 e), normalised by their sum (one of them is 1)
  const float wa = exp2f((la - m) * kLog2e), wb = exp2f((lb - m) * kLog2e);
  const float inv = 1.0f / (wa + wb);
  const float ca = wa * inv, cb = wb * inv;
#pragma unroll 4
  for (int c = 0; c < D; c += 8) {
    float a[8], b[8];
    load8(oa + c, a);
    load8(op + c, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = fmaf(a[i], ca, b[i] * cb);
    store8(oa + c, a);
  }
  lse_acc[row] = m + log2f(wa + wb) * kLn2;
}

template <int D>
__global__ void __launch_bounds__(256) k_finish(const float* __restrict__ o_acc,
                                                __half* __restrict__ os, int64_t rows) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // chunk of 8
  if (i >= rows * (D / 8)) return;
  float x[8];
  load8(o_acc + 8 * i, x);
  uint32_t sat = 0;  // |o| <= max |v| <= 65504 for a convex combination of fp16 rows
  store8_h(os + 8 * i, x, sat);
}

__global__ void __launch_bounds__(256) k_accumulate(float* __restrict__ acc,
                                                    const float* __restrict__ x, int64_t n4) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = reinterpret_cast<float4*>(acc)[i];
  const float4 b = __ldg(reinterpret_cast<const float4*>(x) + i);
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
  reinterpret_cast<float4*>(acc)[i] = a;
}

inline bool al16(const void* p) { return p && (((uintptr_t)p) & 15u) == 0; }
inline unsigned blocks(int64_t n, int b) { return (unsigned)((n + b - 1) / b); }

lh_status block_shape_ok(const lh_shape* s) {
  lh_status st = lh_validate(s, LH_BF16);
  if (st != LH_OK) return st;
  return (int64_t)s->S == s->N ? LH_OK : LH_ERR_SHAPE;  // one block of S rows
}

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" {

lh_status lh_block_attn_fwd(const lh_shape* shape, int causal, const void* qs, const void* ks,
                            const void* vs, float scale, void* os, float* lse, lh_stream_t stream) {
  lh_status s = block_shape_ok(shape);
  if (s != LH_OK) return s;
  if (causal != 0 && causal != 1) return LH_ERR_INVALID_ARG;
  if (!al16(qs) || !al16(ks) || !al16(vs) || !al16(os) || !al16(lse)) return LH_ERR_INVALID_ARG;
  if (!causal && !attn_fwd_uses_tc()) return LH_ERR_UNSUPPORTED;
  if (causal) return lh_subseq_attn_fwd(shape, qs, ks, vs, scale, os, lse, stream);
  const Geom g = make_geom(*shape);
  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)g.d);
  return launch_attn_fwd_tc(g, static_cast<const __half*>(qs), static_cast<const __half*>(ks),
                            static_cast<const __half*>(vs), sc, static_cast<__half*>(os), lse,
                            stream, 1) == cudaSuccess
             ? LH_OK
             : LH_ERR_CUDA;
}

lh_status lh_block_attn_merge(int64_t rows, int32_t d, float* o_acc, float* lse_acc,
                              const void* o_part, const float* lse_part, int first,
                              lh_stream_t stream) {
  if (rows < 0 || (d != 64 && d != 128) || (first != 0 && first != 1)) return LH_ERR_INVALID_ARG;
  if (!al16(o_acc) || !al16(lse_acc) || !al16(o_part) || !al16(lse_part)) return LH_ERR_INVALID_ARG;
  if (rows == 0) return LH_OK;
  if (blocks(rows, 256) > 0x7fffffffu) return LH_ERR_SHAPE;
  auto* op = static_cast<const __half*>(o_part);
  if (d == 64)
    k_merge<64><<<blocks(rows, 256), 256, 0, stream>>>(o_acc, lse_acc, op, lse_part, rows, first);
  else
    k_merge<128><<<blocks(rows, 256), 256, 0, stream>>>(o_acc, lse_acc, op, lse_part, rows, first);
  return cudaGetLastError() == cudaSuccess ? LH_OK : LH_ERR_CUDA;
}

lh_status lh_block_attn_finish(int64_t rows, int32_t d, const float* o_acc, void* os,
                               lh_stream_t stream) {
  if (rows < 0 || (d != 64 && d != 128)) return LH_ERR_INVALID_ARG;
  if (!al16(o_acc) || !al16(os)) return LH_ERR_INVALID_ARG;
  if (rows == 0) return LH_OK;
  const int64_t n = rows * (d / 8);
  if (blocks(n, 256) > 0x7fffffffu) return LH_ERR_SHAPE;
  auto* o = static_cast<__half*>(os);
  if (d == 64)
    k_finish<64><<<blocks(n, 256), 256, 0, stream>>>(o_acc, o, rows);
  else
    k_finish<128><<<blocks(n, 256), 256, 0, stream>>>(o_acc, o, rows);
  return cudaGetLastError() == cudaSuccess ? LH_OK : LH_ERR_CUDA;
}

lh_status lh_block_attn_bwd(const lh_shape* shape, int causal, const void* qs, const void* ks,
                            const void* vs, const void* os, const float* lse, const void* dos,
                            float scale, float* dqs, float* dks, float* dvs, void* ws,
                            size_t ws_bytes, lh_stream_t stream) {
  lh_status s = block_shape_ok(shape);
  if (s != LH_OK) return s;
  if (causal != 0 && causal != 1) return LH_ERR_INVALID_ARG;
  if (!al16(qs) || !al16(ks) || !al16(vs) || !al16(os) || !al16(lse) || !al16(dos) ||
      !al16(dqs) || !al16(dks) || !al16(dvs))
    return LH_ERR_INVALID_ARG;
  if (ws_bytes < lh_attn_bwd_workspace_bytes(shape)) return LH_ERR_WORKSPACE;
  if (!al16(ws)) return LH_ERR_INVALID_ARG;
  const Geom g = make_geom(*shape);
  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)g.d);
  return attn_bwd(g, static_cast<const __half*>(qs), static_cast<const __half*>(ks),
                  static_cast<const __half*>(vs), static_cast<const __half*>(os), lse,
                  static_cast<const __half*>(dos), sc, dqs, dks, dvs, static_cast<float*>(ws),
                  stream, causal ? 0 : 1);
}

lh_status lh_accumulate(int64_t n, float* acc, const float* x, lh_stream_t stream) {
  if (n < 0 || (n & 3) || !al16(acc) || !al16(x)) return LH_ERR_INVALID_ARG;
  if (n == 0) return LH_OK;
  const int64_t n4 = n / 4;
  if (blocks(n4, 256) > 0x7fffffffu) return LH_ERR_SHAPE;
  k_accumulate<<<blocks(n4, 256), 256, 0, stream>>>(acc, x, n4);
  return cudaGetLastError() == cudaSuccess ? LH_OK : LH_ERR_CUDA;
}

}  // extern "C"
