// lh_selftest.cu -- test hooks for device helpers of the attention kernels that
// no entry point of liblighthouse.so exposes on their own.  Built into a
// separate library (liblh_selftest.so) that only the tests load; the product
// library does not contain these entry points.
//
//   lh_selftest_ex2_fma2: evaluates ex2_fma2 (tc_common.cuh), the FMA-pipe 2^x
//   that the forward attention uses for a quarter of its exponentials, on n
//   values, so a test can hold it to its stated error bound;
//   lh_selftest_bounds: the debug build's bounds predicates (lh_internal.cuh),
//   compiled for the host, so a CPU test can feed them out-of-range indices
//   (no kernel ever gets a bad index on purpose).
#include "../csrc/tc_common.cuh"

namespace {

__global__ void k_ex2_fma2(const float* __restrict__ x, float* __restrict__ y, int64_t pairs) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= pairs) return;
  const float2 v = reinterpret_cast<const float2*>(x)[i];
  reinterpret_cast<float2*>(y)[i] = lh::tc::ex2_fma2(v);
}

}  // namespace

// x, y: device pointers to n fp32 values (n even, 8-byte aligned).  Returns 0, or
// a cudaError_t code (1 for bad arguments).
extern "C" int lh_selftest_ex2_fma2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0 || (n & 1) || (((uintptr_t)x | (uintptr_t)y) & 7u)) return 1;
  const int64_t pairs = n / 2;
  if (pairs == 0) return 0;
  const int block = 256;
  const int64_t grid = (pairs + block - 1) / block;
  if (grid > 0x7fffffff) return 1;
  k_ex2_fma2<<<(unsigned)grid, block, 0, static_cast<cudaStream_t>(stream)>>>(x, y, pairs);
  return (int)cudaGetLastError();
}

// which: 0 in_range(a, b), 1 slot_ok(a, b), 2 rows_ok(a, b, c), 3 entry_ok(a, b, c).
// Returns 1 (true), 0 (false) or -1 (unknown predicate).
extern "C" int lh_selftest_bounds(int which, int64_t a, int64_t b, int64_t c) {
  switch (which) {
    case 0: return lh::dbg::in_range(a, b) ? 1 : 0;
    case 1: return lh::dbg::slot_ok(a, b) ? 1 : 0;
    case 2: return lh::dbg::rows_ok(a, b, c) ? 1 : 0;
    case 3: return lh::dbg::entry_ok(a, b, c) ? 1 : 0;
  }
  return -1;
}
