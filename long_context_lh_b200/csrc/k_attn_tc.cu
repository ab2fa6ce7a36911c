// k_attn_tc.cu -- placeholder until the tcgen05/TMEM attention kernels land.
#include "lh_internal.cuh"

namespace lh {

__device__ uint32_t g_device_status = 0;

cudaError_t device_status_read_clear(uint32_t* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
}

bool attn_tc_available() { return false; }
int attn_tc_fwd_launches(const Geom&) { return 0; }
int attn_tc_bwd_launches(const Geom&) { return 0; }

cudaError_t launch_attn_fwd_tc(const Geom&, const __half*, const __half*,
                               const __half*, float, __half*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_attn_bwd_tc(const Geom&, const __half*, const __half*,
                               const __half*, const __half*, const float*,
                               const float*, float, float*, float*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lh
