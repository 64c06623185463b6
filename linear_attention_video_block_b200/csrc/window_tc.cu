// tcgen05 / TMEM / TMA window softmax for bf16 (sm_100a).
#include "vdn_internal.cuh"

namespace vdn {

// Device-side status word of this translation unit.
__device__ int g_vdn_status = 0;

cudaError_t read_and_clear_tc_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_vdn_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_vdn_status, &zero, sizeof(int));
}

bool window_tc_supported(const Layout&, int) { return false; }

cudaError_t launch_window_tc(const Layout&, const void*, const void*, const void*, const void*,
                             const void*, void*, bool, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace vdn
