// qg_gemm_wonly.cu -- weight-only GEMMs (W8A16, W4A16) on the sm_100a tensor
// cores.  (Kernels are added in the next step; the launchers report
// QG_ERR_UNSUPPORTED until then.)
#include <cuda_runtime.h>

#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

static __device__ unsigned long long g_status_wonly;

unsigned long long read_clear_status_wonly(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_wonly, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_wonly, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

qg_status launch_w8a16(const void*, int64_t, const int8_t*, int64_t, const float*, const float*,
                       void*, int64_t, int64_t, int64_t, int64_t, cudaStream_t) {
  return fail(QG_ERR_UNSUPPORTED, "W8A16 kernel not built yet");
}

qg_status launch_w4a16(const void*, int64_t, const int32_t*, const void*, const void*, const float*,
                       void*, int64_t, int64_t, int64_t, int64_t, cudaStream_t) {
  return fail(QG_ERR_UNSUPPORTED, "W4A16 kernel not built yet");
}

}  // namespace qg
