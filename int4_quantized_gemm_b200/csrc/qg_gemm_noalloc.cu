// qg_gemm_noalloc.cu -- W4A16 decode GEMM whose scratch memory is a static
// device array of the library, for callers that may not allocate device memory.
//
// The stream-K W4A16 decode kernel combines the partial tiles that several CTAs
// share through a scratch buffer (arrival counters + fp32 partial tiles).  Some
// callers cannot hand it one: code embedded in a runtime that owns every byte
// of device memory through its own pool and forbids allocation at execute
// time, and latency-bound loops that cannot afford cudaMalloc/cudaFree, which
// may synchronize the device and take far longer than the GEMM itself.  This
// entry point gives them the same kernel with its scratch in g_static_scratch
// below: a fixed array that every device loading the library holds until the
// process exits.  It allocates nothing: no cudaMalloc, no cudaFree, no
// allocating library call.

#include <mutex>

#include "qg_internal.h"

namespace qg {
namespace {

// 4 MiB: the counters plus one double-buffered 128x16 fp32 partial tile per
// CTA -- enough for M <= 16 (16-wide decode tiles) on up to 255 SMs.
constexpr size_t kStaticScratchBytes = (size_t)4 << 20;
constexpr int64_t kStaticScratchMaxM = 16;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device.  In host code the
// name g_static_scratch is only a host-side stand-in, never a device address,
// so the address is asked of the runtime once per device (with that device
// current) and cached.
qg_status static_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(QG_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices)
    return fail(QG_ERR_UNSUPPORTED, "device ordinal %d: the static scratch serves devices 0..%d", dev,
                kMaxDevices - 1);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(QG_ERR_CUDA, "cudaGetSymbolAddress(static scratch) on device %d: %s", dev,
                  cudaGetErrorString(e));
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return QG_OK;
}

}  // namespace
}  // namespace qg

using namespace qg;

extern "C" qg_status qg_gemm_w4a16_noalloc(const void* x, int64_t ldx, const int32_t* qweight,
                                           const void* scale, const void* zero, int64_t group,
                                           const float* bias, void* y, int64_t ldy, int64_t M,
                                           int64_t N, int64_t K, qg_stream_t stream) {
  if (M > kStaticScratchMaxM)
    return fail(QG_ERR_UNSUPPORTED,
                "qg_gemm_w4a16_noalloc: M=%lld is above %lld, the largest M its %zu-byte static "
                "scratch serves; call qg_gemm_w4a16 instead",
                (long long)M, (long long)kStaticScratchMaxM, kStaticScratchBytes);
  // Every argument and the device are checked before the shared array is
  // touched: a rejected call leaves it (and any kernel still using it) alone.
  W4A16Work work;
  qg_status st = check_gemm_w4a16(x, ldx, qweight, scale, zero, group, bias, y, ldy, M, N, K, QG_ACT_NONE, &work);
  if (st != QG_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (work == W4A16Work::kNone) return QG_OK;
  if (work == W4A16Work::kBiasOnly) return launch_fill_bias(bias, y, QG_F16, ldy, M, N, s);  // no scratch
  const size_t need = qg_gemm_workspace_size(M, N, K);
  if (need > kStaticScratchBytes)
    return fail(QG_ERR_UNSUPPORTED,
                "qg_gemm_w4a16_noalloc: M=%lld needs %zu bytes of scratch on this device, more than "
                "the %zu-byte static scratch",
                (long long)M, need, kStaticScratchBytes);
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != QG_OK) return st;
  // The array keeps whatever the previous call left; the arrival counters must
  // start at zero (a call that timed out may have left them set).  Cleared on
  // `stream` right before the kernel that uses them.
  st = check_cuda(cudaMemsetAsync(scratch, 0, decode_ticket_bytes(), s), "clearing the static scratch counters");
  if (st != QG_OK) return st;
  return launch_decode_w4a16(x, ldx, qweight, scale, zero, bias, y, ldy, M, N, K, scratch, s);
}
