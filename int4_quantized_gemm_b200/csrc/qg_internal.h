// qg_internal.h -- host-side helpers shared by the library's translation units
// (not part of the public C ABI in include/qg.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/qg.h"

namespace qg {

// Record a one-line message for qg_last_error_message() and return `st`.
qg_status fail(qg_status st, const char* fmt, ...);

// Map a CUDA runtime error to QG_ERR_CUDA with its message (QG_OK if none).
qg_status check_cuda(cudaError_t e, const char* what);

// Number of SMs of the current device (cached per device).
int sm_count();

// Per-device one-time setup (a kernel's shared-memory attribute, an occupancy
// query): `setup(dev)` runs for the first call on each device ordinal 0..63;
// concurrent first calls from several host threads are serialized, later
// calls take one atomic load.  A setup that fails is retried by the next call.
// Whatever `setup` writes is visible to every caller once run() returns QG_OK.
struct PerDeviceOnce {
  std::atomic<bool> done[64] = {};
  std::mutex mu;
  template <class F>
  qg_status run(F&& setup) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return setup(dev);  // not cached
    if (done[dev].load(std::memory_order_acquire)) return QG_OK;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev].load(std::memory_order_relaxed)) return QG_OK;
    const qg_status st = setup(dev);
    if (st == QG_OK) done[dev].store(true, std::memory_order_release);
    return st;
  }
};

// Tuning switches.  Each starts from its environment variable, read once per
// process on first use (unset: the measured default, 0 = automatic), and can
// be changed later through qg_set_tuning() (tests compare kernel variants that
// way).  Names:
//   QG_W8A8_PAIR      1: prefill W8A8 above 128 rows on CTA pairs; 0: one-SM tiles
//   QG_PAIR_STAGES    ring stages of the CTA-pair kernel (6, or 7)
//   QG_W8A8_SPLITS    W8A8 decode cluster size (K splits), 0 = automatic
//   QG_W8A16_SPLITS   weight-only W8A16 decode cluster size, 0 = automatic
//   QG_W4A16_SPLITS   weight-only W4A16 decode cluster size, 0 = automatic
//   QG_WONLY_BN       weight-only X tile width (16/32/64/128/256), 0 = automatic
//   QG_PAIR_N         CTA-pair tile width (output columns, a multiple of 16 in
//                     128..256), 0 = automatic
// Fault injection for tests (qg_debug_inject_timeout): the armed wait limit
// in microseconds for kernel family `family` (a qg_debug_family), disarming
// it, or 0 when nothing is armed.  Launchers put a nonzero result in their
// kernel parameters (withhold one copy, short waits).
uint32_t take_debug_injection(int family);

enum TuneId { kTuneW8A8Pair = 0, kTunePairStages, kTuneW8A8Splits, kTuneW8A16Splits, kTuneW4A16Splits,
              kTuneWonlyBn, kTunePairN, kTuneCount };
int tuning(TuneId id);

// Fill a launch configuration: grid, block, dynamic shared memory, stream,
// programmatic dependent launch allowed, and an optional cluster size along x.
struct LaunchCfg {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  LaunchCfg(unsigned grid, unsigned block, size_t smem, cudaStream_t s, unsigned cluster_x = 1) {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster_x > 1) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = cluster_x;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.numAttrs = 2;
    }
  }
};

// Encode a 2-D tiled TMA descriptor for a row-major matrix of `rows` x `cols`
// elements (cols innermost) with leading dimension `ld` elements.  Box is
// box_cols x box_rows.  Out-of-range elements of a box read as zero.
qg_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                       int elem_bytes, uint64_t cols, uint64_t rows, uint64_t ld,
                       uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// Per-translation-unit device status words: read and clear.
unsigned long long read_clear_status_quantize(cudaStream_t s);
unsigned long long read_clear_status_w8a8(cudaStream_t s);
unsigned long long read_clear_status_wonly(cudaStream_t s);
unsigned long long read_clear_status_decode(cudaStream_t s);
unsigned long long read_clear_status_pair(cudaStream_t s);

// Launchers (arguments already validated by the C ABI layer).
qg_status launch_quantize_rowwise(const void* x, int64_t ldx, int8_t* xq, int64_t ldq, float* xs,
                                  int64_t M, int64_t K, cudaStream_t s);
qg_status launch_quantize_rowwise_asym(const void* x, int64_t ldx, int8_t* xq, int64_t ldq, float* xs,
                                       float* xz, int32_t* qsum, int64_t M, int64_t K, cudaStream_t s);
qg_status launch_quantize_block_sym4(const void* w, int64_t ldw, int32_t* qweight, void* scale, int64_t N,
                                     int64_t K, cudaStream_t s);
qg_status launch_quantize_channel_sym4(const void* w, int64_t ldw, int32_t* qweight, float* scale, int64_t N,
                                       int64_t K, cudaStream_t s);
qg_status launch_quantize_block_asym4(const void* w, int64_t ldw, int32_t* qweight, void* scale,
                                      void* zero, int64_t N, int64_t K, cudaStream_t s);
// `act` is a qg_activation applied to the fp32 epilogue value (0: none).
// `flags`: qg_flags bits (QG_FLAG_STATIC_WEIGHTS).
qg_status launch_w8a8(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                      const float* xs, const float* ws, const float* bias, void* y, int dtype,
                      int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t s, int act = 0,
                      unsigned flags = 0);
qg_status launch_w8a16(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw, const float* ws,
                       const float* bias, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                       cudaStream_t s, int act = 0, unsigned flags = 0);
qg_status launch_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                       const void* zero, const float* bias, void* y, int64_t ldy, int64_t M,
                       int64_t N, int64_t K, cudaStream_t s, int act = 0, unsigned flags = 0);
// W4A8 for M <= 64 on the weight-only decode pipeline (int8 codes into the
// tensor-memory A operand, kind::i8), W8A8 epilogue; qg_gemm_wonly.cu.
qg_status launch_w4a8_decode(const int8_t* xq, int64_t ldx, const int32_t* qweight, const float* xs,
                             const float* ws, const float* bias, void* y, int dtype, int64_t ldy, int64_t M,
                             int64_t N, int64_t K, cudaStream_t s);
// W4A8: per-column symmetric int4 weights (packed [N, K/8]) unpacked to int8 on chip.
qg_status launch_w4a8(const int8_t* xq, int64_t ldx, const int32_t* qweight, const float* xs,
                      const float* ws, const float* bias, void* y, int dtype, int64_t ldy, int64_t M,
                      int64_t N, int64_t K, cudaStream_t s, int act = 0);
// Zero-point W8A8: per-row zero points and code sums (each nullable).
qg_status launch_w8a8_zp(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw, const float* xs,
                         const float* xz, const int32_t* xsum, const float* ws, const float* wz,
                         const int32_t* wsum, const float* bias, void* y, int dtype, int64_t ldy,
                         int64_t M, int64_t N, int64_t K, cudaStream_t s);
// Fused per-row int8 quantization of X + W8A8 decode GEMM (M <= 64, K >= 1).
qg_status launch_quantize_w8a8(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                               const float* ws, const float* bias, void* y, int dtype, int64_t ldy,
                               int8_t* xq_out, int64_t ldxq, float* xs_out, int64_t M, int64_t N,
                               int64_t K, cudaStream_t s);
// Symmetric group-int4 W4A16 (two's-complement codes, fp16 scale [K/64, N], no zero points).
qg_status launch_w4a16_sym(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                           const float* bias, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           cudaStream_t s, int act = 0);
// Stream-K decode kernels (M <= 64) and the workspace they need.
size_t decode_workspace_bytes(int64_t M, int64_t N);
// Leading bytes of a stream-K workspace that must be zero when a launch starts
// (the tile arrival counters); the rest is written before it is read.
size_t decode_ticket_bytes();
qg_status launch_decode_w8a8(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                             const float* xs, const float* ws, const float* bias, void* y, int dtype,
                             int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                             cudaStream_t s);
qg_status launch_decode_w8a16(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                              const float* ws, const float* bias, void* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, void* workspace, cudaStream_t s);
qg_status launch_decode_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                              const void* zero, const float* bias, void* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, void* workspace, cudaStream_t s);
// Argument checks of qg_gemm_w4a16 (everything it verifies before enqueuing,
// the device included), shared with the allocation-free entry point.  On QG_OK
// *work says what the call has to do.
enum class W4A16Work { kNone, kBiasOnly, kProduct };
qg_status check_gemm_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                           const void* zero, int64_t group, const float* bias, const void* y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, int act, W4A16Work* work);
// Weight-only GEMMs for M > 64 on wide token tiles (BN = 128/256; bn_force 0:
// automatic); w and ldw_bytes are the int8 [N, K] or packed int4 [N, K/8]
// weight and its row pitch in bytes.
qg_status launch_wonly_wide(bool w4, const void* x, int64_t ldx, const void* w, int64_t ldw_bytes,
                            const void* scale, const void* zero, const float* ws, const float* bias, void* y,
                            int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t s, int act, bool sym,
                            unsigned flags, int bn_force);
unsigned long long read_clear_status_wide(cudaStream_t s);
// Y = bias (or 0) for the empty sum K == 0.
qg_status launch_fill_bias(const float* bias, void* y, int dtype, int64_t ldy, int64_t M,
                           int64_t N, cudaStream_t s, int act = 0);

}  // namespace qg
