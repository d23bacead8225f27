// qg_abi.cu -- the extern "C" entry points of libqg.so (declared in
// include/qg.h): argument validation, TMA descriptor encoding, dispatch to the
// kernels' launchers, status codes, launch plans.  Nothing here computes on
// the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/qg.h"
#include "qg_device.cuh"
#include "qg_internal.h"

#define QG_VERSION 100  // 0.1.0

namespace qg {

static thread_local char g_msg[512] = "";

qg_status fail(qg_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

qg_status check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return QG_OK;
  return fail(QG_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int sm_count() {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// ---------------------------------------------------------------------------
// Tuning switches: environment once per process, then qg_set_tuning().
// ---------------------------------------------------------------------------
static const char* const kTuneNames[kTuneCount] = {"QG_W8A8_PAIR",    "QG_PAIR_STAGES",  "QG_W8A8_SPLITS",
                                                   "QG_W8A16_SPLITS", "QG_W4A16_SPLITS", "QG_WONLY_BN",
                                                   "QG_PAIR_N"};
static const int kTuneDefaults[kTuneCount] = {1, 6, 0, 0, 0, 0, 0};
static std::atomic<int> g_tune[kTuneCount];
static std::once_flag g_tune_once;

static void tuning_init() {
  std::call_once(g_tune_once, [] {
    for (int i = 0; i < kTuneCount; ++i) {
      const char* v = std::getenv(kTuneNames[i]);
      g_tune[i].store(v ? std::atoi(v) : kTuneDefaults[i], std::memory_order_relaxed);
    }
  });
}

int tuning(TuneId id) {
  tuning_init();
  return g_tune[id].load(std::memory_order_relaxed);
}

// ---------------------------------------------------------------------------
// Test-only fault injection: one armed launch per kernel family.
// ---------------------------------------------------------------------------
static std::atomic<uint32_t> g_inject[3];

uint32_t take_debug_injection(int family) {
  if (family < 1 || family > 2) return 0;
  if (g_inject[family].load(std::memory_order_relaxed) == 0) return 0;  // the usual case: one load
  return g_inject[family].exchange(0, std::memory_order_acq_rel);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library has no link-time dependency on libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A descriptor depends only on its encode arguments, so recently encoded ones
// are reused (per host thread, direct-mapped on a hash of the arguments):
// decode-sized calls otherwise spend a good part of their host time encoding.
struct TmapKey {
  const void* base;
  uint64_t cols, rows, ld;
  uint32_t box_cols, box_rows;
  int dtype, elem_bytes, swizzle;
  bool operator==(const TmapKey& o) const {
    return base == o.base && cols == o.cols && rows == o.rows && ld == o.ld && box_cols == o.box_cols &&
           box_rows == o.box_rows && dtype == o.dtype && elem_bytes == o.elem_bytes && swizzle == o.swizzle;
  }
};

struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  bool valid;
};

static TmapEntry* tmap_slot(const TmapKey& k) {
  constexpr int kSlots = 64;
  static thread_local TmapEntry cache[kSlots] = {};
  uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
  h ^= (k.cols * 31 + k.rows) * 0xC2B2AE3D27D4EB4Full;
  h ^= (k.ld * 131 + k.box_cols * 7 + k.box_rows) * 0x165667B19E3779F9ull;
  h ^= (uint64_t)(k.dtype * 17 + k.elem_bytes * 5 + k.swizzle);
  return &cache[(h >> 32) % kSlots];
}

qg_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                       uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_cols,
                       uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  const TmapKey key = {base, cols, rows, ld, box_cols, box_rows, (int)dtype, elem_bytes, (int)swizzle};
  TmapEntry* e = tmap_slot(key);
  if (e->valid && e->key == key) {
    *map = e->map;
    return QG_OK;
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(QG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(QG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu, ld %llu", (int)r,
                (unsigned long long)cols, (unsigned long long)rows, (unsigned long long)ld);
  e->key = key;
  e->map = *map;
  e->valid = true;
  return QG_OK;
}

}  // namespace qg

using namespace qg;

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 31;
constexpr int64_t kMaxKInt8 = 133144;  // 2^31 / 127^2: int32 accumulation stays exact
constexpr int64_t kMaxKZp = 131071;    // 2^31 / 128^2 - 1: the same with codes in [-128, 127]

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

qg_status check_dims(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return fail(QG_ERR_INVALID_ARG, "negative size (M=%lld N=%lld K=%lld)", (long long)M, (long long)N, (long long)K);
  if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim) return fail(QG_ERR_UNSUPPORTED, "size >= 2^31");
  return QG_OK;
}

qg_status check_matrix(const void* p, int64_t ld, int64_t cols, int elem, const char* name) {
  if (!p) return fail(QG_ERR_INVALID_ARG, "%s is NULL", name);
  if (ld < cols) return fail(QG_ERR_INVALID_ARG, "%s: leading dimension %lld < %lld", name, (long long)ld, (long long)cols);
  if (!aligned(p, 16)) return fail(QG_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
  if ((ld * elem) % 16 != 0) return fail(QG_ERR_ALIGNMENT, "%s: leading dimension %lld x %d bytes is not a multiple of 16", name, (long long)ld, elem);
  return QG_OK;
}

qg_status check_vec(const void* p, size_t align, const char* name, bool nullable) {
  if (!p) return nullable ? QG_OK : fail(QG_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(QG_ERR_ALIGNMENT, "%s is not %zu-byte aligned", name, align);
  return QG_OK;
}

qg_status check_device() {
  static std::atomic<bool> ok_dev[64] = {};  // device known to be compute capability 10.x
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(QG_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  }
  if (dev >= 0 && dev < 64 && ok_dev[dev].load(std::memory_order_relaxed)) return QG_OK;
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major == 10 && dev >= 0 && dev < 64) ok_dev[dev].store(true, std::memory_order_relaxed);
  if (major != 10) return fail(QG_ERR_NO_DEVICE, "device %d is compute capability %d.x; libqg needs sm_100", dev, major);
  return QG_OK;
}

// A usable stream-K workspace for this problem, or NULL (cluster split-K).
qg_status check_act(int act) {
  if (act != QG_ACT_NONE && act != QG_ACT_GELU) return fail(QG_ERR_INVALID_ARG, "unknown activation %d", act);
  return QG_OK;
}

qg_status check_flags(unsigned flags) {
  if (flags & ~(unsigned)QG_FLAG_STATIC_WEIGHTS) return fail(QG_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  return QG_OK;
}

void* usable_workspace(void* ws, size_t bytes, int64_t M, int64_t N, int64_t K) {
  if (!ws || M > 64 || !aligned(ws, 16)) return nullptr;
  return bytes >= qg_gemm_workspace_size(M, N, K) ? ws : nullptr;
}

#define QG_TRY(expr)                   \
  do {                                 \
    qg_status _st = (expr);            \
    if (_st != QG_OK) return _st;      \
  } while (0)

}  // namespace

namespace qg {

qg_status check_gemm_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                           const void* zero, int64_t group, const float* bias, const void* y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, int act, W4A16Work* work) {
  *work = W4A16Work::kNone;
  QG_TRY(check_dims(M, N, K));
  QG_TRY(check_act(act));
  if (group != 64) return fail(QG_ERR_UNSUPPORTED, "group %lld: only 64 is implemented", (long long)group);
  if (K % group != 0) return fail(QG_ERR_INVALID_ARG, "K=%lld is not a multiple of the group %lld", (long long)K, (long long)group);
  if (M == 0 || N == 0) return QG_OK;
  if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
  if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
  QG_TRY(check_vec(y, 2, "y", false));
  QG_TRY(check_vec(bias, 4, "bias", true));
  QG_TRY(check_device());
  if (K == 0) {
    *work = W4A16Work::kBiasOnly;
    return QG_OK;
  }
  QG_TRY(check_matrix(x, ldx, K, 2, "x"));
  QG_TRY(check_matrix(qweight, K / 8, K / 8, 4, "qweight"));
  QG_TRY(check_vec(scale, 16, "scale", false));
  QG_TRY(check_vec(zero, 16, "zero", false));
  if ((N * 2) % 16 != 0) return fail(QG_ERR_ALIGNMENT, "scale/zero rows of N=%lld fp16 are not a multiple of 16 bytes", (long long)N);
  *work = W4A16Work::kProduct;
  return QG_OK;
}

}  // namespace qg

extern "C" {

const char* qg_status_string(int status) {
  switch (status) {
    case QG_OK: return "QG_OK";
    case QG_ERR_INVALID_ARG: return "QG_ERR_INVALID_ARG";
    case QG_ERR_ALIGNMENT: return "QG_ERR_ALIGNMENT";
    case QG_ERR_UNSUPPORTED: return "QG_ERR_UNSUPPORTED";
    case QG_ERR_CUDA: return "QG_ERR_CUDA";
    case QG_ERR_TIMEOUT: return "QG_ERR_TIMEOUT";
    case QG_ERR_NO_DEVICE: return "QG_ERR_NO_DEVICE";
    case QG_ERR_DEBUG_CHECK: return "QG_ERR_DEBUG_CHECK";
    default: return "QG_ERR_UNKNOWN";
  }
}

int qg_debug_checks(void) {
#ifdef QG_DEBUG
  return 1;
#else
  return 0;
#endif
}

const char* qg_last_error_message(void) { return g_msg; }

int qg_version(void) { return QG_VERSION; }

qg_status qg_debug_inject_timeout(int family, int wait_limit_us) {
  if (family != QG_DEBUG_WEIGHT_ONLY && family != QG_DEBUG_STREAM_K)
    return fail(QG_ERR_INVALID_ARG, "unknown kernel family %d", family);
  if (wait_limit_us < 100 || wait_limit_us > 1000000)
    return fail(QG_ERR_INVALID_ARG, "wait limit %d us outside [100, 1000000]", wait_limit_us);
  g_inject[family].store((uint32_t)wait_limit_us, std::memory_order_release);
  return QG_OK;
}

qg_status qg_set_tuning(const char* name, int value) {
  if (!name) return fail(QG_ERR_INVALID_ARG, "tuning switch name is NULL");
  tuning_init();
  for (int i = 0; i < kTuneCount; ++i)
    if (std::strcmp(name, kTuneNames[i]) == 0) {
      g_tune[i].store(value, std::memory_order_relaxed);
      return QG_OK;
    }
  return fail(QG_ERR_INVALID_ARG, "unknown tuning switch \"%s\"", name);
}

size_t qg_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > 64) return 0;
  return decode_workspace_bytes(M, N);
}

qg_status qg_check_device_errors(qg_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  QG_TRY(check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize"));
  unsigned long long words[6] = {read_clear_status_quantize(s), read_clear_status_w8a8(s),
                                 read_clear_status_wonly(s), read_clear_status_decode(s),
                                 read_clear_status_pair(s), read_clear_status_wide(s)};
  QG_TRY(check_cuda(cudaGetLastError(), "reading device status"));
  static const char* names[6] = {"quantize", "w8a8", "weight-only", "decode", "w8a8 pair", "weight-only wide"};
  for (int i = 0; i < 6; ++i) {
    if (words[i] != 0) {
      const unsigned code = (unsigned)(words[i] & 0xFF);
      const unsigned site = (unsigned)((words[i] >> 8) & 0xFFFF);
      const unsigned long long block = words[i] >> 24;
      const qg_status st = code == kDevTimeout ? QG_ERR_TIMEOUT : code == kDevDebugCheck ? QG_ERR_DEBUG_CHECK : QG_ERR_CUDA;
      return fail(st, "%s kernel: device status code %u at %s site %u, block %llu", names[i], code,
                  code == kDevDebugCheck ? "check" : "wait", site, block);
    }
  }
  return QG_OK;
}

qg_status qg_quantize_rowwise_int8(const void* x, int64_t ldx, int8_t* xq, int64_t ldxq,
                                   float* x_scale, int64_t M, int64_t K, qg_stream_t stream) {
  QG_TRY(check_dims(M, 0, K));
  if (M == 0) return QG_OK;
  QG_TRY(check_matrix(x, ldx, K, 2, "x"));
  QG_TRY(check_matrix(xq, ldxq, K, 1, "xq"));
  QG_TRY(check_vec(x_scale, 4, "x_scale", false));
  QG_TRY(check_device());
  return launch_quantize_rowwise(x, ldx, xq, ldxq, x_scale, M, K,
                                 reinterpret_cast<cudaStream_t>(stream));
}

qg_status qg_quantize_rowwise_asym_int8(const void* x, int64_t ldx, int8_t* xq, int64_t ldxq,
                                        float* scale, float* zero, int32_t* qsum, int64_t M, int64_t K,
                                        qg_stream_t stream) {
  QG_TRY(check_dims(M, 0, K));
  if (K > kMaxKZp) return fail(QG_ERR_UNSUPPORTED, "K=%lld exceeds %lld (int32 code sums and products)", (long long)K, (long long)kMaxKZp);
  if (M == 0) return QG_OK;
  if (K > 0) QG_TRY(check_matrix(x, ldx, K, 2, "x"));
  QG_TRY(check_matrix(xq, ldxq, K, 1, "xq"));
  QG_TRY(check_vec(scale, 4, "scale", false));
  QG_TRY(check_vec(zero, 4, "zero", false));
  QG_TRY(check_vec(qsum, 4, "qsum", true));
  QG_TRY(check_device());
  return launch_quantize_rowwise_asym(x, ldx, xq, ldxq, scale, zero, qsum, M, K,
                                      reinterpret_cast<cudaStream_t>(stream));
}

qg_status qg_quantize_block_sym4(const void* w, int64_t ldw, int32_t* qweight, void* scale, int64_t N,
                                 int64_t K, int64_t group, qg_stream_t stream) {
  QG_TRY(check_dims(0, N, K));
  if (group != 64) return fail(QG_ERR_UNSUPPORTED, "group %lld: only 64 is implemented", (long long)group);
  if (K % group != 0) return fail(QG_ERR_INVALID_ARG, "K=%lld is not a multiple of the group %lld", (long long)K, (long long)group);
  if (N == 0 || K == 0) return QG_OK;
  QG_TRY(check_matrix(w, ldw, K, 2, "w"));
  QG_TRY(check_matrix(qweight, K / 8, K / 8, 4, "qweight"));
  QG_TRY(check_vec(scale, 2, "scale", false));
  QG_TRY(check_device());
  return launch_quantize_block_sym4(w, ldw, qweight, scale, N, K, reinterpret_cast<cudaStream_t>(stream));
}

qg_status qg_quantize_channel_sym4(const void* w, int64_t ldw, int32_t* qweight, float* scale, int64_t N,
                                   int64_t K, qg_stream_t stream) {
  QG_TRY(check_dims(0, N, K));
  if (K % 32 != 0) return fail(QG_ERR_INVALID_ARG, "K=%lld is not a multiple of 32", (long long)K);
  if (N == 0) return QG_OK;
  if (K > 0) {
    QG_TRY(check_matrix(w, ldw, K, 2, "w"));
    QG_TRY(check_matrix(qweight, K / 8, K / 8, 4, "qweight"));
  }
  QG_TRY(check_vec(scale, 4, "scale", false));
  QG_TRY(check_device());
  return launch_quantize_channel_sym4(w, ldw, qweight, scale, N, K, reinterpret_cast<cudaStream_t>(stream));
}

qg_status qg_quantize_block_asym4(const void* w, int64_t ldw, int32_t* qweight, void* scale,
                                  void* zero, int64_t N, int64_t K, int64_t group,
                                  qg_stream_t stream) {
  QG_TRY(check_dims(0, N, K));
  if (group != 64) return fail(QG_ERR_UNSUPPORTED, "group %lld: only 64 is implemented", (long long)group);
  if (K % group != 0) return fail(QG_ERR_INVALID_ARG, "K=%lld is not a multiple of the group %lld", (long long)K, (long long)group);
  if (N == 0 || K == 0) return QG_OK;
  QG_TRY(check_matrix(w, ldw, K, 2, "w"));
  QG_TRY(check_matrix(qweight, K / 8, K / 8, 4, "qweight"));
  QG_TRY(check_vec(scale, 2, "scale", false));
  QG_TRY(check_vec(zero, 2, "zero", false));
  QG_TRY(check_device());
  return launch_quantize_block_asym4(w, ldw, qweight, scale, zero, N, K,
                                     reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

qg_status gemm_w8a8(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw, const float* x_scale,
                    const float* w_scale, const float* bias, void* y, int y_dtype, int64_t ldy, int64_t M,
                    int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int act,
                    unsigned flags, qg_stream_t stream) {
  QG_TRY(check_dims(M, N, K));
  QG_TRY(check_act(act));
  QG_TRY(check_flags(flags));
  if (act != QG_ACT_NONE && y_dtype == QG_I32) return fail(QG_ERR_INVALID_ARG, "an activation needs a floating-point output");
  if (y_dtype < QG_F32 || y_dtype > QG_I32) return fail(QG_ERR_INVALID_ARG, "unknown output dtype %d", y_dtype);
  if (K > kMaxKInt8) return fail(QG_ERR_UNSUPPORTED, "K=%lld exceeds %lld (int32 accumulation bound)", (long long)K, (long long)kMaxKInt8);
  if (M == 0 || N == 0) return QG_OK;
  const int es = (y_dtype == QG_F16 || y_dtype == QG_BF16) ? 2 : 4;
  if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
  if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
  QG_TRY(check_vec(y, (size_t)es, "y", false));
  const bool raw = y_dtype == QG_I32;
  QG_TRY(check_vec(x_scale, 4, "x_scale", raw));
  QG_TRY(check_vec(w_scale, 4, "w_scale", raw));
  QG_TRY(check_vec(bias, 4, "bias", true));
  QG_TRY(check_device());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return launch_fill_bias(raw ? nullptr : bias, y, y_dtype, ldy, M, N, s, act);
  QG_TRY(check_matrix(xq, ldx, K, 1, "xq"));
  QG_TRY(check_matrix(wq, ldw, K, 1, "wq"));
  if (act == QG_ACT_NONE)
    if (void* ws = usable_workspace(workspace, workspace_bytes, M, N, K))
      return launch_decode_w8a8(xq, ldx, wq, ldw, x_scale, w_scale, bias, y, y_dtype, ldy, M, N, K, ws, s);
  return launch_w8a8(xq, ldx, wq, ldw, x_scale, w_scale, bias, y, y_dtype, ldy, M, N, K, s, act, flags);
}

qg_status gemm_w8a16(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw, const float* w_scale,
                     const float* bias, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                     void* workspace, size_t workspace_bytes, int act, unsigned flags, qg_stream_t stream) {
  QG_TRY(check_dims(M, N, K));
  QG_TRY(check_act(act));
  QG_TRY(check_flags(flags));
  if (M == 0 || N == 0) return QG_OK;
  if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
  if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
  QG_TRY(check_vec(y, 2, "y", false));
  QG_TRY(check_vec(w_scale, 4, "w_scale", false));
  QG_TRY(check_vec(bias, 4, "bias", true));
  QG_TRY(check_device());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return launch_fill_bias(bias, y, QG_F16, ldy, M, N, s);
  QG_TRY(check_matrix(x, ldx, K, 2, "x"));
  QG_TRY(check_matrix(wq, ldw, K, 1, "wq"));
  if (act == QG_ACT_NONE)
    if (void* ws = usable_workspace(workspace, workspace_bytes, M, N, K))
      return launch_decode_w8a16(x, ldx, wq, ldw, w_scale, bias, y, ldy, M, N, K, ws, s);
  return launch_w8a16(x, ldx, wq, ldw, w_scale, bias, y, ldy, M, N, K, s, act, flags);
}

qg_status gemm_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                     const void* zero, int64_t group, const float* bias, void* y, int64_t ldy, int64_t M,
                     int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int act,
                     unsigned flags, qg_stream_t stream) {
  QG_TRY(check_flags(flags));
  W4A16Work work;
  QG_TRY(check_gemm_w4a16(x, ldx, qweight, scale, zero, group, bias, y, ldy, M, N, K, act, &work));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (work == W4A16Work::kNone) return QG_OK;
  if (work == W4A16Work::kBiasOnly) return launch_fill_bias(bias, y, QG_F16, ldy, M, N, s);
  if (act == QG_ACT_NONE)
    if (void* ws = usable_workspace(workspace, workspace_bytes, M, N, K))
      return launch_decode_w4a16(x, ldx, qweight, scale, zero, bias, y, ldy, M, N, K, ws, s);
  return launch_w4a16(x, ldx, qweight, scale, zero, bias, y, ldy, M, N, K, s, act, flags);
}

}  // namespace

extern "C" {

qg_status qg_gemm_w8a8_zp(const int8_t* xq, int64_t ldx, const float* x_scale, const float* x_zero,
                          const int32_t* x_qsum, const int8_t* wq, int64_t ldw, const float* w_scale,
                          const float* w_zero, const int32_t* w_qsum, const float* bias, void* y,
                          int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K, qg_stream_t stream) {
  QG_TRY(check_dims(M, N, K));
  if (y_dtype < QG_F32 || y_dtype > QG_I32) return fail(QG_ERR_INVALID_ARG, "unknown output dtype %d", y_dtype);
  if (K > kMaxKZp) return fail(QG_ERR_UNSUPPORTED, "K=%lld exceeds %lld (int32 accumulation bound)", (long long)K, (long long)kMaxKZp);
  if (w_zero && !x_qsum) return fail(QG_ERR_INVALID_ARG, "w_zero needs x_qsum (the code row sums of Xq)");
  if (x_zero && !w_qsum) return fail(QG_ERR_INVALID_ARG, "x_zero needs w_qsum (the code row sums of the [N,K] Wq)");
  if (M == 0 || N == 0) return QG_OK;
  const int es = (y_dtype == QG_F16 || y_dtype == QG_BF16) ? 2 : 4;
  if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
  if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
  QG_TRY(check_vec(y, (size_t)es, "y", false));
  const bool raw = y_dtype == QG_I32;
  QG_TRY(check_vec(x_scale, 4, "x_scale", raw));
  QG_TRY(check_vec(w_scale, 4, "w_scale", raw));
  QG_TRY(check_vec(x_zero, 4, "x_zero", true));
  QG_TRY(check_vec(w_zero, 4, "w_zero", true));
  QG_TRY(check_vec(x_qsum, 4, "x_qsum", true));
  QG_TRY(check_vec(w_qsum, 4, "w_qsum", true));
  QG_TRY(check_vec(bias, 4, "bias", true));
  QG_TRY(check_device());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return launch_fill_bias(raw ? nullptr : bias, y, y_dtype, ldy, M, N, s);
  QG_TRY(check_matrix(xq, ldx, K, 1, "xq"));
  QG_TRY(check_matrix(wq, ldw, K, 1, "wq"));
  return launch_w8a8_zp(xq, ldx, wq, ldw, x_scale, x_zero, x_qsum, w_scale, w_zero, w_qsum, bias, y,
                        y_dtype, ldy, M, N, K, s);
}

qg_status qg_quantize_gemm_w8a8(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                                const float* w_scale, const float* bias, void* y, int y_dtype,
                                int64_t ldy, int8_t* xq, int64_t ldxq, float* x_scale, int64_t M,
                                int64_t N, int64_t K, qg_stream_t stream) {
  QG_TRY(check_dims(M, N, K));
  if (y_dtype < QG_F32 || y_dtype > QG_I32) return fail(QG_ERR_INVALID_ARG, "unknown output dtype %d", y_dtype);
  if (K > kMaxKInt8) return fail(QG_ERR_UNSUPPORTED, "K=%lld exceeds %lld (int32 accumulation bound)", (long long)K, (long long)kMaxKInt8);
  if (M > 64)
    return fail(QG_ERR_UNSUPPORTED, "M=%lld: the fused quantize + GEMM serves decode batches (M <= 64); "
                "use qg_quantize_rowwise_int8 then qg_gemm_w8a8", (long long)M);
  if (M == 0) return QG_OK;
  if (K > 0) QG_TRY(check_matrix(x, ldx, K, 2, "x"));  // with K == 0, x is never read
  if (xq) QG_TRY(check_matrix(xq, ldxq, K, 1, "xq"));
  QG_TRY(check_vec(x_scale, 4, "x_scale", true));
  if (N == 0 && !xq && !x_scale) return QG_OK;
  const int es = (y_dtype == QG_F16 || y_dtype == QG_BF16) ? 2 : 4;
  const bool raw = y_dtype == QG_I32;
  if (N > 0) {
    if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
    if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
    QG_TRY(check_vec(y, (size_t)es, "y", false));
    QG_TRY(check_vec(w_scale, 4, "w_scale", raw));
    QG_TRY(check_vec(bias, 4, "bias", true));
  }
  QG_TRY(check_device());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0 || N == 0) {
    // No product to fuse with: the row quantizer alone gives x_scale (and the
    // codes), and Y is the empty sum + bias.
    if (K == 0 && x_scale) {
      // no codes to write: the quantizer only stores the scales (its code
      // pointer is never dereferenced for K == 0)
      QG_TRY(launch_quantize_rowwise(x, ldx, xq ? xq : reinterpret_cast<int8_t*>(x_scale), 16, x_scale,
                                     M, 0, s));
    } else if (K > 0 && (x_scale || xq)) {
      if (!xq || !x_scale)
        return fail(QG_ERR_UNSUPPORTED, "with N == 0, request xq and x_scale together");
      QG_TRY(launch_quantize_rowwise(x, ldx, xq, ldxq, x_scale, M, K, s));
    }
    return N > 0 ? launch_fill_bias(raw ? nullptr : bias, y, y_dtype, ldy, M, N, s) : QG_OK;
  }
  QG_TRY(check_matrix(wq, ldw, K, 1, "wq"));
  return launch_quantize_w8a8(x, ldx, wq, ldw, w_scale, bias, y, y_dtype, ldy, xq, ldxq, x_scale, M,
                              N, K, s);
}


qg_status qg_gemm_w4a8(const int8_t* xq, int64_t ldx, const int32_t* qweight, const float* x_scale,
                       const float* w_scale, const float* bias, void* y, int y_dtype, int64_t ldy,
                       int64_t M, int64_t N, int64_t K, qg_stream_t stream) {
  QG_TRY(check_dims(M, N, K));
  if (y_dtype < QG_F32 || y_dtype > QG_I32) return fail(QG_ERR_INVALID_ARG, "unknown output dtype %d", y_dtype);
  if (K % 32 != 0) return fail(QG_ERR_INVALID_ARG, "K=%lld is not a multiple of 32", (long long)K);
  if (K > kMaxKInt8) return fail(QG_ERR_UNSUPPORTED, "K=%lld exceeds %lld (int32 accumulation bound)", (long long)K, (long long)kMaxKInt8);
  if (M == 0 || N == 0) return QG_OK;
  const int es = (y_dtype == QG_F16 || y_dtype == QG_BF16) ? 2 : 4;
  if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
  if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
  QG_TRY(check_vec(y, (size_t)es, "y", false));
  const bool raw = y_dtype == QG_I32;
  QG_TRY(check_vec(x_scale, 4, "x_scale", raw));
  QG_TRY(check_vec(w_scale, 4, "w_scale", raw));
  QG_TRY(check_vec(bias, 4, "bias", true));
  QG_TRY(check_device());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return launch_fill_bias(raw ? nullptr : bias, y, y_dtype, ldy, M, N, s);
  QG_TRY(check_matrix(xq, ldx, K, 1, "xq"));
  QG_TRY(check_matrix(qweight, K / 8, K / 8, 4, "qweight"));
  return launch_w4a8(xq, ldx, qweight, x_scale, w_scale, bias, y, y_dtype, ldy, M, N, K, s);
}

qg_status qg_gemm_w4a16_sym(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                            int64_t group, const float* bias, void* y, int64_t ldy, int64_t M, int64_t N,
                            int64_t K, qg_stream_t stream) {
  QG_TRY(check_dims(M, N, K));
  if (group != 64) return fail(QG_ERR_UNSUPPORTED, "group %lld: only 64 is implemented", (long long)group);
  if (K % group != 0) return fail(QG_ERR_INVALID_ARG, "K=%lld is not a multiple of the group %lld", (long long)K, (long long)group);
  if (M == 0 || N == 0) return QG_OK;
  if (!y) return fail(QG_ERR_INVALID_ARG, "y is NULL");
  if (ldy < N) return fail(QG_ERR_INVALID_ARG, "ldy %lld < N %lld", (long long)ldy, (long long)N);
  QG_TRY(check_vec(y, 2, "y", false));
  QG_TRY(check_vec(bias, 4, "bias", true));
  QG_TRY(check_device());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return launch_fill_bias(bias, y, QG_F16, ldy, M, N, s);
  QG_TRY(check_matrix(x, ldx, K, 2, "x"));
  QG_TRY(check_matrix(qweight, K / 8, K / 8, 4, "qweight"));
  QG_TRY(check_vec(scale, 16, "scale", false));
  if (N % 8 != 0) return fail(QG_ERR_ALIGNMENT, "N=%lld: the scale rows must be 16-byte multiples (N %% 8 == 0)", (long long)N);
  return launch_w4a16_sym(x, ldx, qweight, scale, bias, y, ldy, M, N, K, s);
}

qg_status qg_gemm_w8a8(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                       const float* x_scale, const float* w_scale, const float* bias, void* y,
                       int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                       void* workspace, size_t workspace_bytes, qg_stream_t stream) {
  return gemm_w8a8(xq, ldx, wq, ldw, x_scale, w_scale, bias, y, y_dtype, ldy, M, N, K, workspace,
                   workspace_bytes, QG_ACT_NONE, 0u, stream);
}

qg_status qg_gemm_w8a8_ex(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                          const float* x_scale, const float* w_scale, const float* bias, void* y,
                          int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                          void* workspace, size_t workspace_bytes, unsigned flags, qg_stream_t stream) {
  return gemm_w8a8(xq, ldx, wq, ldw, x_scale, w_scale, bias, y, y_dtype, ldy, M, N, K, workspace,
                   workspace_bytes, QG_ACT_NONE, flags, stream);
}

qg_status qg_gemm_w8a8_act(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                           const float* x_scale, const float* w_scale, const float* bias, void* y,
                           int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K, int activation,
                           qg_stream_t stream) {
  return gemm_w8a8(xq, ldx, wq, ldw, x_scale, w_scale, bias, y, y_dtype, ldy, M, N, K, nullptr, 0,
                   activation, 0u, stream);
}

qg_status qg_gemm_w8a16(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                        const float* w_scale, const float* bias, void* y, int64_t ldy, int64_t M,
                        int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        qg_stream_t stream) {
  return gemm_w8a16(x, ldx, wq, ldw, w_scale, bias, y, ldy, M, N, K, workspace, workspace_bytes,
                    QG_ACT_NONE, 0u, stream);
}

qg_status qg_gemm_w8a16_ex(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                           const float* w_scale, const float* bias, void* y, int64_t ldy, int64_t M,
                           int64_t N, int64_t K, void* workspace, size_t workspace_bytes, unsigned flags,
                           qg_stream_t stream) {
  return gemm_w8a16(x, ldx, wq, ldw, w_scale, bias, y, ldy, M, N, K, workspace, workspace_bytes,
                    QG_ACT_NONE, flags, stream);
}

qg_status qg_gemm_w8a16_act(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                            const float* w_scale, const float* bias, void* y, int64_t ldy, int64_t M,
                            int64_t N, int64_t K, int activation, qg_stream_t stream) {
  return gemm_w8a16(x, ldx, wq, ldw, w_scale, bias, y, ldy, M, N, K, nullptr, 0, activation, 0u, stream);
}

qg_status qg_gemm_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                        const void* zero, int64_t group, const float* bias, void* y, int64_t ldy,
                        int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        qg_stream_t stream) {
  return gemm_w4a16(x, ldx, qweight, scale, zero, group, bias, y, ldy, M, N, K, workspace,
                    workspace_bytes, QG_ACT_NONE, 0u, stream);
}

qg_status qg_gemm_w4a16_ex(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                           const void* zero, int64_t group, const float* bias, void* y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                           unsigned flags, qg_stream_t stream) {
  return gemm_w4a16(x, ldx, qweight, scale, zero, group, bias, y, ldy, M, N, K, workspace,
                    workspace_bytes, QG_ACT_NONE, flags, stream);
}

qg_status qg_gemm_w4a16_act(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                            const void* zero, int64_t group, const float* bias, void* y, int64_t ldy,
                            int64_t M, int64_t N, int64_t K, int activation, qg_stream_t stream) {
  return gemm_w4a16(x, ldx, qweight, scale, zero, group, bias, y, ldy, M, N, K, nullptr, 0, activation,
                    0u, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Launch plans: the bound arguments of one entry point, replayed on a stream.
// A launch goes through the same internal entry as the direct call, argument
// checks included, so both return the same status for the same arguments.
// ---------------------------------------------------------------------------
struct qg_plan {
  enum Op { kQuantize, kW8A8, kW8A16, kW4A16 } op;
  const void* x;     // x (fp16) or xq (int8)
  int64_t ldx;
  const void* w;     // wq, or qweight
  int64_t ldw;
  const void* s0;    // x_scale (quantize: the x_scale output; W8A8), w_scale (W8A16), scale (W4A16)
  const void* s1;    // w_scale (W8A8), zero (W4A16)
  const float* bias;
  void* y;           // y, or xq (quantize)
  int y_dtype;
  int64_t ldy;       // ldy, or ldxq (quantize)
  int64_t M, N, K, group;
  void* workspace;
  size_t workspace_bytes;
  unsigned flags;
};

namespace {

qg_status new_plan(qg_plan** out, const qg_plan& p) {
  if (!out) return fail(QG_ERR_INVALID_ARG, "plan is NULL");
  *out = nullptr;
  qg_plan* h = new (std::nothrow) qg_plan(p);
  if (!h) return fail(QG_ERR_UNSUPPORTED, "out of host memory for a plan");
  *out = h;
  return QG_OK;
}

}  // namespace

extern "C" {

qg_status qg_plan_quantize_rowwise_int8(qg_plan** plan, const void* x, int64_t ldx, int8_t* xq, int64_t ldxq,
                                        float* x_scale, int64_t M, int64_t K) {
  qg_plan p = {};
  p.op = qg_plan::kQuantize;
  p.x = x;
  p.ldx = ldx;
  p.y = xq;
  p.ldy = ldxq;
  p.s0 = x_scale;
  p.M = M;
  p.K = K;
  return new_plan(plan, p);
}

qg_status qg_plan_gemm_w8a8(qg_plan** plan, const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                            const float* x_scale, const float* w_scale, const float* bias, void* y, int y_dtype,
                            int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                            unsigned flags) {
  qg_plan p = {};
  p.op = qg_plan::kW8A8;
  p.x = xq;
  p.ldx = ldx;
  p.w = wq;
  p.ldw = ldw;
  p.s0 = x_scale;
  p.s1 = w_scale;
  p.bias = bias;
  p.y = y;
  p.y_dtype = y_dtype;
  p.ldy = ldy;
  p.M = M;
  p.N = N;
  p.K = K;
  p.workspace = workspace;
  p.workspace_bytes = workspace_bytes;
  p.flags = flags;
  return new_plan(plan, p);
}

qg_status qg_plan_gemm_w8a16(qg_plan** plan, const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                             const float* w_scale, const float* bias, void* y, int64_t ldy, int64_t M, int64_t N,
                             int64_t K, void* workspace, size_t workspace_bytes, unsigned flags) {
  qg_plan p = {};
  p.op = qg_plan::kW8A16;
  p.x = x;
  p.ldx = ldx;
  p.w = wq;
  p.ldw = ldw;
  p.s0 = w_scale;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.M = M;
  p.N = N;
  p.K = K;
  p.workspace = workspace;
  p.workspace_bytes = workspace_bytes;
  p.flags = flags;
  return new_plan(plan, p);
}

qg_status qg_plan_gemm_w4a16(qg_plan** plan, const void* x, int64_t ldx, const int32_t* qweight,
                             const void* scale, const void* zero, int64_t group, const float* bias, void* y,
                             int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                             size_t workspace_bytes, unsigned flags) {
  qg_plan p = {};
  p.op = qg_plan::kW4A16;
  p.x = x;
  p.ldx = ldx;
  p.w = qweight;
  p.s0 = scale;
  p.s1 = zero;
  p.group = group;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.M = M;
  p.N = N;
  p.K = K;
  p.workspace = workspace;
  p.workspace_bytes = workspace_bytes;
  p.flags = flags;
  return new_plan(plan, p);
}

qg_status qg_plan_launch(const qg_plan* p, qg_stream_t stream) {
  if (!p) return fail(QG_ERR_INVALID_ARG, "plan is NULL");
  switch (p->op) {
    case qg_plan::kQuantize:
      return qg_quantize_rowwise_int8(p->x, p->ldx, static_cast<int8_t*>(p->y), p->ldy,
                                      static_cast<float*>(const_cast<void*>(p->s0)), p->M, p->K, stream);
    case qg_plan::kW8A8:
      return gemm_w8a8(static_cast<const int8_t*>(p->x), p->ldx, static_cast<const int8_t*>(p->w), p->ldw,
                       static_cast<const float*>(p->s0), static_cast<const float*>(p->s1), p->bias, p->y,
                       p->y_dtype, p->ldy, p->M, p->N, p->K, p->workspace, p->workspace_bytes, QG_ACT_NONE,
                       p->flags, stream);
    case qg_plan::kW8A16:
      return gemm_w8a16(p->x, p->ldx, static_cast<const int8_t*>(p->w), p->ldw, static_cast<const float*>(p->s0),
                        p->bias, p->y, p->ldy, p->M, p->N, p->K, p->workspace, p->workspace_bytes, QG_ACT_NONE,
                        p->flags, stream);
    case qg_plan::kW4A16:
      return gemm_w4a16(p->x, p->ldx, static_cast<const int32_t*>(p->w), p->s0, p->s1, p->group, p->bias, p->y,
                        p->ldy, p->M, p->N, p->K, p->workspace, p->workspace_bytes, QG_ACT_NONE, p->flags,
                        stream);
  }
  return fail(QG_ERR_INVALID_ARG, "plan of unknown kind");
}

void qg_plan_destroy(qg_plan* plan) { delete plan; }

}  // extern "C"
