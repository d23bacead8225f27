// qg_quantize.cu -- quantization kernels (memory-bound, CUDA cores).
//
//  * quantize_rowwise: symmetric per-row int8 (dynamic per-token activation
//    quantization; also the per-output-column int8 weight quantizer when run
//    on the [N,K] storage of a column-major weight).  Page "量化算法的本质",
//    per_channel_quant_int8 (symmetric branch); page "量化与多精度算子" §二, §六.
//  * quantize_block_asym4: block-64 asymmetric 4-bit weights + nibble packing.
//    Page "从零实现大语言模型 INT8 量化" 第一步/第二步; page "INT4/FP16混合精度GEMM"
//    §3.1, §4.2; scale floor 1e-5 from page "量化算法的本质" (GPTQ MARLIN).
//
// Every floating-point step that decides a code is an explicit IEEE binary32
// intrinsic with round-to-nearest-even (__fdiv_rn, __fmul_rn, rintf), so the
// codes and scales are bit-exact with any correct IEEE implementation of the
// same formulas.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qg_device.cuh"
#include "qg_internal.h"
#include "qg_quant_math.cuh"

namespace qg {

static __device__ unsigned long long g_status_quantize;

unsigned long long read_clear_status_quantize(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_quantize, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_quantize, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

// One group of THREADS_PER_ROW threads per row; ROWS rows per block.
// Pass 1 reads the row (128-bit loads) for the absmax; pass 2 writes 8 codes
// per 64-bit store.  With CACHE > 0 the row is at most CACHE vectors per thread
// (K <= 8 * CACHE * THREADS_PER_ROW) and pass 2 takes them from registers;
// with CACHE = 0 it re-reads the row (from L1/L2).  Rows are 16-byte aligned (ABI).
template <int THREADS_PER_ROW, int ROWS, int CACHE>
__global__ void __launch_bounds__(THREADS_PER_ROW* ROWS)
    quantize_rowwise_kernel(const __half* __restrict__ x, int64_t ldx, int8_t* __restrict__ xq,
                            int64_t ldq, float* __restrict__ xs, int M, int K) {
  constexpr int WARPS_PER_ROW = THREADS_PER_ROW / 32;
  __shared__ float red[ROWS][WARPS_PER_ROW];
  pdl_trigger();
  pdl_wait();
  const int r = threadIdx.x / THREADS_PER_ROW;
  const int t = threadIdx.x % THREADS_PER_ROW;
  const int m = blockIdx.x * ROWS + r;
  const bool active = m < M;
  const __half* row = x + (int64_t)(active ? m : 0) * ldx;
  const uint4* rowv = reinterpret_cast<const uint4*>(row);
  const int nvec = K / 8;

  float a = 0.0f;
  uint4 v[CACHE > 0 ? CACHE : 1];
  if (active) {
    if (CACHE > 0) {
#pragma unroll
      for (int j = 0; j < CACHE; ++j) {
        const int i = t + j * THREADS_PER_ROW;
        v[j] = i < nvec ? __ldg(rowv + i) : make_uint4(0u, 0u, 0u, 0u);  // zeros leave the max unchanged
      }
#pragma unroll
      for (int j = 0; j < CACHE; ++j) a = absmax8(v[j], a);
    } else {
      for (int i = t; i < nvec; i += THREADS_PER_ROW) a = absmax8(__ldg(rowv + i), a);
    }
    for (int k = nvec * 8 + t; k < K; k += THREADS_PER_ROW) a = fmaxf(a, fabsf(__half2float(row[k])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (WARPS_PER_ROW > 1) {
    if ((t & 31) == 0) red[r][t / 32] = a;
    __syncthreads();
    a = red[r][0];
#pragma unroll
    for (int w = 1; w < WARPS_PER_ROW; ++w) a = fmaxf(a, red[r][w]);
  }
  if (!active) return;
  const float inv = quant_inv(a);

  int8_t* qrow = xq + (int64_t)m * ldq;
  uint2* qv = reinterpret_cast<uint2*>(qrow);
  if (CACHE > 0) {
#pragma unroll
    for (int j = 0; j < CACHE; ++j) {
      const int i = t + j * THREADS_PER_ROW;
      if (i < nvec) qv[i] = quant8(v[j], inv);
    }
  } else {
    for (int i = t; i < nvec; i += THREADS_PER_ROW) qv[i] = quant8(__ldg(rowv + i), inv);
  }
  for (int k = nvec * 8 + t; k < K; k += THREADS_PER_ROW)
    qrow[k] = (int8_t)quant1(__half2float(row[k]), inv);
  if (t == 0) xs[m] = quant_scale(a);
}

qg_status launch_quantize_rowwise(const void* x, int64_t ldx, int8_t* xq, int64_t ldq, float* xs,
                                  int64_t M, int64_t K, cudaStream_t s) {
  const __half* xh = static_cast<const __half*>(x);
  cudaError_t e;
  // the row stays in registers up to K = 8 x 4 x threads per row (4 vectors a thread)
  if (K <= 1024) {
    constexpr int R = 8;
    LaunchCfg lc((unsigned)((M + R - 1) / R), 32 * R, 0, s);
    e = cudaLaunchKernelEx(&lc.cfg, quantize_rowwise_kernel<32, R, 4>, xh, ldx, xq, ldq, xs, (int)M, (int)K);
  } else if (K <= 4096) {
    constexpr int R = 2;
    LaunchCfg lc((unsigned)((M + R - 1) / R), 128 * R, 0, s);
    e = cudaLaunchKernelEx(&lc.cfg, quantize_rowwise_kernel<128, R, 4>, xh, ldx, xq, ldq, xs, (int)M, (int)K);
  } else {
    LaunchCfg lc((unsigned)M, 512, 0, s);
    e = cudaLaunchKernelEx(&lc.cfg, quantize_rowwise_kernel<512, 1, 0>, xh, ldx, xq, ldq, xs, (int)M, (int)K);
  }
  return check_cuda(e, "quantize_rowwise launch");
}

// ---------------------------------------------------------------------------
// Asymmetric per-row int8: min/max pass, then codes and their row sum.
// ---------------------------------------------------------------------------
template <int THREADS_PER_ROW, int ROWS>
__global__ void __launch_bounds__(THREADS_PER_ROW* ROWS)
    quantize_rowwise_asym_kernel(const __half* __restrict__ x, int64_t ldx, int8_t* __restrict__ xq,
                                 int64_t ldq, float* __restrict__ xs, float* __restrict__ xz,
                                 int32_t* __restrict__ qsum, int M, int K) {
  constexpr int WARPS_PER_ROW = THREADS_PER_ROW / 32;
  __shared__ float red_mn[ROWS][WARPS_PER_ROW], red_mx[ROWS][WARPS_PER_ROW];
  __shared__ int red_sum[ROWS][WARPS_PER_ROW];
  pdl_trigger();
  pdl_wait();
  const int r = threadIdx.x / THREADS_PER_ROW;
  const int t = threadIdx.x % THREADS_PER_ROW;
  const int m = blockIdx.x * ROWS + r;
  const bool active = m < M;
  const __half* row = x + (int64_t)(active ? m : 0) * ldx;
  const uint4* rowv = reinterpret_cast<const uint4*>(row);
  const int nvec = K / 8;

  float mn = INFINITY, mx = -INFINITY;
  if (active) {
    for (int i = t; i < nvec; i += THREADS_PER_ROW) {
      const uint4 v = __ldg(rowv + i);
      const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        mn = fminf(mn, fminf(f.x, f.y));
        mx = fmaxf(mx, fmaxf(f.x, f.y));
      }
    }
    for (int k = nvec * 8 + t; k < K; k += THREADS_PER_ROW) {
      const float f = __half2float(row[k]);
      mn = fminf(mn, f);
      mx = fmaxf(mx, f);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (WARPS_PER_ROW > 1) {
    if ((t & 31) == 0) {
      red_mn[r][t / 32] = mn;
      red_mx[r][t / 32] = mx;
    }
    __syncthreads();
    mn = red_mn[r][0];
    mx = red_mx[r][0];
#pragma unroll
    for (int w = 1; w < WARPS_PER_ROW; ++w) {
      mn = fminf(mn, red_mn[r][w]);
      mx = fmaxf(mx, red_mx[r][w]);
    }
  }
  if (K == 0) mn = mx = 0.0f;  // the empty row: s = 1e-8, z = -128
  const float sc = asym_scale(mn, mx);
  const float z = asym_zero(mn, sc);

  int sum = 0;
  if (active) {
    int8_t* qrow = xq + (int64_t)m * ldq;
    uint2* qv = reinterpret_cast<uint2*>(qrow);
    for (int i = t; i < nvec; i += THREADS_PER_ROW) {
      const uint4 v = __ldg(rowv + i);
      const __half2* h = reinterpret_cast<const __half2*>(&v);
      uint32_t w[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 f0 = __half22float2(h[2 * j]);
        const float2 f1 = __half22float2(h[2 * j + 1]);
        const int c0 = quant1_asym(f0.x, sc, z), c1 = quant1_asym(f0.y, sc, z);
        const int c2 = quant1_asym(f1.x, sc, z), c3 = quant1_asym(f1.y, sc, z);
        sum += c0 + c1 + c2 + c3;
        w[j] = (uint32_t)(c0 & 0xFF) | ((uint32_t)(c1 & 0xFF) << 8) | ((uint32_t)(c2 & 0xFF) << 16) |
               ((uint32_t)(c3 & 0xFF) << 24);
      }
      qv[i] = make_uint2(w[0], w[1]);
    }
    for (int k = nvec * 8 + t; k < K; k += THREADS_PER_ROW) {
      const int c = quant1_asym(__half2float(row[k]), sc, z);
      sum += c;
      qrow[k] = (int8_t)c;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (WARPS_PER_ROW > 1) {
    if ((t & 31) == 0) red_sum[r][t / 32] = sum;
    __syncthreads();
    sum = 0;
#pragma unroll
    for (int w = 0; w < WARPS_PER_ROW; ++w) sum += red_sum[r][w];
  }
  if (active && t == 0) {
    xs[m] = sc;
    xz[m] = z;
    if (qsum) qsum[m] = sum;
  }
}

qg_status launch_quantize_rowwise_asym(const void* x, int64_t ldx, int8_t* xq, int64_t ldq, float* xs,
                                       float* xz, int32_t* qsum, int64_t M, int64_t K, cudaStream_t s) {
  const __half* xh = static_cast<const __half*>(x);
  cudaError_t e;
  if (K <= 1024) {
    constexpr int R = 8;
    LaunchCfg lc((unsigned)((M + R - 1) / R), 32 * R, 0, s);
    e = cudaLaunchKernelEx(&lc.cfg, quantize_rowwise_asym_kernel<32, R>, xh, ldx, xq, ldq, xs, xz, qsum,
                           (int)M, (int)K);
  } else if (K <= 4096) {
    constexpr int R = 2;
    LaunchCfg lc((unsigned)((M + R - 1) / R), 128 * R, 0, s);
    e = cudaLaunchKernelEx(&lc.cfg, quantize_rowwise_asym_kernel<128, R>, xh, ldx, xq, ldq, xs, xz, qsum,
                           (int)M, (int)K);
  } else {
    LaunchCfg lc((unsigned)M, 512, 0, s);
    e = cudaLaunchKernelEx(&lc.cfg, quantize_rowwise_asym_kernel<512, 1>, xh, ldx, xq, ldq, xs, xz, qsum,
                           (int)M, (int)K);
  }
  return check_cuda(e, "quantize_rowwise_asym launch");
}

// ---------------------------------------------------------------------------
// Block-64 asymmetric 4-bit quantization: one warp per (column n, block b).
// Lane l holds k = 64b + 2l and 64b + 2l + 1.
// ---------------------------------------------------------------------------
constexpr int kGroup = 64;

__global__ void __launch_bounds__(256)
    quantize_block_asym4_kernel(const __half* __restrict__ w, int64_t ldw,
                                uint32_t* __restrict__ qweight, __half* __restrict__ scale,
                                __half* __restrict__ zero, int N, int K) {
  pdl_trigger();
  pdl_wait();
  const int warp = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int nblk = K / kGroup;
  if (warp >= N * nblk) return;
  const int n = warp / nblk;
  const int b = warp % nblk;

  const __half2 h = reinterpret_cast<const __half2*>(w + (int64_t)n * ldw + b * kGroup)[lane];
  const float2 v = __half22float2(h);
  float mn = fminf(v.x, v.y), mx = fmaxf(v.x, v.y);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float s32 = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), 15.0f), 1e-5f);
  const __half sh = __float2half_rn(s32);
  const float s = __half2float(sh);
  const float zr = rintf(__fdiv_rn(-mn, s));
  const int zi = zr < 0.0f ? 0 : (zr > 15.0f ? 15 : (int)zr);
  const float z = (float)zi;
  const float t0 = __fadd_rn(rintf(__fdiv_rn(v.x, s)), z);
  const float t1 = __fadd_rn(rintf(__fdiv_rn(v.y, s)), z);
  const uint32_t c0 = (uint32_t)fminf(fmaxf(t0, 0.0f), 15.0f);
  const uint32_t c1 = (uint32_t)fminf(fmaxf(t1, 0.0f), 15.0f);

  // Lanes 4p..4p+3 hold k = 8p..8p+7: gather the eight nibbles into word p.
  uint32_t byte = c0 | (c1 << 4);
  uint32_t word = byte;
  word |= __shfl_down_sync(0xffffffffu, byte, 1) << 8;
  word |= __shfl_down_sync(0xffffffffu, byte, 2) << 16;
  word |= __shfl_down_sync(0xffffffffu, byte, 3) << 24;
  if ((lane & 3) == 0) qweight[(int64_t)n * (K / 8) + b * 8 + (lane >> 2)] = word;
  if (lane == 0) {
    scale[(int64_t)b * N + n] = sh;
    zero[(int64_t)b * N + n] = __float2half_rn(z);
  }
}

// ---------------------------------------------------------------------------
// Block-64 symmetric int4: one warp per (column n, block b), as above;
// s = fp16(max(max|w| / 7, 1e-5)), quantized with the stored fp16 value.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    quantize_block_sym4_kernel(const __half* __restrict__ w, int64_t ldw, uint32_t* __restrict__ qweight,
                               __half* __restrict__ scale, int N, int K) {
  pdl_trigger();
  pdl_wait();
  const int warp = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int nblk = K / kGroup;
  if (warp >= N * nblk) return;
  const int n = warp / nblk;
  const int b = warp % nblk;
  const __half2 h = reinterpret_cast<const __half2*>(w + (int64_t)n * ldw + b * kGroup)[lane];
  const float2 v = __half22float2(h);
  float a = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  const float s32 = fmaxf(__fdiv_rn(a, 7.0f), 1e-5f);
  const __half sh = __float2half_rn(s32);
  const float sc = __half2float(sh);
  const uint32_t c0 = (uint32_t)quant1_sym4(v.x, sc) & 0xFu;
  const uint32_t c1 = (uint32_t)quant1_sym4(v.y, sc) & 0xFu;
  uint32_t byte = c0 | (c1 << 4);
  uint32_t word = byte;
  word |= __shfl_down_sync(0xffffffffu, byte, 1) << 8;
  word |= __shfl_down_sync(0xffffffffu, byte, 2) << 16;
  word |= __shfl_down_sync(0xffffffffu, byte, 3) << 24;
  if ((lane & 3) == 0) qweight[(int64_t)n * (K / 8) + b * 8 + (lane >> 2)] = word;
  if (lane == 0) scale[(int64_t)b * N + n] = sh;
}

// ---------------------------------------------------------------------------
// Per-column symmetric int4 for the int8 tensor path: one block of 128 threads
// per column; s = max(max|w|, 1e-10) / 7 in fp32.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    quantize_channel_sym4_kernel(const __half* __restrict__ w, int64_t ldw, uint32_t* __restrict__ qweight,
                                 float* __restrict__ scale, int N, int K) {
  __shared__ float red[4];
  pdl_trigger();
  pdl_wait();
  const int n = blockIdx.x;
  const int t = threadIdx.x;
  const __half* row = w + (int64_t)n * ldw;
  const uint4* rowv = reinterpret_cast<const uint4*>(row);
  const int nvec = K / 8;  // K % 8 == 0 (ABI)
  float a = 0.0f;
  for (int i = t; i < nvec; i += 128) a = absmax8(__ldg(rowv + i), a);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((t & 31) == 0) red[t >> 5] = a;
  __syncthreads();
  a = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float sc = __fdiv_rn(fmaxf(a, 1e-10f), 7.0f);
  for (int i = t; i < nvec; i += 128) {
    const uint4 v = __ldg(rowv + i);
    const __half2* h = reinterpret_cast<const __half2*>(&v);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(h[j]);
      word |= ((uint32_t)quant1_sym4(f.x, sc) & 0xFu) << (8 * j);
      word |= ((uint32_t)quant1_sym4(f.y, sc) & 0xFu) << (8 * j + 4);
    }
    qweight[(int64_t)n * nvec + i] = word;
  }
  if (t == 0) scale[n] = sc;
}

qg_status launch_quantize_block_sym4(const void* w, int64_t ldw, int32_t* qweight, void* scale, int64_t N,
                                     int64_t K, cudaStream_t s) {
  const int64_t warps = N * (K / kGroup);
  const int64_t blocks = (warps * 32 + 255) / 256;
  LaunchCfg lc((unsigned)blocks, 256, 0, s);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, quantize_block_sym4_kernel, static_cast<const __half*>(w), ldw,
                                       reinterpret_cast<uint32_t*>(qweight), static_cast<__half*>(scale),
                                       (int)N, (int)K),
                    "quantize_block_sym4 launch");
}

qg_status launch_quantize_channel_sym4(const void* w, int64_t ldw, int32_t* qweight, float* scale, int64_t N,
                                       int64_t K, cudaStream_t s) {
  LaunchCfg lc((unsigned)N, 128, 0, s);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, quantize_channel_sym4_kernel, static_cast<const __half*>(w),
                                       ldw, reinterpret_cast<uint32_t*>(qweight), scale, (int)N, (int)K),
                    "quantize_channel_sym4 launch");
}

qg_status launch_quantize_block_asym4(const void* w, int64_t ldw, int32_t* qweight, void* scale,
                                      void* zero, int64_t N, int64_t K, cudaStream_t s) {
  const int64_t warps = N * (K / kGroup);
  const int64_t blocks = (warps * 32 + 255) / 256;
  LaunchCfg lc((unsigned)blocks, 256, 0, s);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, quantize_block_asym4_kernel,
                                       static_cast<const __half*>(w), ldw,
                                       reinterpret_cast<uint32_t*>(qweight),
                                       static_cast<__half*>(scale), static_cast<__half*>(zero),
                                       (int)N, (int)K),
                    "quantize_block_asym4 launch");
}

}  // namespace qg
