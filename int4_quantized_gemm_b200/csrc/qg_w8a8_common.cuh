// qg_w8a8_common.cuh -- parameters and epilogue helpers shared by the W8A8
// kernels (one-SM tiles in qg_gemm_w8a8.cu, CTA-pair tiles in
// qg_gemm_w8a8_pair.cu): the kernel parameter block, the tile order, output
// conversion/stores and the zero-point correction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/qg.h"

namespace qg {

constexpr int kBK = 128;  // bytes of K per stage (one 128-byte swizzle row)

struct W8A8Params {
  int M, N, K;
  int tiles_a, tiles_b;  // tiles along the A rows (MMA M) and B rows (MMA N)
  int nkb;               // number of K blocks of kBK
  int splits;            // CTAs per cluster sharing one tile along K (decode)
  const float* x_scale;
  const float* w_scale;
  // fused quantize + decode only: fp16 X, and optional copies of its codes/scales
  const __half* x;
  int64_t ldx;
  int8_t* xq_out;
  int64_t ldxq;
  float* xs_out;
  // zero-point W8A8 only (each nullable): per-row zero points and code sums
  const float* x_zero;
  const int32_t* x_qsum;
  const float* w_zero;
  const int32_t* w_qsum;
  const float* bias;
  void* y;
  int64_t ldy;
  int out_dtype;
  int act;  // qg_activation applied to the fp32 value before the output conversion
  // Decode (swap-AB) only: the caller guarantees that no kernel still in
  // flight writes the weights, so the first ring stages of weight tiles are
  // loaded before the wait on the preceding kernel.
  int static_w;
  // CTA-pair prefill only: output columns (MMA N) per pair tile, a multiple of
  // 16 in 128..256; each CTA stages pair_n / 2 rows of Wq per K block.
  int pair_n;
};

// Map a tile index to (tile along A rows, tile along B rows): A tiles vary
// fastest inside groups of 64, so CTAs running at the same time share B tiles
// and the group's A tiles stay in L2 while the B tiles stream past.  For a
// prefill of up to 64 A tiles (M <= 16384 on pair tiles) each operand is then
// read from DRAM about once (8192 x 11008 x 4096: the ~74 tiles in flight hold
// all of X and a few weight columns, ~35 MB); groups of 8 re-read every
// weight tile once per group (180 MB for 45 MB of weights), and measured
// 2-3 % slower there.  Decode launches (one B tile) map tile t to A tile t.
__device__ __forceinline__ void tile_coords(int tile, int tiles_a, int tiles_b, int& ta, int& tb) {
  constexpr int G = 64;
  const int group_size = G * tiles_b;
  const int g = tile / group_size;
  const int first_a = g * G;
  const int ga = min(tiles_a - first_a, G);
  const int local = tile - g * group_size;
  ta = first_a + local % ga;
  tb = local / ga;
}

__device__ __forceinline__ void store_out(void* y, int dtype, int64_t idx, float v, int32_t raw) {
  switch (dtype) {
    case QG_F32: static_cast<float*>(y)[idx] = v; break;
    case QG_F16: static_cast<__half*>(y)[idx] = __float2half_rn(v); break;
    case QG_BF16: static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v); break;
    default: static_cast<int32_t*>(y)[idx] = raw; break;
  }
}

// Zero-point W8A8 (page "量化与多精度算子" §二): with x ~= s_x (q_x - z_x) and
// w ~= s_w (q_w - z_w), sum_k x w = s_x s_w (acc - z_w sum q_x - z_x sum q_w +
// K z_x z_w).  The bracket is formed in fp64 (the correction terms are large
// and nearly cancel), rounded once to fp32, then scaled like the symmetric
// accumulator.
__device__ __forceinline__ float zp_corrected(int32_t acc, float xz, int32_t xsum, float wz, int32_t wsum,
                                              int K) {
  const double t = (double)acc - (double)wz * (double)xsum - (double)xz * (double)wsum +
                   (double)K * (double)xz * (double)wz;
  return (float)t;
}

// 16 consecutive outputs of one row: vector stores when aligned, else scalar.
__device__ __forceinline__ void store_row16(void* y, int dtype, int64_t base, int ncols_valid,
                                            const float (&v)[16], const uint32_t (&raw)[16]) {
  const int esize = dtype == QG_F16 || dtype == QG_BF16 ? 2 : 4;
  char* p = static_cast<char*>(y) + base * esize;
  const bool vec = ncols_valid == 16 && ((reinterpret_cast<uintptr_t>(p) & 15) == 0);
  if (vec) {
    if (dtype == QG_F16) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        __half2 h = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      reinterpret_cast<uint4*>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      reinterpret_cast<uint4*>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else if (dtype == QG_BF16) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      reinterpret_cast<uint4*>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      reinterpret_cast<uint4*>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else if (dtype == QG_F32) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<float4*>(p)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<uint4*>(p)[j] = make_uint4(raw[4 * j], raw[4 * j + 1], raw[4 * j + 2], raw[4 * j + 3]);
    }
  } else {
    for (int j = 0; j < ncols_valid; ++j) store_out(y, dtype, base + j, v[j], (int32_t)raw[j]);
  }
}

// Prefill W8A8 on 256 x 256 tiles of two-CTA clusters (qg_gemm_w8a8_pair.cu);
// p carries M, N, K, nkb, the scales, bias, output and epilogue fields.
template <bool ZP>
qg_status launch_w8a8_pair(W8A8Params p, const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                           cudaStream_t s);

}  // namespace qg
