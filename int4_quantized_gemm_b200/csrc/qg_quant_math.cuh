// qg_quant_math.cuh -- the per-row int8 quantizer's arithmetic, shared by the
// stand-alone quantize kernel and the fused quantize + W8A8 decode kernel so
// that both take every code decision with the same binary32 operations.
//
// Page "量化算法的本质", per_channel_quant_int8 (symmetric branch); page
// "量化与多精度算子" §二 (z = 0, range [-127, 127]) and §六 (rounding):
//   a = max(max_k |x[k]|, 1e-10);  inv = 127 / a;
//   q[k] = clamp(rint(x[k] * inv), -127, 127);  scale = a / 127.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace qg {

// running max |x| over 8 fp16 values (exact: max is order-independent)
__device__ __forceinline__ float absmax8(uint4 v, float a) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return a;
}

// inv = 127 / max(amax, 1e-10)  (binary32, round to nearest even)
__device__ __forceinline__ float quant_inv(float amax) { return __fdiv_rn(127.0f, fmaxf(amax, 1e-10f)); }

// x_scale = max(amax, 1e-10) / 127
__device__ __forceinline__ float quant_scale(float amax) { return __fdiv_rn(fmaxf(amax, 1e-10f), 127.0f); }

__device__ __forceinline__ int quant1(float x, float inv) {
  int q = __float2int_rn(__fmul_rn(x, inv));  // binary32 product, then half-to-even
  return max(-127, min(127, q));
}

// 8 fp16 -> 8 int8 codes, low byte first
__device__ __forceinline__ uint2 quant8(uint4 v, float inv) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t w[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float2 f0 = __half22float2(h[2 * j]);
    float2 f1 = __half22float2(h[2 * j + 1]);
    uint32_t b0 = (uint32_t)(quant1(f0.x, inv) & 0xFF);
    uint32_t b1 = (uint32_t)(quant1(f0.y, inv) & 0xFF);
    uint32_t b2 = (uint32_t)(quant1(f1.x, inv) & 0xFF);
    uint32_t b3 = (uint32_t)(quant1(f1.y, inv) & 0xFF);
    w[j] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
  }
  return make_uint2(w[0], w[1]);
}

// ---------------------------------------------------------------------------
// Asymmetric per-row int8 (page "量化算法的本质", per_channel_quant_int8,
// asymmetric branch), binary32 in the page's order:
//   s = max((max - min) / 255, 1e-8);  z = -min / s - 128  (not rounded);
//   q = clamp(rint(x / s + z), -128, 127).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float asym_scale(float mn, float mx) {
  return fmaxf(__fdiv_rn(__fsub_rn(mx, mn), 255.0f), 1e-8f);
}

__device__ __forceinline__ float asym_zero(float mn, float s) { return __fsub_rn(__fdiv_rn(-mn, s), 128.0f); }

__device__ __forceinline__ int quant1_asym(float x, float s, float z) {
  const float r = rintf(__fadd_rn(__fdiv_rn(x, s), z));
  return (int)fminf(fmaxf(r, -128.0f), 127.0f);
}

// ---------------------------------------------------------------------------
// Symmetric int4 (page "INT4/FP16混合精度GEMM" §5.1: scale = max|w| / 7,
// q = round(w / scale), range [-8, 7]); two's-complement nibbles.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int quant1_sym4(float w, float s) {
  return (int)fminf(fmaxf(rintf(__fdiv_rn(w, s)), -8.0f), 7.0f);
}

}  // namespace qg
