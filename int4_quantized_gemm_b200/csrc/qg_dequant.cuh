// qg_dequant.cuh -- on-chip dequantization of int8 / int4 weight codes into the
// fp16 A operand of the weight-only GEMMs (shared by the cluster split-K and
// stream-K kernels).  Page "量化与多精度算子" §四 (weights stored as INT8/INT4,
// dequantized to FP16 inside the kernel); page "INT4/FP16混合精度GEMM" §3.2/§4.2
// ((w >> 4i) & 0xF, (q - zp) * scale).
#pragma once

#include <stdint.h>

namespace qg {

// The dequantizers below work on fp16x2 values held in plain 32-bit registers
// (inline PTX), so no value is ever split into or rebuilt from 16-bit halves.

// int8 x4 (one 32-bit word, k..k+3) -> two fp16x2 (k, k+1), (k+2, k+3): biased to
// unsigned, placed in the low byte of fp16 1024 + u, then 1024 + 128 subtracted
// (all exact).
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b32 u;\n\t"
      "xor.b32 u, %2, 0x80808080;\n\t"
      "prmt.b32 %0, u, 0x64646464, 0x5140;\n\t"
      "prmt.b32 %1, u, 0x64646464, 0x7362;\n\t"
      "sub.rn.f16x2 %0, %0, %3;\n\t"
      "sub.rn.f16x2 %1, %1, %3;\n\t}"
      : "=&r"(lo), "=&r"(hi)
      : "r"(w), "r"(0x64806480u));  // 1152 in both halves
}

// 8 nibbles (k..k+7, nibble j at bits 4j) -> four fp16x2 of (q - z) * s in the
// pair order (k, k+4), (k+1, k+5), (k+2, k+6), (k+3, k+7): the order in which
// masking the word yields them, so no byte permutes are needed (X is permuted
// the same way inside every 8-element group, see permute_x_chunk).  The
// magic exponent 0x64 turns a nibble at bits 0..3 of a half into 1024 + q and
// one at bits 4..7 into 1024 + 16q; one add (or fma by 1/16) makes q - z
// exactly, one multiply rounds (q - z) * s.  c_lo = -(1024 + z) and
// c_hi = -(64 + z) in both halves, s2 = s in both halves.  The masked nibbles
// are combined with the magic by xor ((a & b) ^ c, equal to an or since the
// magic has no bits under the mask); m_lo / m_hi are the magic with, for
// two's-complement codes, the nibble sign bits also set, which turns each code
// q into its offset form q + 8 (then z = 8) at no extra cost.
__device__ __forceinline__ void u4x8_to_h2x4(uint32_t w, uint32_t s2, uint32_t c_lo, uint32_t c_hi,
                                             uint32_t m_lo, uint32_t m_hi, uint32_t* o) {
  asm("{\n\t.reg .b32 t0, t1, t2, t3, w8;\n\t"
      "lop3.b32 t0, %4, 0x000F000F, %9, 0x6A;\n\t"   // (a & b) ^ c
      "lop3.b32 t1, %4, 0x00F000F0, %10, 0x6A;\n\t"
      "shr.b32 w8, %4, 8;\n\t"
      "lop3.b32 t2, w8, 0x000F000F, %9, 0x6A;\n\t"
      "lop3.b32 t3, w8, 0x00F000F0, %10, 0x6A;\n\t"
      "add.rn.f16x2 t0, t0, %6;\n\t"
      "fma.rn.f16x2 t1, t1, %8, %7;\n\t"                     // x 1/16
      "add.rn.f16x2 t2, t2, %6;\n\t"
      "fma.rn.f16x2 t3, t3, %8, %7;\n\t"
      "mul.rn.f16x2 %0, t0, %5;\n\t"
      "mul.rn.f16x2 %1, t1, %5;\n\t"
      "mul.rn.f16x2 %2, t2, %5;\n\t"
      "mul.rn.f16x2 %3, t3, %5;\n\t}"
      : "=&r"(o[0]), "=&r"(o[1]), "=&r"(o[2]), "=&r"(o[3])  // written before s2 is last read
      : "r"(w), "r"(s2), "r"(c_lo), "r"(c_hi), "r"(0x2C002C00u),  // 1/16 in both halves
        "r"(m_lo), "r"(m_hi));
}

// Per-group constants of u4x8_to_h2x4 from the fp16 bit patterns of the scale
// s and zero point z: s2 = (s, s), c_lo = -(1024 + z), c_hi = -(64 + z) in both
// halves.  The two subtractions run in fp16x2 and round once, exactly as the
// binary32 difference rounded to fp16 would (for integer z in 0..15 they are
// exact), with no conversion instructions.
__device__ __forceinline__ void u4_group_consts(uint32_t s_bits, uint32_t z_bits, uint32_t& s2, uint32_t& c_lo,
                                                uint32_t& c_hi) {
  asm("{\n\t.reg .b32 z2;\n\t"
      "prmt.b32 %0, %3, 0, 0x1010;\n\t"
      "prmt.b32 z2, %4, 0, 0x1010;\n\t"
      "sub.rn.f16x2 %1, %5, z2;\n\t"
      "sub.rn.f16x2 %2, %6, z2;\n\t}"
      : "=&r"(s2), "=&r"(c_lo), "=r"(c_hi)
      : "r"(s_bits), "r"(z_bits), "r"(0xE400E400u), "r"(0xD400D400u));  // -1024, -64 in both halves
}

// Reorder one 16-byte chunk of X (8 consecutive k) to k = 0,4,1,5,2,6,3,7,
// matching the A operand's pair order above.  The dot product over the chunk
// is unchanged because A and B use the same order.
__device__ __forceinline__ void permute_x_chunk(uint8_t* p) {
  uint4 v = *reinterpret_cast<uint4*>(p);
  uint4 o;
  o.x = __byte_perm(v.x, v.z, 0x5410);  // (x0, x4)
  o.y = __byte_perm(v.x, v.z, 0x7632);  // (x1, x5)
  o.z = __byte_perm(v.y, v.w, 0x5410);  // (x2, x6)
  o.w = __byte_perm(v.y, v.w, 0x7632);  // (x3, x7)
  *reinterpret_cast<uint4*>(p) = o;
}

// 8 two's-complement nibbles (k..k+7, nibble j at bits 4j) -> 8 int8 in k order
// (lo: k..k+3, hi: k+4..k+7).  Even and odd nibbles are masked into bytes and
// sign-extended per byte without carries between bytes: with b in [0, 15],
// ((b ^ 0x88) - 0x08) ^ 0x80 = b - 16 * (b >> 3) as an int8 (setting bit 7
// first keeps the subtraction from borrowing across bytes); then a byte
// interleave puts the codes in k order.
__device__ __forceinline__ void s4x8_to_s8x8(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b32 e, o;\n\t"
      "lop3.b32 e, %2, 0x0F0F0F0F, 0x88888888, 0x6A;\n\t"   // (w & 0x0F..) ^ 0x88..
      "shr.b32 o, %2, 4;\n\t"
      "lop3.b32 o, o, 0x0F0F0F0F, 0x88888888, 0x6A;\n\t"
      "sub.u32 e, e, 0x08080808;\n\t"
      "sub.u32 o, o, 0x08080808;\n\t"
      "xor.b32 e, e, 0x80808080;\n\t"                         // codes k, k+2, k+4, k+6
      "xor.b32 o, o, 0x80808080;\n\t"                         // codes k+1, k+3, k+5, k+7
      "prmt.b32 %0, e, o, 0x5140;\n\t"
      "prmt.b32 %1, e, o, 0x7362;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

}  // namespace qg
