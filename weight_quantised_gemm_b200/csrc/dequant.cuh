// Device dequantisation of one 8-element chunk (8 consecutive k of one row)
// into 8 bf16 values packed in a uint4, under the bit-exact contract of
// include/qgemm.h:
//   affine   wdeq = bf16_rn(fp32(s) * q + fp32(b))   (product exact, one FMA)
//   ternary  wdeq = t * bf16_rn(fp32(s))
//   1-bit    wdeq = c * bf16_rn(fp32(s))
// The large-M kernel applies these to every packed tile before writing it to
// tensor memory; qgemm_dequant_tile exposes the same routines for the
// bit-exact gate.
#pragma once

#include "ptx.cuh"

namespace qg {
namespace deq {

// fp32 with bits 0x4B000000 | q equals 2^23 + q for q < 2^23.
constexpr uint32_t kMagic = 0x4B000000u;
constexpr float kMagicF = 8388608.0f;

__device__ __forceinline__ float magic_byte(uint32_t src, uint32_t byte_sel) {
  // bytes [src.byte_sel, 0x00, 0x00, 0x4B] -> 2^23 + that byte
  return __uint_as_float(ptx::prmt(src, kMagic, 0x7650u | byte_sel));
}

// Two codes (already as 2^23 + q floats) -> one bf16x2 of s*q + b.
__device__ __forceinline__ uint32_t affine_pair(float m0, float m1, float2 s2, float2 b2) {
  const float2 q = ptx::add2(make_float2(m0, m1), make_float2(-kMagicF, -kMagicF));  // exact
  const float2 v = ptx::fma2(q, s2, b2);  // s*q exact, one rounding of the sum
  return ptx::cvt_bf16x2(v.x, v.y);
}

// 4-bit: one word = 8 consecutive k. In-word offset 2i sits in bits 4i..4i+3,
// offset 2i+1 in bits 16+4i..19+4i.
__device__ __forceinline__ uint4 chunk_4bit(uint32_t w, float s, float b) {
  const uint32_t lo = w & 0x0F0F0F0Fu;         // bytes: k0, k4, k1, k5
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // bytes: k2, k6, k3, k7
  const float2 s2 = make_float2(s, s), b2 = make_float2(b, b);
  uint4 o;
  o.x = affine_pair(magic_byte(lo, 0), magic_byte(lo, 2), s2, b2);  // k0, k1
  o.y = affine_pair(magic_byte(hi, 0), magic_byte(hi, 2), s2, b2);  // k2, k3
  o.z = affine_pair(magic_byte(lo, 1), magic_byte(lo, 3), s2, b2);  // k4, k5
  o.w = affine_pair(magic_byte(hi, 1), magic_byte(hi, 3), s2, b2);  // k6, k7
  return o;
}

// 8-bit: two words, byte j of word i holds k = 4i + j.
__device__ __forceinline__ uint4 chunk_8bit(uint32_t w0, uint32_t w1, float s, float b) {
  const float2 s2 = make_float2(s, s), b2 = make_float2(b, b);
  uint4 o;
  o.x = affine_pair(magic_byte(w0, 0), magic_byte(w0, 1), s2, b2);
  o.y = affine_pair(magic_byte(w0, 2), magic_byte(w0, 3), s2, b2);
  o.z = affine_pair(magic_byte(w1, 0), magic_byte(w1, 1), s2, b2);
  o.w = affine_pair(magic_byte(w1, 2), magic_byte(w1, 3), s2, b2);
  return o;
}

// Ternary pair i of a word (in-word offsets 2i and 2i+1, codes in bits 2i and
// 16+2i) as bf16x2 of {-2, 0, +2}: the two's-complement code shifted into a
// bf16's top two bits is exactly sign|0x4000.
template <int I>
__device__ __forceinline__ uint32_t ternary_pair_pm2(uint32_t w) {
  return (w << (14 - 2 * I)) & 0xC000C000u;
}

// bf16x2 of bf16_rn(fp32(s)) / 2 in both lanes (halving a bf16 is exact).
__device__ __forceinline__ uint32_t ternary_half_scale2(float s) {
  const float sb = __bfloat162float(__float2bfloat16_rn(s));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(sb * 0.5f));
  return h | (h << 16);
}

// Ternary: 8 consecutive k = one half of a 16-code word (HALF 0: k 0..7).
// (+-2) * (sb/2) = +-sb exactly, and 0 * x = +0.
template <int HALF>
__device__ __forceinline__ uint4 chunk_ternary(uint32_t w, uint32_t half_scale2) {
  uint4 o;
  o.x = ptx::mul_bf16x2(ternary_pair_pm2<4 * HALF + 0>(w), half_scale2);
  o.y = ptx::mul_bf16x2(ternary_pair_pm2<4 * HALF + 1>(w), half_scale2);
  o.z = ptx::mul_bf16x2(ternary_pair_pm2<4 * HALF + 2>(w), half_scale2);
  o.w = ptx::mul_bf16x2(ternary_pair_pm2<4 * HALF + 3>(w), half_scale2);
  return o;
}

__device__ __forceinline__ uint4 chunk_ternary_dyn(uint32_t w, int half, uint32_t half_scale2) {
  return half ? chunk_ternary<1>(w, half_scale2) : chunk_ternary<0>(w, half_scale2);
}

// 1-bit (Q1_0_g128): pair i of a 32-code word (in-word offsets 2i and 2i+1,
// codes in bits i and 16+i; bit 1 = +1) as bf16x2 of +-sb: the scale's bf16
// bits in both lanes with the sign bit set where the code bit is 0. The shift
// brings bits i and 16+i to 15 and 31, the sign positions of the two lanes.
template <int I>
__device__ __forceinline__ uint32_t binary_pair(uint32_t w, uint32_t scale2) {
  return ((~w << (15 - I)) & 0x80008000u) | scale2;
}

// bf16x2 of bf16_rn(fp32(s)) in both lanes.
__device__ __forceinline__ uint32_t bf16_scale2(float s) {
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(s));
  return h | (h << 16);
}

// 1-bit: 8 consecutive k = quarter Q of a 32-code word (Q 0: k 0..7), each
// weight exactly c * bf16_rn(s).
template <int Q>
__device__ __forceinline__ uint4 chunk_binary(uint32_t w, uint32_t scale2) {
  uint4 o;
  o.x = binary_pair<4 * Q + 0>(w, scale2);
  o.y = binary_pair<4 * Q + 1>(w, scale2);
  o.z = binary_pair<4 * Q + 2>(w, scale2);
  o.w = binary_pair<4 * Q + 3>(w, scale2);
  return o;
}

__device__ __forceinline__ uint4 chunk_binary_dyn(uint32_t w, int quarter, uint32_t scale2) {
  switch (quarter) {
    case 0: return chunk_binary<0>(w, scale2);
    case 1: return chunk_binary<1>(w, scale2);
    case 2: return chunk_binary<2>(w, scale2);
    default: return chunk_binary<3>(w, scale2);
  }
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

}  // namespace deq
}  // namespace qg
