// Device helpers shared by the small-M kernels (the one-problem kernel in
// small_m.cu and the grouped kernel in small_m_grouped.cu): launch-overlap
// controls, the warp-level bf16 MMA, bulk copies, bounded warp waits and the
// code -> bf16 decode of one quad thread's packed word.
#pragma once

#include <cuda.h>

#include "dequant.cuh"
#include "small_m_layout.cuh"

namespace qg {
namespace sm {

using ptx::griddep_launch_dependents;
using ptx::griddep_wait;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t lim, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, lim, abort);
  return __all_sync(0xffffffffu, ok);
}


// The A operand of one MMA step from a packed word: its codes
// 4 quad .. 4 quad + 3 as two bf16x2 registers (code pairs (0, 1) and (2, 3)
// of the four).
template <int BITS>
__device__ __forceinline__ void decode_quad(uint32_t x, int quad, uint32_t& b0, uint32_t& b1) {
  if constexpr (BITS == 1) {
    // in-word offsets 4 quad .. +3 are bits i, 16 + i for i = 2 quad, 2 quad + 1:
    // bf16 {-1, +1}, the sign set where the code bit is 0 (moved to bits 15 and 31)
    const int i0 = 2 * quad;
    b0 = ((~x << (15 - i0)) & 0x80008000u) | 0x3F803F80u;
    b1 = ((~x << (14 - i0)) & 0x80008000u) | 0x3F803F80u;
  } else if constexpr (BITS == 2) {
    // pairs 2 quad and 2 quad + 1 of the 16-code word: bf16 {-2, 0, +2}
    b0 = (x << (14 - 4 * quad)) & 0xC000C000u;
    b1 = (x << (12 - 4 * quad)) & 0xC000C000u;
  } else if constexpr (BITS == 4) {
    // pairs 2 quad and 2 quad + 1 of the 8-code word: bf16 128 + q
    const int sh = 8 * quad;
    b0 = ((x >> sh) & 0x000F000Fu) | 0x43004300u;
    b1 = ((x >> (sh + 4)) & 0x000F000Fu) | 0x43004300u;
  } else {
    // byte j is code j of the word (quad 0); exact q through an fp32 magic number
    (void)quad;
    const float2 q01 = ptx::add2(make_float2(__uint_as_float(ptx::prmt(x, deq::kMagic, 0x7650u)),
                                             __uint_as_float(ptx::prmt(x, deq::kMagic, 0x7651u))),
                                 make_float2(-deq::kMagicF, -deq::kMagicF));
    const float2 q23 = ptx::add2(make_float2(__uint_as_float(ptx::prmt(x, deq::kMagic, 0x7652u)),
                                             __uint_as_float(ptx::prmt(x, deq::kMagic, 0x7653u))),
                                 make_float2(-deq::kMagicF, -deq::kMagicF));
    b0 = ptx::cvt_bf16x2(q01.x, q01.y);
    b1 = ptx::cvt_bf16x2(q23.x, q23.y);
  }
}

// A thread's packed chunk of one row and group (Chunk<BITS>::BYTES bytes at a
// 4-, 8- or 16-byte aligned shared-memory address) as 32-bit words.
template <int BITS>
__device__ __forceinline__ void load_chunk(const uint8_t* p, uint32_t (&w)[Chunk<BITS>::WORDS]) {
  if constexpr (Chunk<BITS>::BYTES == 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
  } else if constexpr (Chunk<BITS>::BYTES == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// The activation fragment of step s from a thread's chunk of one token row
// (G / 4 consecutive bf16 held as 16-byte pieces): 4 bf16 at k 4s .. 4s + 3.
template <int XV>
__device__ __forceinline__ uint2 x_step(const uint4 (&v)[XV], int s) {
  const uint4 p = v[s >> 1];
  return (s & 1) ? make_uint2(p.z, p.w) : make_uint2(p.x, p.y);
}

}  // namespace sm
}  // namespace qg
