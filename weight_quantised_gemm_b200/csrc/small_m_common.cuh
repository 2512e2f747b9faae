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

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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


// B operand of one step for quad thread c from its word: codes 4c .. 4c+3 as
// two bf16x2 registers (k pairs (4c, 4c+1) and (4c+2, 4c+3)).
template <int BITS>
__device__ __forceinline__ void decode_word(uint32_t x, int c, int k, uint32_t& b0, uint32_t& b1) {
  if constexpr (BITS == 1) {
    // pairs 8(k%2) + 2c and +1 of the 32-code word: bf16 {-1, +1}, the sign
    // set where the code bit is 0 (bits i and 16+i moved to 15 and 31)
    const int i0 = 8 * (k & 1) + 2 * c;
    b0 = ((~x << (15 - i0)) & 0x80008000u) | 0x3F803F80u;
    b1 = ((~x << (14 - i0)) & 0x80008000u) | 0x3F803F80u;
  } else if constexpr (BITS == 2) {
    // pairs 2c and 2c+1 of the 16-code word: bf16 {-2, 0, +2}
    b0 = (x << (14 - 4 * c)) & 0xC000C000u;
    b1 = (x << (12 - 4 * c)) & 0xC000C000u;
  } else if constexpr (BITS == 4) {
    // pairs 2(c%2) and 2(c%2)+1 of the 8-code word: bf16 128 + q
    const int sh = 8 * (c & 1);
    b0 = ((x >> sh) & 0x000F000Fu) | 0x43004300u;
    b1 = ((x >> (sh + 4)) & 0x000F000Fu) | 0x43004300u;
  } else {
    // byte j is code 4c + j; exact q through an fp32 magic number
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

}  // namespace sm
}  // namespace qg
