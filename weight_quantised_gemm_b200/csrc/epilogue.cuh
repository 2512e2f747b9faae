// The fused epilogues of qgemm_fused, applied to one output element
// v = acc + bias (fp32) before its single rounding to bf16:
//   QGEMM_EPI_NONE           v
//   QGEMM_EPI_GELU_TANH      0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))
//   QGEMM_EPI_RESIDUAL_GATE  residual + gate * v
// These are the elementwise steps on either side of a FLUX block's linears:
// the up projection's GELU and the residual-writing layers' gated update of
// the residual stream (stable-diffusion.rs README, introduction, names those
// layers; the formulas are FLUX's).
#pragma once

#include <cuda_bf16.h>

#include "qgemm.h"

#include <cstdint>

namespace qg {
namespace epi {

// 0.5 v (1 + tanh(u)) written as v / (1 + exp(-2u)): one exponential and one
// approximate division (relative error of a few ulp). Both tails come out
// right: a denominator past 2^126 gives 0, exp -> 0 gives v.
__device__ __forceinline__ float gelu_tanh(float v) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
  return __fdividef(v, 1.f + __expf(-2.f * u));
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __bfloat162float(__ushort_as_bfloat16(b)); }

// v = acc + bias; r and g are the residual and gate bf16 bits (unused unless
// op is the residual update).
template <int OP>
__device__ __forceinline__ float apply(float v, uint16_t r, float g) {
  if constexpr (OP == QGEMM_EPI_GELU_TANH) return gelu_tanh(v);
  else if constexpr (OP == QGEMM_EPI_RESIDUAL_GATE) return fmaf(g, v, bf16_to_f32(r));
  else return v;
}

__device__ __forceinline__ float apply_dyn(int op, float v, uint16_t r, float g) {
  return op == QGEMM_EPI_GELU_TANH ? gelu_tanh(v) : op == QGEMM_EPI_RESIDUAL_GATE ? fmaf(g, v, bf16_to_f32(r)) : v;
}

}  // namespace epi
}  // namespace qg
