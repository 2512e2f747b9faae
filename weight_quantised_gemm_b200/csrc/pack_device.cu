// qgemm_pack_device: the at-rest packing of qgemm_pack, run on the GPU over a
// device fp32 weight, bit-identical to the host packer. The method stores its
// weights packed (stable-diffusion.rs README, introduction); this makes the
// packing a device pass for weights that already live in HBM.
//
// One thread packs one (row, group): it takes the same steps in the same
// order as the host packer (min / max or max |w| in fp64, or the exact sum of
// |w|; one division; one round-to-nearest-even to fp16; rint per code), so scales,
// biases and codes match it bit for bit. A group's codes fill whole 32-bit
// words, so no two threads write the same word. Non-finite weights and
// fp16 overflow are reported through the device status word.

#include <cuda_fp16.h>

#include "exact_abs_sum.h"
#include "ptx.cuh"
#include "qgemm_internal.h"

namespace qg {
namespace {

__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) { return __half_as_ushort(__double2half(v)); }
__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
  return static_cast<double>(__half2float(__ushort_as_half(h)));
}
__device__ __forceinline__ bool f16_finite(uint16_t h) { return (h & 0x7C00u) != 0x7C00u; }

// In-word bit position of offset j (the layout of include/qgemm.h).
__device__ __forceinline__ int code_shift(int bits, int j) { return bits == 8 ? 8 * j : ((j & 1) ? 16 : 0) + bits * (j >> 1); }

template <int BITS>
__global__ void pack_kernel(const float* __restrict__ W, int N, int K, uint32_t* __restrict__ packed,
                            uint16_t* __restrict__ scales, uint16_t* __restrict__ biases, unsigned int* status) {
  constexpr int G = BITS <= 2 ? 128 : 64;
  constexpr int PER_WORD = 32 / BITS;
  constexpr int WORDS = G / PER_WORD;  // words per row and group
  const int groups = K / G;
  const int64_t total = static_cast<int64_t>(N) * groups;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(idx / groups), g = static_cast<int>(idx % groups);
    const float* wg = W + static_cast<size_t>(n) * K + static_cast<size_t>(g) * G;
    const size_t sidx = static_cast<size_t>(g) * N + n;  // group-major [K/G, N]
    bool finite = true;
    for (int i = 0; i < G; ++i) finite = finite && isfinite(wg[i]);
    if (!finite) ptx::set_status(status, kStatusPackNonfinite);
    double s = 0.0, b = 0.0;
    if constexpr (BITS == 1) {
      ExactAbsSum sum;  // the exact mean |w|, rounded once (G = 128 = 2^7)
      for (int i = 0; i < G; ++i) sum.add(wg[i]);
      const uint16_t s16 = sum.to_f16_rn(7);
      if (!f16_finite(s16)) ptx::set_status(status, kStatusPackOverflow);
      scales[sidx] = s16;
    } else if constexpr (BITS == 2) {
      double amax = 0.0;
      for (int i = 0; i < G; ++i) {
        const double a = fabs(static_cast<double>(wg[i]));
        amax = amax < a ? a : amax;  // the host's std::max, kept as written
      }
      const uint16_t s16 = f64_to_f16_bits(amax);
      if (!f16_finite(s16)) ptx::set_status(status, kStatusPackOverflow);
      scales[sidx] = s16;
      s = f16_bits_to_f64(s16);
    } else {
      const double qmax = static_cast<double>((1 << BITS) - 1);
      double lo = static_cast<double>(wg[0]), hi = lo;
      for (int i = 1; i < G; ++i) {
        // the host's std::min / std::max exactly: on equal values (+0 and -0)
        // the running value stays
        const double v = static_cast<double>(wg[i]);
        lo = v < lo ? v : lo;
        hi = hi < v ? v : hi;
      }
      lo = lo + 0.0;  // a zero minimum is stored as +0
      hi = hi + 0.0;  // and a zero range gives a +0 scale, whichever zeros the group holds
      const uint16_t s16 = f64_to_f16_bits((hi - lo) / qmax);
      const uint16_t b16 = f64_to_f16_bits(lo);
      if (!f16_finite(s16) || !f16_finite(b16)) ptx::set_status(status, kStatusPackOverflow);
      scales[sidx] = s16;
      biases[sidx] = b16;
      s = f16_bits_to_f64(s16);
      b = f16_bits_to_f64(b16);
    }
    uint32_t* words = packed + (static_cast<size_t>(n) * K + static_cast<size_t>(g) * G) / PER_WORD;
    for (int wd = 0; wd < WORDS; ++wd) {
      uint32_t word = 0u;
      for (int j = 0; j < PER_WORD; ++j) {
        const double w = static_cast<double>(wg[wd * PER_WORD + j]);
        int code;
        if constexpr (BITS == 1) {
          code = w >= 0.0 ? 1 : 0;
        } else if constexpr (BITS == 2) {
          code = s != 0.0 ? static_cast<int>(fmin(1.0, fmax(-1.0, rint(w / s)))) : 0;
        } else {
          const double qmax = static_cast<double>((1 << BITS) - 1);
          code = s != 0.0 ? static_cast<int>(fmin(qmax, fmax(0.0, rint((w - b) / s)))) : 0;
        }
        word |= static_cast<uint32_t>(code & ((1 << BITS) - 1)) << code_shift(BITS, j);
      }
      words[wd] = word;
    }
  }
}

}  // namespace

int launch_pack_device(const float* W, int N, int K, int bits, void* packed, uint16_t* scales, uint16_t* biases,
                       cudaStream_t stream) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  unsigned int* status;
  if ((st = status_word(&status)) != QGEMM_OK) return st;
  const int G = bits <= 2 ? 128 : 64;
  const int64_t total = static_cast<int64_t>(N) * (K / G);
  const int threads = 128;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 32LL * nsm ? want : 32LL * nsm);
  uint32_t* pw = static_cast<uint32_t*>(packed);
  switch (bits) {
    case 1: pack_kernel<1><<<blocks, threads, 0, stream>>>(W, N, K, pw, scales, biases, status); break;
    case 2: pack_kernel<2><<<blocks, threads, 0, stream>>>(W, N, K, pw, scales, biases, status); break;
    case 4: pack_kernel<4><<<blocks, threads, 0, stream>>>(W, N, K, pw, scales, biases, status); break;
    default: pack_kernel<8><<<blocks, threads, 0, stream>>>(W, N, K, pw, scales, biases, status);
  }
  return cuda_check(cudaGetLastError(), "pack_kernel launch");
}

}  // namespace qg
