// qgemm_dequant_tile: the dequantised weight of any [rows, cols] window, from
// the same device routines the large-M kernel runs on its packed tiles.
// Used to hold the dequantisation bit-exact to its definition.

#include "dequant.cuh"
#include "qgemm_internal.h"

namespace qg {
namespace {

template <int BITS>
__global__ void dequant_tile_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ scales,
                                    const uint16_t* __restrict__ biases, int N, int K, int n0, int k0, int rows,
                                    int cols, uint4* __restrict__ out) {
  constexpr int G = BITS <= 2 ? 128 : 64;
  const int chunks_per_row = cols / 8;
  const int64_t total = static_cast<int64_t>(rows) * chunks_per_row;
  const size_t row_bytes = static_cast<size_t>(K) * BITS / 8;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(idx / chunks_per_row);
    const int cc = static_cast<int>(idx % chunks_per_row);
    const int n = n0 + r;
    const int k = k0 + 8 * cc;  // first k of the chunk (a multiple of 8)
    const int grp = k / G;
    const size_t sidx = static_cast<size_t>(grp) * N + n;  // scales are [K/G, N]
    const uint8_t* row = packed + static_cast<size_t>(n) * row_bytes;
    uint4 o;
    if constexpr (BITS == 4) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(row + k / 2);
      o = deq::chunk_4bit(w, deq::h2f(scales[sidx]), deq::h2f(biases[sidx]));
    } else if constexpr (BITS == 8) {
      const uint2 w = *reinterpret_cast<const uint2*>(row + k);
      o = deq::chunk_8bit(w.x, w.y, deq::h2f(scales[sidx]), deq::h2f(biases[sidx]));
    } else if constexpr (BITS == 2) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(row + (k / 16) * 4);
      o = deq::chunk_ternary_dyn(w, (k / 8) & 1, deq::ternary_half_scale2(deq::h2f(scales[sidx])));
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(row + (k / 32) * 4);
      o = deq::chunk_binary_dyn(w, (k / 8) & 3, deq::bf16_scale2(deq::h2f(scales[sidx])));
    }
    out[idx] = o;
  }
}

}  // namespace

int launch_dequant_tile(const Problem& p, int n0, int k0, int rows, int cols) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  const int64_t chunks = static_cast<int64_t>(rows) * (cols / 8);
  const int threads = 256;
  const int64_t want = (chunks + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 8LL * nsm ? want : 8LL * nsm);
  uint4* out = static_cast<uint4*>(p.out);
  switch (p.bits) {
    case 4:
      dequant_tile_kernel<4><<<blocks, threads, 0, p.stream>>>(p.packed, p.scales, p.biases, p.N, p.K, n0, k0, rows,
                                                               cols, out);
      break;
    case 8:
      dequant_tile_kernel<8><<<blocks, threads, 0, p.stream>>>(p.packed, p.scales, p.biases, p.N, p.K, n0, k0, rows,
                                                               cols, out);
      break;
    case 1:
      dequant_tile_kernel<1><<<blocks, threads, 0, p.stream>>>(p.packed, p.scales, p.biases, p.N, p.K, n0, k0, rows,
                                                               cols, out);
      break;
    default:
      dequant_tile_kernel<2><<<blocks, threads, 0, p.stream>>>(p.packed, p.scales, p.biases, p.N, p.K, n0, k0, rows,
                                                               cols, out);
  }
  return cuda_check(cudaGetLastError(), "dequant_tile_kernel launch");
}

}  // namespace qg
