// Small-M path (M <= 16): a memory-bound GEMV-like kernel.
//
// The packed weights stream from HBM with 8- or 16-byte loads straight into
// registers; each thread turns its codes into bf16 in registers and feeds
// them to the tensor cores through warp-level mma.sync (m16n8k16, bf16 in,
// fp32 accumulate). The activations are the 16-row A operand (rows past M
// are zero), the weights the 8-column B operand.
//
// Scale and bias are applied per group on the fp32 partial sums instead of
// per weight, which is algebraically the same product:
//     sum_k x_k (s q_k + b) = s * sum_k x_k q_k + b * sum_k x_k
// so the per-weight register work is only "code -> bf16": q as an exact bf16
// integer (4-bit: 128 + q, the offset removed per group; 8-bit: q), ternary
// t as the bf16 {-2, 0, +2} (the factor 2 folded into s / 2). sum_k x_k per
// group comes from one extra mma against a B operand of ones.
//
// The k order inside one mma step is free (the tensor core sums over all 16
// slots), so each thread of a quad takes 4 consecutive k of its quarter of
// the group: its activation loads are plain contiguous vectors and its code
// pairs sit where the packed layout puts them (even/odd k in the two
// half-words of a 32-bit word).
//
// Work split: a CTA owns 16 weight rows (two mma n8 blocks); its 4 warps split
// the K range by whole groups, and their partial sums meet in shared memory.

#include "dequant.cuh"
#include "qgemm_internal.h"

namespace qg {
namespace {

constexpr int kRowsPerCta = 16;
constexpr int kKSplit = 4;
constexpr int kThreads = 32 * kKSplit;

struct SmallParams {
  const uint16_t* X;       // bf16 [M, K]
  const uint8_t* packed;   // [N, K*bits/8]
  const uint16_t* scales;  // fp16 [K/G, N]
  const uint16_t* biases;  // fp16 [K/G, N] (affine)
  const uint16_t* bias;    // bf16 [N] or null
  uint16_t* out;           // bf16 [M, N]
  int M, N, K;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int BITS>
struct SmallFmt {
  static constexpr int G = BITS == 2 ? 128 : 64;  // group size
  static constexpr int STEPS = G / 16;            // mma k-steps per group
  static constexpr int QCODES = G / 4;            // codes per thread per group (its quarter)
  static constexpr int QWORDS = QCODES * BITS / 32;  // 32-bit words per thread per group and row
  static constexpr int XWORDS = QCODES / 2;       // bf16x2 words of X per thread per group and token row
};

// B operand (two bf16x2 registers) for step `st` from the thread's words.
template <int BITS, int ST>
__device__ __forceinline__ void decode_step(const uint32_t* w, uint32_t& b0, uint32_t& b1) {
  if constexpr (BITS == 4) {
    // 8 codes per word; step ST uses in-word offsets 4(ST%2) .. +3 of word ST/2
    const uint32_t x = w[ST / 2];
    constexpr int I0 = 2 * (ST % 2);
    b0 = ((x >> (4 * I0)) & 0x000F000Fu) | 0x43004300u;        // bf16 128 + q
    b1 = ((x >> (4 * (I0 + 1))) & 0x000F000Fu) | 0x43004300u;
  } else if constexpr (BITS == 2) {
    // 16 codes per word; step ST uses offsets 4(ST%4) .. +3 of word ST/4
    const uint32_t x = w[ST / 4];
    constexpr int I0 = 2 * (ST % 4);
    b0 = deq::ternary_pair_pm2<I0>(x);                          // bf16 {-2, 0, 2}
    b1 = deq::ternary_pair_pm2<I0 + 1>(x);
  } else {
    // 4 codes per word, one word per step: exact integer q in bf16
    const uint32_t x = w[ST];
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

template <int BITS, int ST, int STEPS>
struct StepLoop {
  template <int MT>
  __device__ __forceinline__ static void run(const uint32_t (&xg)[SmallFmt<BITS>::XWORDS],
                                             const uint32_t (&xg8)[SmallFmt<BITS>::XWORDS],
                                             const uint32_t (&w)[2][SmallFmt<BITS>::QWORDS], float (&tmp)[2][4],
                                             float (&xs)[4]) {
    uint32_t a[4];
    a[0] = xg[2 * ST];
    a[2] = xg[2 * ST + 1];
    a[1] = MT > 8 ? xg8[2 * ST] : 0u;
    a[3] = MT > 8 ? xg8[2 * ST + 1] : 0u;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      uint32_t b0, b1;
      decode_step<BITS, ST>(w[b], b0, b1);
      mma_bf16_16816(tmp[b], a, b0, b1);
    }
    if constexpr (BITS != 2) mma_bf16_16816(xs, a, 0x3F803F80u, 0x3F803F80u);  // sum of x over the step
    StepLoop<BITS, ST + 1, STEPS>::template run<MT>(xg, xg8, w, tmp, xs);
  }
};

template <int BITS, int STEPS>
struct StepLoop<BITS, STEPS, STEPS> {
  template <int MT>
  __device__ __forceinline__ static void run(const uint32_t (&)[SmallFmt<BITS>::XWORDS],
                                             const uint32_t (&)[SmallFmt<BITS>::XWORDS],
                                             const uint32_t (&)[2][SmallFmt<BITS>::QWORDS], float (&)[2][4],
                                             float (&)[4]) {}
};

template <int BITS, int MT>
__global__ void __launch_bounds__(kThreads) small_m_kernel(const SmallParams p) {
  using F = SmallFmt<BITS>;
  constexpr int G = F::G;
  __shared__ float red[kKSplit][MT][kRowsPerCta];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n_base = blockIdx.x * kRowsPerCta;
  const int groups = p.K / G;
  const int per_warp = (groups + kKSplit - 1) / kKSplit;
  const int g_begin = warp * per_warp;
  const int g_end = min(groups, g_begin + per_warp);
  const size_t row_bytes = static_cast<size_t>(p.K) * BITS / 8;

  // rows this thread decodes (B operand column g of each n8 block)
  const uint8_t* wrow[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) wrow[b] = p.packed + static_cast<size_t>(n_base + 8 * b + g) * row_bytes;
  // activation rows of the A operand (zero past M)
  const bool xg_ok = g < p.M;
  const bool xg8_ok = MT > 8 && (g + 8) < p.M;
  const uint16_t* xrow_g = p.X + static_cast<size_t>(xg_ok ? g : 0) * p.K;
  const uint16_t* xrow_g8 = p.X + static_cast<size_t>(xg8_ok ? g + 8 : 0) * p.K;

  float acc[2][4];
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[b][j] = 0.f;

  uint32_t w_cur[2][F::QWORDS], w_nxt[2][F::QWORDS];
  uint32_t xg_cur[F::XWORDS], xg_nxt[F::XWORDS], xg8_cur[F::XWORDS], xg8_nxt[F::XWORDS];

  auto load_group = [&](int gi, uint32_t (&w)[2][F::QWORDS], uint32_t (&xa)[F::XWORDS],
                        uint32_t (&xb)[F::XWORDS]) {
    const size_t wofs = static_cast<size_t>(gi) * (G * BITS / 8) + c * (F::QWORDS * 4);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if constexpr (F::QWORDS == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(wrow[b] + wofs));
        w[b][0] = v.x; w[b][1] = v.y; w[b][2] = v.z; w[b][3] = v.w;
      } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(wrow[b] + wofs));
        w[b][0] = v.x; w[b][1] = v.y;
      }
    }
    const int k0 = gi * G + c * F::QCODES;
#pragma unroll
    for (int i = 0; i < F::XWORDS / 4; ++i) {
      uint4 v = xg_ok ? __ldg(reinterpret_cast<const uint4*>(xrow_g + k0) + i) : make_uint4(0, 0, 0, 0);
      xa[4 * i] = v.x; xa[4 * i + 1] = v.y; xa[4 * i + 2] = v.z; xa[4 * i + 3] = v.w;
      if constexpr (MT > 8) {
        v = xg8_ok ? __ldg(reinterpret_cast<const uint4*>(xrow_g8 + k0) + i) : make_uint4(0, 0, 0, 0);
        xb[4 * i] = v.x; xb[4 * i + 1] = v.y; xb[4 * i + 2] = v.z; xb[4 * i + 3] = v.w;
      } else {
        xb[4 * i] = xb[4 * i + 1] = xb[4 * i + 2] = xb[4 * i + 3] = 0u;
      }
    }
  };

  if (g_begin < g_end) load_group(g_begin, w_nxt, xg_nxt, xg8_nxt);
  for (int gi = g_begin; gi < g_end; ++gi) {
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int i = 0; i < F::QWORDS; ++i) w_cur[b][i] = w_nxt[b][i];
#pragma unroll
    for (int i = 0; i < F::XWORDS; ++i) {
      xg_cur[i] = xg_nxt[i];
      xg8_cur[i] = xg8_nxt[i];
    }
    if (gi + 1 < g_end) load_group(gi + 1, w_nxt, xg_nxt, xg8_nxt);

    // scale / bias of the two adjacent weight rows this thread's accumulators
    // cover: one 32-bit load each from the group-major [K/G, N] arrays
    float s[2][2], bb[2][2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const size_t si = static_cast<size_t>(gi) * p.N + n_base + 8 * b + 2 * c;
      const uint32_t sv = __ldg(reinterpret_cast<const uint32_t*>(p.scales + si));
      s[b][0] = deq::h2f(static_cast<uint16_t>(sv & 0xFFFFu));
      s[b][1] = deq::h2f(static_cast<uint16_t>(sv >> 16));
      if constexpr (BITS != 2) {
        const uint32_t bv = __ldg(reinterpret_cast<const uint32_t*>(p.biases + si));
        bb[b][0] = deq::h2f(static_cast<uint16_t>(bv & 0xFFFFu));
        bb[b][1] = deq::h2f(static_cast<uint16_t>(bv >> 16));
      } else {
        bb[b][0] = bb[b][1] = 0.f;
      }
    }

    float tmp[2][4], xs[4];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int j = 0; j < 4; ++j) tmp[b][j] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) xs[j] = 0.f;

    StepLoop<BITS, 0, F::STEPS>::template run<MT>(xg_cur, xg8_cur, w_cur, tmp, xs);

#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float ss = s[b][j & 1];
        if constexpr (BITS == 2) {
          acc[b][j] = fmaf(0.5f * ss, tmp[b][j], acc[b][j]);
        } else {
          const float d = BITS == 4 ? fmaf(-128.f, xs[j], tmp[b][j]) : tmp[b][j];
          const float e = fmaf(bb[b][j & 1], xs[j], acc[b][j]);
          acc[b][j] = fmaf(ss, d, e);
        }
      }
  }

  // partial sums of this warp's K range -> shared memory
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = g + (j >= 2 ? 8 : 0);
      if (m < MT) red[warp][m][8 * b + 2 * c + (j & 1)] = acc[b][j];
    }
  __syncthreads();
  for (int idx = threadIdx.x; idx < MT * kRowsPerCta; idx += kThreads) {
    const int m = idx / kRowsPerCta, col = idx % kRowsPerCta;
    if (m >= p.M) continue;
    float v = red[0][m][col];
#pragma unroll
    for (int w = 1; w < kKSplit; ++w) v += red[w][m][col];
    const int n = n_base + col;
    if (p.bias) v += __bfloat162float(__ushort_as_bfloat16(p.bias[n]));
    p.out[static_cast<size_t>(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

template <int BITS>
void launch_fmt(const SmallParams& sp, int grid, cudaStream_t stream) {
  if (sp.M <= 8)
    small_m_kernel<BITS, 8><<<grid, kThreads, 0, stream>>>(sp);
  else
    small_m_kernel<BITS, 16><<<grid, kThreads, 0, stream>>>(sp);
}

}  // namespace

int launch_small_m(const Problem& p) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  if (p.M > 16) return fail(QGEMM_ERR_UNSUPPORTED, "small-M path takes M <= 16");
  SmallParams sp{static_cast<const uint16_t*>(p.X), p.packed, p.scales, p.biases, p.bias,
                 static_cast<uint16_t*>(p.out), p.M, p.N, p.K};
  const int grid = p.N / kRowsPerCta;
  switch (p.bits) {
    case 4: launch_fmt<4>(sp, grid, p.stream); break;
    case 8: launch_fmt<8>(sp, grid, p.stream); break;
    default: launch_fmt<2>(sp, grid, p.stream);
  }
  return cuda_check(cudaGetLastError(), "small_m_kernel launch");
}

}  // namespace qg
