// Small-M path (M <= 16): a memory-bound kernel that streams the packed
// weights once.
//
// pictor's README ("Extreme quantization is first-class") has GEMV paths
// designed around weights narrower than a byte; at decode-sized M the packed
// bytes set the time,
// so this kernel is built around keeping HBM busy from its first microsecond:
//
// * One CTA per SM owns 16 * NP consecutive weight rows (it takes most of the
//   SM's shared memory, so two CTAs of one grid never share an SM and split
//   its load bandwidth). A producer warp streams the rows through a
//   shared-memory ring, one stage per 8 scale groups of K. A stage takes one 3-D TMA box for the packed codes of all the CTA's
//   rows (viewed as [row][unit][U bytes], U = 128, 64 or 32, the box lands as
//   [unit][row][U bytes] with the U-byte swizzle, so the per-lane row reads
//   are free of bank conflicts) and one 2-D box each for the stage's fp16
//   scales and biases. The activations normally do not pass through the
//   ring: the consumer warps load their B fragments straight from global
//   memory (every CTA reads the same rows, so they come from L2), before
//   waiting for the stage's weights. A TMA copy costs the SM's copy unit on
//   the order of a hundred cycles whatever its size; one per token row per
//   stage made M = 16 pay for 48 (ternary) to 384 (8-bit, K = 12288) of them.
//   Split-row CTAs (below) are the exception: a warp there takes two groups
//   per stage, and holding both groups' fragments across the wait spills
//   registers, so the producer bulk-copies their activation rows into the
//   stage.
// * Eight consumer warps. Normally warp w takes scale group w of every stage
//   for all the CTA's rows; where that would not fit in registers (16 tokens
//   and 6 or more 16-row pairs) the rows split into two halves and warps w and
//   w + 4 take groups w % 4 and w % 4 + 4 of every stage, each for its half.
//   A warp turns codes into bf16 in registers and feeds warp-level mma.sync
//   (m16n8k16, bf16 in, fp32 accumulate): the weights are the 16-row A
//   operand, the activations the 8-column B (tokens past M are zero). At the
//   end the warps' fp32 partial sums meet in shared memory (token-major,
//   bank-conflict free) and a coalesced pass adds them, adds the bias and
//   writes bf16.
// * Overlap (programmatic dependent launch, when the caller asks for it): the
//   producer puts the first stages' weight, scale and bias loads in flight and
//   lets the next grid in the stream launch; whoever reads the activations
//   (the consumers, or for split-row CTAs the producer's copies) waits for
//   the previous grid to finish first, and every thread waits for it before
//   it reads the bias or writes the output. A
//   CTA of the next launch then takes an SM the moment this grid's CTA there
//   exits, and its weight stream overlaps the other SMs' last stages instead
//   of waiting for the whole grid and a fresh launch. Without the launch
//   attribute both steps are no-ops.
//
// Scale and bias are applied per group on the fp32 partial sums instead of
// per weight, which is the same product:
//     sum_k x_k (s q_k + b) = s * sum_k x_k q_k + b * sum_k x_k
// so the per-weight work is only "code -> bf16": 4-bit q as bf16 128 + q (the
// offset removed per group as -128 * sum x), ternary t as bf16 {-2, 0, +2}
// (the factor 2 folded into s / 2), 8-bit q exactly through an fp32 magic
// number. sum_k x_k per group comes from one extra mma against ones.
//
// Inside one mma step (16 consecutive k of one group) thread c of each quad
// takes k = 4c .. 4c+3: the tensor core sums all 16 slots, so any assignment
// works, and this one makes each activation fetch one 8-byte vector and puts
// the thread's code pairs where the packed layout keeps them (even and odd k
// in the two half-words of a 32-bit word).

#include <cuda.h>

#include <mutex>

#include "dequant.cuh"
#include "epilogue.cuh"
#include "qgemm_internal.h"
#include "small_m_layout.cuh"

namespace qg {
namespace sm {

constexpr int NUM_CONSUMER_WARPS = 8;
constexpr int WARP_PRODUCER = NUM_CONSUMER_WARPS;
constexpr int NUM_THREADS = 32 * (NUM_CONSUMER_WARPS + 1);  // 288
constexpr int MAX_STAGES = 8;
constexpr int SMEM_LIMIT = 232448;      // the most a CTA may have
constexpr int RING_BUDGET = 196608;     // bytes of shared memory for the ring
constexpr int SMEM_FLOOR = 118784;      // at least this much, so that one grid's CTAs never share an SM

// Row halves for a CTA of NP pairs and MT tokens: 2 where one warp's
// accumulators for all NP pairs would not fit in registers.
__host__ __device__ constexpr int split_rows(int MT, int NP) { return MT > 8 && NP >= 6 ? 2 : 1; }
// Split-row CTAs give each warp two groups per stage; holding both groups'
// activation fragments in registers across the stage wait spills, so their
// activations come through the ring (one bulk copy per token row) instead of
// straight from global memory.
__host__ __device__ constexpr bool x_in_ring(int MT, int NP) { return split_rows(MT, NP) == 2; }

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

struct Params {
  const uint16_t* X;     // bf16 [M, K]
  const uint16_t* bias;  // bf16 [N] or null
  uint16_t* out;         // bf16 [M, N]
  int epi;               // QGEMM_EPI_*
  const uint16_t* residual;  // bf16 [M, N] (residual update only; may equal out)
  const uint16_t* gate;      // bf16 [N] (residual update only)
  int M, N, K;
  int num_stages;        // ceil(K / KS)
  int ring;              // ring depth
  int unit_shift;        // log2 of U, the bytes per swizzled row piece (128, 64 or 32)
  int stage_bytes;       // bytes per ring stage (multiple of 1024)
  int data_bytes;        // ring (or the partial sums, if larger); the mbarriers follow
  int off_s, off_b;      // offsets of the scales and biases inside a stage
  int off_x, x_stride;   // activations in the ring (split-row CTAs): offset, token row stride in bytes
  int overlap;           // launched with programmatic dependent launch
  uint64_t wait_limit_ns;
  unsigned int* status;
};

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

template <int BITS, int MT, int NP>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    small_m_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_b, const Params p) {
  using F = Fmt<BITS>;
  constexpr int STEPS = F::STEPS;
  constexpr int R = 16 * NP;                 // weight rows of the CTA
  constexpr int PH = split_rows(MT, NP);     // row halves (1 or 2)
  constexpr int GROUP_LANES = NUM_CONSUMER_WARPS / PH;  // warps w and w + GROUP_LANES share a group lane
  constexpr int NPH = NP / PH;               // 16-row pairs per warp
  constexpr int GPL = GS / GROUP_LANES;      // groups per warp and stage
  constexpr int TH = MT > 8 ? 2 : 1;         // 8-token halves
  constexpr int NLP = R + 4;                 // row pitch of the partial sums: 2 * NLP = 8 (mod 32) banks
  constexpr bool XR = x_in_ring(MT, NP);     // activations through the ring, else from global memory
  static_assert(NP % PH == 0, "the halves take whole 16-row pairs");
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled boxes need it; uniform across the block
    if (threadIdx.x == 0) ptx::set_status(p.status, kStatusLayout);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = blockIdx.x * R;
  const int U = 1 << p.unit_shift;

  const uint32_t bar0 = sbase + p.data_bytes;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (MAX_STAGES + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.data_bytes + 16 * MAX_STAGES);
  const uint64_t lim = p.wait_limit_ns;
  // Each CTA walks the K stages starting at its own offset: every CTA reads
  // the same activations, and rotating the order spreads those reads over
  // the L2 instead of sending all CTAs to the same lines at once.
  const int rot = blockIdx.x % p.num_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), NUM_CONSUMER_WARPS);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  auto give_up = [&]() {
    *abort_flag = 1;
    ptx::set_status(p.status, kStatusTimeout);
  };

  // acc[q][h][j]: weight rows 16q + g (j < 2) and 16q + g + 8 (j >= 2) of this
  // warp's half, tokens 8h + 2c + (j & 1)
  float acc[NPH][TH][4];
#pragma unroll
  for (int q = 0; q < NPH; ++q)
#pragma unroll
    for (int h = 0; h < TH; ++h)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[q][h][j] = 0.f;

  if (warp == WARP_PRODUCER) {
    // ---------------- producer: TMA boxes and bulk copies into the ring ----------------
    constexpr int sb_bytes = GS * R * 2;
    const int units = F::ROWB / U;  // row pieces per stage
    const int pre = p.ring < p.num_stages ? p.ring : p.num_stages;
    auto stage_k = [&](int t, int& kt, int& valid) {
      kt = (t + rot) % p.num_stages;  // which K stage ring round t carries
      valid = min(F::KS, p.K - kt * F::KS);
    };
    auto load_weights = [&](int t, int s) {  // lane 0: the stage's packed codes, scales and biases
      int kt, valid;
      stage_k(t, kt, valid);
      const uint32_t st = sbase + s * p.stage_bytes;
      ptx::mbar_arrive_expect_tx(full(s), R * F::ROWB + sb_bytes * (BITS <= 2 ? 1 : 2) + (XR ? p.M * valid * 2 : 0));
      ptx::tma_load_3d(st, &tm_w, 0, n0, kt * units, full(s));
      ptx::tma_load_2d(st + p.off_s, &tm_s, n0, kt * GS, full(s));
      if (BITS > 2) ptx::tma_load_2d(st + p.off_b, &tm_b, n0, kt * GS, full(s));
    };
    auto load_x = [&](int t, int s) {  // all lanes: one bulk copy per token row
      int kt, valid;
      stage_k(t, kt, valid);
      const uint32_t st = sbase + s * p.stage_bytes;
      for (int m = lane; m < p.M; m += 32)
        bulk_copy_g2s(st + p.off_x + m * p.x_stride, p.X + static_cast<size_t>(m) * p.K + kt * F::KS, valid * 2,
                      full(s));
    };
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tm_w);
      ptx::tma_prefetch_desc(&tm_s);
      if (BITS > 2) ptx::tma_prefetch_desc(&tm_b);
    }
    if (!XR || p.overlap) {
      // The weights do not depend on the previous grid: the first stages go
      // out at once, and the next grid may launch (both no-ops without the
      // launch attribute). Ring activations follow once that grid is done
      // (the TMA unit takes copies in issue order, so they queue behind).
      if (lane == 0)
        for (int t = 0; t < pre; ++t) load_weights(t, t);
      griddep_launch_dependents();
      if constexpr (XR) {
        griddep_wait();
        __syncwarp();  // the transaction counts are raised before any activation copy can land
        for (int t = 0; t < pre; ++t) load_x(t, t);
      }
    } else {
      // Nothing to wait for: each stage's activations right behind its
      // weights, so that the first stage is complete as early as possible.
      for (int t = 0; t < pre; ++t) {
        if (lane == 0) load_weights(t, t);
        __syncwarp();
        load_x(t, t);
      }
    }
    int t = pre;
    for (; t < p.num_stages; ++t) {
      const int s = t % p.ring;
      if (!warp_wait(empty(s), ((t / p.ring) & 1) ^ 1, lim, abort_flag)) {
        if (lane == 0) give_up();
        break;
      }
      if (lane == 0) load_weights(t, s);
      if constexpr (XR) {
        __syncwarp();
        load_x(t, s);
      }
    }
    // Let every copy issued above land before the block can exit.
    if (lane == 0) {
      const int first = t > p.ring ? t - p.ring : 0;
      for (int i = first; i < t; ++i) ptx::mbar_wait(full(i % p.ring), (i / p.ring) & 1, lim, nullptr);
    }
  } else {
    // ---------------- consumers ----------------
    griddep_launch_dependents();
    if constexpr (!XR) griddep_wait();  // the activations may be the previous grid's output
    const int ush = p.unit_shift;
    const int key16 = swizzle_key16(g, ush);
    const int gl = warp % GROUP_LANES;  // group lane: groups gl, gl + GROUP_LANES, ... of every stage
    const int q0 = (warp / GROUP_LANES) * NPH;  // first 16-row pair of this warp's half
    const bool ga = g < p.M, gb = MT > 8 && g + 8 < p.M;  // tokens g and g + 8 exist
    for (int t = 0; t < p.num_stages; ++t) {
      const int s = t % p.ring;
      const int kt = (t + rot) % p.num_stages;
      // The activations of this warp's groups (the B operand: tokens g and
      // g + 8, k = gs*G + 16*step + 4c .. +3) straight from global memory,
      // where every CTA reads the same rows (L2 hits); issued before the
      // stage's weights are waited for, so the two latencies overlap.
      uint2 xr[XR ? 1 : GPL][STEPS][TH];
#pragma unroll
      for (int gi = 0; gi < (XR ? 0 : GPL); ++gi) {
        const int k0 = kt * F::KS + (gl + GROUP_LANES * gi) * F::G;
        const bool in = k0 < p.K;
        const uint2* x0p = reinterpret_cast<const uint2*>(p.X + static_cast<size_t>(g) * p.K + k0 + 4 * c);
        const uint2* x1p = reinterpret_cast<const uint2*>(p.X + static_cast<size_t>(g + 8) * p.K + k0 + 4 * c);
#pragma unroll
        for (int k = 0; k < STEPS; ++k) {
          xr[gi][k][0] = (in && ga) ? __ldg(x0p + 4 * k) : make_uint2(0u, 0u);
          if constexpr (TH > 1) xr[gi][k][TH - 1] = (in && gb) ? __ldg(x1p + 4 * k) : make_uint2(0u, 0u);
        }
      }
      if (!warp_wait(full(s), (t / p.ring) & 1, lim, abort_flag)) {
        if (lane == 0) give_up();
        break;
      }
      const uint8_t* st = smem + s * p.stage_bytes;
#pragma unroll
      for (int gi = 0; gi < GPL; ++gi) {
        const int gs = gl + GROUP_LANES * gi;
        if (kt * F::KS + gs * F::G >= p.K) break;
        float xs[TH][4];  // sum of x over the group per token (affine)
        float tmp[NPH][TH][4];
#pragma unroll
        for (int h = 0; h < TH; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) xs[h][j] = 0.f;
#pragma unroll
        for (int q = 0; q < NPH; ++q)
#pragma unroll
          for (int h = 0; h < TH; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) tmp[q][h][j] = 0.f;
#pragma unroll
        for (int k = 0; k < STEPS; ++k) {
          uint2 x0, x1;
          if constexpr (XR) {
            const uint8_t* xg = st + p.off_x + g * p.x_stride + (gs * F::G + 16 * k + 4 * c) * 2;
            x0 = ga ? *reinterpret_cast<const uint2*>(xg) : make_uint2(0u, 0u);
            x1 = gb ? *reinterpret_cast<const uint2*>(xg + 8 * p.x_stride) : make_uint2(0u, 0u);
          } else {
            x0 = xr[gi][k][0];
            x1 = xr[gi][k][TH - 1];
          }
          if constexpr (BITS > 2) {
            const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
            mma_bf16_16816(xs[0], ones, x0.x, x0.y);
            if constexpr (TH > 1) mma_bf16_16816(xs[TH - 1], ones, x1.x, x1.y);
          }
          const uint8_t* wk = st + piece_offset<R>(word_offset<BITS>(gs, k, c), ush, key16);
#pragma unroll
          for (int q = 0; q < NPH; ++q) {
            // rows 16q + g and 16q + g + 8 share the swizzle key
            const int r0 = 16 * (q0 + q) + g;
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(wk + (r0 << ush));
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(wk + ((r0 + 8) << ush));
            uint32_t a[4];
            decode_word<BITS>(w0, c, k, a[0], a[2]);  // row g: k pairs (4c, 4c+1), (4c+2, 4c+3)
            decode_word<BITS>(w1, c, k, a[1], a[3]);  // row g + 8
            mma_bf16_16816(tmp[q][0], a, x0.x, x0.y);
            if constexpr (TH > 1) mma_bf16_16816(tmp[q][TH - 1], a, x1.x, x1.y);
          }
        }
        // apply the group's scale (and bias) of rows 16q + g and 16q + g + 8
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + p.off_s) + gs * R;
        const uint16_t* bi = reinterpret_cast<const uint16_t*>(st + p.off_b) + gs * R;
#pragma unroll
        for (int q = 0; q < NPH; ++q) {
          const int r0 = 16 * (q0 + q) + g;
          const float s2[2] = {deq::h2f(sc[r0]), deq::h2f(sc[r0 + 8])};
          float b2[2] = {0.f, 0.f};
          if constexpr (BITS > 2) {
            b2[0] = deq::h2f(bi[r0]);
            b2[1] = deq::h2f(bi[r0 + 8]);
          }
#pragma unroll
          for (int h = 0; h < TH; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float sj = s2[j >> 1];
              if constexpr (BITS == 1) {
                acc[q][h][j] = fmaf(sj, tmp[q][h][j], acc[q][h][j]);
              } else if constexpr (BITS == 2) {
                acc[q][h][j] = fmaf(0.5f * sj, tmp[q][h][j], acc[q][h][j]);
              } else {
                const float d = BITS == 4 ? fmaf(-128.f, xs[h][j], tmp[q][h][j]) : tmp[q][h][j];
                const float e = fmaf(b2[j >> 1], xs[h][j], acc[q][h][j]);
                acc[q][h][j] = fmaf(sj, d, e);
              }
            }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(empty(s));
    }
  }

  // ---------------- the warps' partial sums meet in shared memory ----------------
  griddep_wait();   // the previous grid is done before this one writes the output or reads the bias
  __syncthreads();  // the ring is drained: reuse it
  float* red = reinterpret_cast<float*>(smem);  // [group lane][token][NLP]
  if (warp < NUM_CONSUMER_WARPS) {
    const int gl = warp % GROUP_LANES, q0 = (warp / GROUP_LANES) * NPH;
#pragma unroll
    for (int q = 0; q < NPH; ++q)
#pragma unroll
      for (int h = 0; h < TH; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = 8 * h + 2 * c + (j & 1), nl = 16 * (q0 + q) + g + 8 * (j >> 1);
          red[(gl * MT + m) * NLP + nl] = acc[q][h][j];
        }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.M * R; i += NUM_THREADS) {
    const int m = i / R, nl = i - m * R;
    const int n = n0 + nl;
    if (n >= p.N) continue;
    float v = 0.f;
#pragma unroll
    for (int l = 0; l < GROUP_LANES; ++l) v += red[(l * MT + m) * NLP + nl];
    if (p.bias) v += __bfloat162float(__ushort_as_bfloat16(p.bias[n]));
    const size_t o = static_cast<size_t>(m) * p.N + n;
    if (p.epi != QGEMM_EPI_NONE)
      v = epi::apply_dyn(p.epi, v, p.epi == QGEMM_EPI_RESIDUAL_GATE ? p.residual[o] : uint16_t(0),
                         p.epi == QGEMM_EPI_RESIDUAL_GATE ? epi::bf16_to_f32(p.gate[n]) : 0.f);
    p.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int BITS, int MT, int NP>
int launch_fmt(const Problem& pr, int grid) {
  using F = Fmt<BITS>;
  constexpr int R = 16 * NP;
  int st = smem_opt_in(reinterpret_cast<const void*>(small_m_kernel<BITS, MT, NP>), SMEM_LIMIT,
                       "cudaFuncSetAttribute(small_m_kernel)");
  if (st != QGEMM_OK) return st;

  Params kp;
  kp.X = static_cast<const uint16_t*>(pr.X);
  kp.bias = pr.bias;
  kp.out = static_cast<uint16_t*>(pr.out);
  kp.epi = pr.epi;
  kp.residual = pr.residual;
  kp.gate = pr.gate;
  kp.M = pr.M;
  kp.N = pr.N;
  kp.K = pr.K;
  kp.num_stages = (pr.K + F::KS - 1) / F::KS;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;  // packed bytes per weight row
  const int unit = wbytes % 128 == 0 ? 128 : wbytes % 64 == 0 ? 64 : 32;  // K % 128 == 0 makes it at least 32
  kp.unit_shift = unit == 128 ? 7 : unit == 64 ? 6 : 5;
  if (F::ROWB % unit || wbytes % unit)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: small-M rows are not whole %d-byte pieces", unit);
  const int sb = GS * R * 2;
  // TMA tile destinations start on 128-byte boundaries (the packed box on a
  // 1024-byte one, for its swizzle); bulk copies need 16 bytes.
  kp.off_s = R * F::ROWB;
  kp.off_b = (kp.off_s + sb + 127) & ~127;
  kp.off_x = (kp.off_b + (BITS <= 2 ? 0 : sb) + 127) & ~127;
  kp.x_stride = F::KS * 2 + 32;  // +32 B: token rows 8 banks apart, so the 8-byte B fetches do not collide
  kp.stage_bytes = (kp.off_x + (x_in_ring(MT, NP) ? pr.M * kp.x_stride : 0) + 1023) & ~1023;
  int ring = RING_BUDGET / kp.stage_bytes;
  ring = ring < MAX_STAGES ? ring : MAX_STAGES;
  ring = ring < kp.num_stages ? ring : kp.num_stages;
  kp.ring = ring < 1 ? 1 : ring;
  const int red_bytes = NUM_CONSUMER_WARPS / split_rows(MT, NP) * MT * (R + 4) * 4;
  kp.data_bytes = kp.ring * kp.stage_bytes > red_bytes ? kp.ring * kp.stage_bytes : red_bytes;
  if (kp.data_bytes < SMEM_FLOOR) kp.data_bytes = SMEM_FLOOR;
  const int smem = kp.data_bytes + 16 * MAX_STAGES + 16;
  if (smem > SMEM_LIMIT) return fail(QGEMM_ERR_UNSUPPORTED, "small-M stage of %d bytes does not fit", kp.stage_bytes);
  if (kp.off_s % 1024 || kp.off_b % 128 || kp.off_x % 128 || kp.x_stride % 16 || kp.stage_bytes % 1024 ||
      kp.data_bytes % 8)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: small-M stage layout misaligned");
  kp.wait_limit_ns = wait_limit_ns();
  if ((st = status_word(&kp.status)) != QGEMM_OK) return st;

  CUtensorMap tm_w, tm_s, tm_b;
  const uint64_t groups = static_cast<uint64_t>(pr.K) / F::G;
  // packed codes as [row][piece][U bytes]; the box is U bytes x R rows x the stage's pieces
  const uint64_t wdims[3] = {static_cast<uint64_t>(unit), static_cast<uint64_t>(pr.N), wbytes / unit};
  const uint64_t wstrides[2] = {wbytes, static_cast<uint64_t>(unit)};
  const uint32_t wbox[3] = {static_cast<uint32_t>(unit), static_cast<uint32_t>(R),
                            static_cast<uint32_t>(F::ROWB / unit)};
  const CUtensorMapSwizzle wswz = unit == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : unit == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
  if ((st = make_tensor_map_3d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.packed, wdims, wstrides, wbox, wswz, "W")) !=
      QGEMM_OK)
    return st;
  if ((st = make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.scales, pr.N, groups,
                               uint64_t(pr.N) * 2, R, GS, CU_TENSOR_MAP_SWIZZLE_NONE, "scales")) != QGEMM_OK)
    return st;
  if (BITS > 2) {
    if ((st = make_tensor_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.biases, pr.N, groups,
                                 uint64_t(pr.N) * 2, R, GS, CU_TENSOR_MAP_SWIZZLE_NONE, "biases")) != QGEMM_OK)
      return st;
  } else {
    tm_b = tm_s;  // unused for ternary
  }
  kp.overlap = pr.overlap ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = pr.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pr.overlap ? 1 : 0;
  return cuda_check(cudaLaunchKernelEx(&cfg, small_m_kernel<BITS, MT, NP>, tm_w, tm_s, tm_b, kp),
                    "small_m_kernel launch");
}

// Rows per CTA: the fewest 16-row pairs (from the compiled set) that cover N
// with at most one CTA per SM.
template <int BITS, int MT>
int launch_rows(const Problem& pr, int nsm) {
  const int pairs = pr.N / 16;
  const int need = (pairs + nsm - 1) / nsm;
  const int np = need <= 2 ? 2 : need <= 4 ? 4 : need <= 6 ? 6 : 8;
  const int grid = (pairs + np - 1) / np;
  switch (np) {
    case 2: return launch_fmt<BITS, MT, 2>(pr, grid);
    case 4: return launch_fmt<BITS, MT, 4>(pr, grid);
    case 6: return launch_fmt<BITS, MT, 6>(pr, grid);
    default: return launch_fmt<BITS, MT, 8>(pr, grid);
  }
}

template <int BITS>
int launch_bits(const Problem& pr, int nsm) {
  return pr.M <= 8 ? launch_rows<BITS, 8>(pr, nsm) : launch_rows<BITS, 16>(pr, nsm);
}

}  // namespace sm

int launch_small_m(const Problem& p) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  if (p.M > 16) return fail(QGEMM_ERR_UNSUPPORTED, "small-M path takes M <= 16");
  switch (p.bits) {
    case 4: return sm::launch_bits<4>(p, nsm);
    case 8: return sm::launch_bits<8>(p, nsm);
    case 1: return sm::launch_bits<1>(p, nsm);
    default: return sm::launch_bits<2>(p, nsm);
  }
}

}  // namespace qg
