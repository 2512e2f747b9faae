// Small-M path (up to 32 tokens per launch; the API runs M = 33-64 as
// launches of 32 token rows): a memory-bound kernel that streams the packed
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
//   and 6 or more 16-row pairs, 32 tokens and 4 or 8 pairs) the rows split
//   into halves or quarters whose warps share out the stage's groups, each
//   for its part. A warp turns codes into bf16 in registers and feeds
//   warp-level mma.sync (m16n8k16, bf16 in, fp32 accumulate): the weights are
//   the 16-row A operand, the activations the 8-column B tiles (one, two or
//   four of 8 tokens; tokens past M are zero). At the
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
// Thread c of each quad owns a contiguous quarter of every group, codes
// c G/4 .. (c + 1) G/4 - 1, and MMA step s takes codes 4s .. 4s + 3 of it: the
// tensor core sums all 16 slots of a step, so any assignment works as long as
// the activations follow it. This one makes a thread's codes of a group one
// shared-memory load per row and its activations of a group one to four
// 16-byte loads, and keeps each step's code pairs where the packed layout has
// them (even and odd k in the two half-words of a 32-bit word).

#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "dequant.cuh"
#include "epilogue.cuh"
#include "qgemm_internal.h"
#include "small_m_common.cuh"
#include "small_m_layout.cuh"
#include "small_m_plan.h"

namespace qg {
namespace sm {

constexpr int NUM_CONSUMER_WARPS = 8;
constexpr int WARP_PRODUCER = NUM_CONSUMER_WARPS;
constexpr int NUM_THREADS = 32 * (NUM_CONSUMER_WARPS + 1);  // 288
constexpr int MAX_STAGES = 8;
constexpr int SMEM_LIMIT = 232448;      // the most a CTA may have
constexpr int RING_BUDGET = 196608;     // bytes of shared memory for the ring
constexpr int SMEM_FLOOR = 118784;      // at least this much, so that one grid's CTAs never share an SM

// Row parts for a CTA of NP pairs and MT tokens: where one warp's
// accumulators for all NP pairs would not fit in registers the rows split
// into halves (16 tokens and 6 or more pairs, 32 tokens and 4 pairs) or
// quarters (32 tokens and 8 pairs), the warps of a part sharing out the
// stage's groups. 32-token CTAs take 2, 4 or 8 pairs.
__host__ __device__ constexpr int split_rows(int MT, int NP) {
  return MT == 32 ? (NP >= 8 ? 4 : NP >= 4 ? 2 : 1) : (MT == 16 && NP >= 6 ? 2 : 1);
}
// Split-row CTAs give each warp two groups per stage; holding both groups'
// activation fragments in registers across the stage wait spills, so their
// activations come through the ring (one bulk copy per token row) instead of
// straight from global memory. So do 32-token CTAs, whose four 8-token
// fragments per step would not fit either.
__host__ __device__ constexpr bool x_in_ring(int MT, int NP) { return MT > 16 || split_rows(MT, NP) == 2; }

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
  int ksplit;            // K slices per row block: the CTAs of one thread-block cluster (1 = no cluster)
  int floor_only;        // stream the weights through the ring and compute nothing (the streaming floor)
  uint64_t wait_limit_ns;
  unsigned int* status;
};

// Thread-block cluster helpers (K-split launches): a load from a peer CTA's
// shared memory.
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
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
  constexpr int TH = MT / 8;                 // 8-token MMA column tiles (1, 2 or 4)
  constexpr int NLP = R + 4;                 // row pitch of the partial sums: 2 * NLP = 8 (mod 32) banks
  constexpr bool XR = x_in_ring(MT, NP);     // activations through the ring, else from global memory
  static_assert(NP % PH == 0, "the halves take whole 16-row pairs");
  static_assert(MT == 8 || MT == 16 || MT == 32, "8, 16 or 32 tokens");
  static_assert(TH <= 2 || XR, "four token tiles take their activations from the ring");
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled boxes need it; uniform across the block (and the cluster)
    if (threadIdx.x == 0) ptx::set_status(p.status, kStatusLayout);
    if (p.ksplit > 1) {  // the cluster's peers pass both of its barriers whatever happens here
      ptx::cluster_sync();
      ptx::cluster_sync();
    }
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  // K-split launches: the CTAs of a cluster share one row block, CTA `kslice`
  // taking K stages [ks0, ks0 + ns) of it; the partial sums meet at the end.
  const int kslice = p.ksplit > 1 ? static_cast<int>(ptx::cluster_ctarank()) : 0;
  const int n0 = (blockIdx.x / p.ksplit) * R;
  const int ks0 = kslice * p.num_stages / p.ksplit;
  const int ns = (kslice + 1) * p.num_stages / p.ksplit - ks0;
  const int U = 1 << p.unit_shift;

  const uint32_t bar0 = sbase + p.data_bytes;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (MAX_STAGES + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.data_bytes + 16 * MAX_STAGES);
  const uint64_t lim = p.wait_limit_ns;
  // Each CTA walks the K stages starting at its own offset: every CTA reads
  // the same activations, and rotating the order spreads those reads over
  // the L2 instead of sending all CTAs to the same lines at once.
  const int rot = (blockIdx.x / p.ksplit) % ns;

  constexpr int sb_bytes = GS * R * 2;
  const int units = F::ROWB / U;  // row pieces per stage
  const int pre = p.ring < ns ? p.ring : ns;
  auto stage_k = [&](int t, int& kt, int& valid) {
    kt = ks0 + (t + rot) % ns;  // which K stage ring round t carries
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
  // The producer's lane 0 sets up the barriers and puts the first stage's
  // weight loads in flight before the block-wide barrier, so that the weight
  // stream starts as soon as this warp runs (measured: 0.4-0.7 us less per
  // decode GEMV). Only the first stage: issuing all of them here held the
  // other warps at the barrier and cost more than it saved on 4-bit.
  if (threadIdx.x == 32 * WARP_PRODUCER) {
    for (int s = 0; s < p.ring; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), NUM_CONSUMER_WARPS);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
    if (pre > 0) load_weights(0, 0);
    ptx::tma_prefetch_desc(&tm_w);
    ptx::tma_prefetch_desc(&tm_s);
    if (BITS > 2) ptx::tma_prefetch_desc(&tm_b);
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
    if (!XR || p.overlap) {
      // The weights do not depend on the previous grid: the first stages go
      // out at once (the first already has), and the next grid may launch
      // (both no-ops without the launch attribute). Ring activations follow
      // once that grid is done (the TMA unit takes copies in issue order, so
      // they queue behind).
      if (lane == 0)
        for (int t = 1; t < pre; ++t) load_weights(t, t);
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
        if (lane == 0 && t > 0) load_weights(t, t);
        __syncwarp();
        load_x(t, t);
      }
    }
    int t = pre;
    for (; t < ns; ++t) {
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
    bool gt[TH];  // token g + 8 h exists
#pragma unroll
    for (int h = 0; h < TH; ++h) gt[h] = g + 8 * h < p.M;
    const bool compute = !p.floor_only;
    for (int t = 0; t < ns; ++t) {
      const int s = t % p.ring;
      const int kt = ks0 + (t + rot) % ns;
      // The activations of this warp's groups (the B operand: tokens g and
      // g + 8, thread c's chunk k = gs*G + c*G/4 .. + G/4 - 1) straight from
      // global memory, where every CTA reads the same rows (L2 hits); issued
      // before the stage's weights are waited for, so the two latencies overlap.
      constexpr int XV = F::G / 32;  // 16-byte pieces of a thread's activation chunk
      uint4 xr[XR ? 1 : GPL][TH][XV];
#pragma unroll
      for (int gi = 0; gi < (XR ? 0 : GPL); ++gi) {
        const int k0 = kt * F::KS + (gl + GROUP_LANES * gi) * F::G + c * (F::G / 4);
        const bool in = compute && k0 < p.K;
        const uint4* x0p = reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(g) * p.K + k0);
        const uint4* x1p = reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(g + 8) * p.K + k0);
#pragma unroll
        for (int v = 0; v < XV; ++v) {
          xr[gi][0][v] = (in && gt[0]) ? __ldg(x0p + v) : make_uint4(0u, 0u, 0u, 0u);
          if constexpr (TH == 2) xr[gi][1][v] = (in && gt[1]) ? __ldg(x1p + v) : make_uint4(0u, 0u, 0u, 0u);
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
        if (!compute || kt * F::KS + gs * F::G >= p.K) break;
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
        // this thread's packed chunks of the group for rows 16q + g and
        // 16q + g + 8 of every pair (the two rows share the swizzle key): one
        // shared-memory load per row for all of the group's steps
        constexpr int CW = Chunk<BITS>::WORDS;
        uint32_t w0[NPH][CW], w1[NPH][CW];
        {
          const uint8_t* wc = st + piece_offset<R>(chunk_offset<BITS>(gs, c), ush, key16);
#pragma unroll
          for (int q = 0; q < NPH; ++q) {
            const int r0 = 16 * (q0 + q) + g;
            load_chunk<BITS>(wc + (r0 << ush), w0[q]);
            load_chunk<BITS>(wc + ((r0 + 8) << ush), w1[q]);
          }
        }
#pragma unroll
        for (int k = 0; k < STEPS; ++k) {
          uint2 xh[TH];  // B fragments: token g + 8 h of tile h, this thread's k of the step
          if constexpr (XR) {
            const uint8_t* xg = st + p.off_x + g * p.x_stride + (gs * F::G + c * (F::G / 4) + 4 * k) * 2;
#pragma unroll
            for (int h = 0; h < TH; ++h)
              xh[h] = gt[h] ? *reinterpret_cast<const uint2*>(xg + 8 * h * p.x_stride) : make_uint2(0u, 0u);
          } else {
            xh[0] = x_step(xr[gi][0], k);
            if constexpr (TH == 2) xh[1] = x_step(xr[gi][1], k);
          }
          if constexpr (BITS > 2) {
            const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
#pragma unroll
            for (int h = 0; h < TH; ++h) mma_bf16_16816(xs[h], ones, xh[h].x, xh[h].y);
          }
#pragma unroll
          for (int q = 0; q < NPH; ++q) {
            uint32_t a[4];
            decode_quad<BITS>(w0[q][step_word<BITS>(k)], step_quad<BITS>(k), a[0], a[2]);  // row g
            decode_quad<BITS>(w1[q][step_word<BITS>(k)], step_quad<BITS>(k), a[1], a[3]);  // row g + 8
#pragma unroll
            for (int h = 0; h < TH; ++h) mma_bf16_16816(tmp[q][h], a, xh[h].x, xh[h].y);
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
  if (p.ksplit == 1) {
    if (p.floor_only) return;
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
    return;
  }
  // K-split: each CTA first sums its own group lanes into loc[m][R], then,
  // once every slice of the cluster has, finishes outputs i = kslice, kslice
  // + ksplit, ... by adding the slices' sums in slice order over distributed
  // shared memory. The second cluster barrier keeps every CTA (and so its
  // shared memory) alive until its peers have read it.
  float* loc = red + GROUP_LANES * MT * NLP;
  for (int i = threadIdx.x; i < p.M * R; i += NUM_THREADS) {
    const int m = i / R, nl = i - m * R;
    float v = 0.f;
#pragma unroll
    for (int l = 0; l < GROUP_LANES; ++l) v += red[(l * MT + m) * NLP + nl];
    loc[i] = v;
  }
  ptx::cluster_sync();
  if (!p.floor_only) {
    const uint32_t loc_addr = ptx::smem_u32(loc);
    for (int i = threadIdx.x + kslice * NUM_THREADS; i < p.M * R; i += p.ksplit * NUM_THREADS) {
      const int m = i / R, nl = i - m * R;
      const int n = n0 + nl;
      if (n >= p.N) continue;
      float v = 0.f;
      for (int r = 0; r < p.ksplit; ++r) v += ld_shared_cluster_f32(ptx::mapa_shared(loc_addr + 4u * i, r));
      if (p.bias) v += __bfloat162float(__ushort_as_bfloat16(p.bias[n]));
      const size_t o = static_cast<size_t>(m) * p.N + n;
      if (p.epi != QGEMM_EPI_NONE)
        v = epi::apply_dyn(p.epi, v, p.epi == QGEMM_EPI_RESIDUAL_GATE ? p.residual[o] : uint16_t(0),
                           p.epi == QGEMM_EPI_RESIDUAL_GATE ? epi::bf16_to_f32(p.gate[n]) : 0.f);
      p.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
  ptx::cluster_sync();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// The stage layout and kernel parameters of one configuration (format BITS,
// MT tokens, 16 NP rows per CTA, `ksplit` K slices per row block) for a
// problem, and the dynamic shared memory it takes.
template <int BITS, int MT, int NP>
int make_params(const Problem& pr, int ksplit, Params& kp, int& smem) {
  using F = Fmt<BITS>;
  constexpr int R = 16 * NP;
  kp = Params{};
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
  kp.ksplit = ksplit;
  if (ksplit < 1 || ksplit > kp.num_stages)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: %d K slices for %d stages", ksplit, kp.num_stages);
  const int slice_stages = (kp.num_stages + ksplit - 1) / ksplit;  // the longest slice
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
  // +16 B: consecutive token rows 4 banks apart. A half-warp's 8-byte B fetches
  // (4 token rows x the 4 quad threads' chunks, G / 2 bytes apart) then meet
  // at most two to a bank, the least a 16-byte-aligned row stride allows.
  kp.x_stride = F::KS * 2 + 16;
  kp.stage_bytes = (kp.off_x + (x_in_ring(MT, NP) ? pr.M * kp.x_stride : 0) + 1023) & ~1023;
  // Stages that carry the activations are up to twice as large: those rings
  // take all of shared memory (two 100 KB stages for 32 tokens x 128 rows).
  const int budget = x_in_ring(MT, NP) ? SMEM_LIMIT - 16 * MAX_STAGES - 16 : RING_BUDGET;
  int ring = budget / kp.stage_bytes;
  ring = ring < MAX_STAGES ? ring : MAX_STAGES;
  ring = ring < slice_stages ? ring : slice_stages;
  kp.ring = ring < 1 ? 1 : ring;
  // the warps' partial sums (and, K-split, the CTA's own sums over them) reuse the ring at the end
  const int red_bytes = NUM_CONSUMER_WARPS / split_rows(MT, NP) * MT * (R + 4) * 4 + (ksplit > 1 ? MT * R * 4 : 0);
  kp.data_bytes = kp.ring * kp.stage_bytes > red_bytes ? kp.ring * kp.stage_bytes : red_bytes;
  if (kp.data_bytes < SMEM_FLOOR) kp.data_bytes = SMEM_FLOOR;
  smem = kp.data_bytes + 16 * MAX_STAGES + 16;
  if (smem > SMEM_LIMIT) return fail(QGEMM_ERR_UNSUPPORTED, "small-M stage of %d bytes does not fit", kp.stage_bytes);
  if (kp.off_s % 1024 || kp.off_b % 128 || kp.off_x % 128 || kp.x_stride % 16 || kp.stage_bytes % 1024 ||
      kp.data_bytes % 8)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: small-M stage layout misaligned");
  kp.overlap = pr.overlap ? 1 : 0;
  kp.floor_only = pr.floor_only ? 1 : 0;
  kp.wait_limit_ns = wait_limit_ns();
  return status_word(&kp.status);
}

template <int BITS, int MT, int NP>
int launch_fmt(const Problem& pr, int ksplit, int grid) {
  using F = Fmt<BITS>;
  constexpr int R = 16 * NP;
  const void* fn = reinterpret_cast<const void*>(small_m_kernel<BITS, MT, NP>);
  int st = smem_opt_in(fn, SMEM_LIMIT, "cudaFuncSetAttribute(small_m_kernel)");
  if (st != QGEMM_OK) return st;
  Params kp;
  int smem = 0;
  if ((st = make_params<BITS, MT, NP>(pr, ksplit, kp, smem)) != QGEMM_OK) return st;
  const int unit = 1 << kp.unit_shift;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;

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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = pr.stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (ksplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = ksplit;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pr.overlap) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cuda_check(cudaLaunchKernelEx(&cfg, small_m_kernel<BITS, MT, NP>, tm_w, tm_s, tm_b, kp),
                    "small_m_kernel launch");
}

// Whether `clusters` clusters of `ksplit` CTAs of this configuration are
// resident on the device at once (queried once per configuration and device).
template <int BITS, int MT, int NP>
int clusters_fit(const Problem& pr, int ksplit, int clusters, bool* ok) {
  const void* fn = reinterpret_cast<const void*>(small_m_kernel<BITS, MT, NP>);
  int st = smem_opt_in(fn, SMEM_LIMIT, "cudaFuncSetAttribute(small_m_kernel)");
  if (st != QGEMM_OK) return st;
  Params kp;
  int smem = 0;
  if ((st = make_params<BITS, MT, NP>(pr, ksplit, kp, smem)) != QGEMM_OK) return st;
  int dev = 0;
  if ((st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) != QGEMM_OK) return st;
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, int>, int> cache;  // (device, kernel, ksplit, smem) -> clusters
  const auto key = std::make_tuple(dev, fn, ksplit, smem);
  int n = -1;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) n = it->second;
  }
  if (n < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(clusters * ksplit);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ksplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((st = cuda_check(cudaOccupancyMaxActiveClusters(&n, fn, &cfg), "cudaOccupancyMaxActiveClusters")) != QGEMM_OK)
      return st;
    std::lock_guard<std::mutex> lk(mu);
    cache[key] = n;
  }
  *ok = n >= clusters;
  return QGEMM_OK;
}

// Launch shapes: Plan and plan_candidates (small_m_plan.h).

template <int BITS, int MT, int NP>
int try_plan(const Problem& pr, const Plan& pl, bool* launched) {
  *launched = false;
  if (pl.ksplit > 1) {
    bool ok = false;
    int st = clusters_fit<BITS, MT, NP>(pr, pl.ksplit, pl.grid / pl.ksplit, &ok);
    if (st != QGEMM_OK) return st;
    if (!ok) return QGEMM_OK;
  }
  *launched = true;
  return launch_fmt<BITS, MT, NP>(pr, pl.ksplit, pl.grid);
}

// 32-token CTAs take 2, 4 or 8 pairs: 6 would leave three pairs per warp,
// more accumulators than the registers hold.
template <int BITS, int MT>
int launch_rows(const Problem& pr, int nsm) {
  using F = Fmt<BITS>;
  constexpr unsigned NP_MASK = MT == 32 ? (1u << 2 | 1u << 4 | 1u << 8) : (1u << 2 | 1u << 4 | 1u << 6 | 1u << 8);
  const int pairs = pr.N / 16;
  const int nst = (pr.K + F::KS - 1) / F::KS;
  Plan cands[kMaxPlans];
  int count = 0;
  plan_candidates(pairs, nst, nsm, NP_MASK, MT == 32, cands, &count);
  for (int i = 0; i < count; ++i) {
    const Plan& pl = cands[i];
    bool launched = false;
    int st = QGEMM_OK;
    switch (pl.np) {
      case 2: st = try_plan<BITS, MT, 2>(pr, pl, &launched); break;
      case 4: st = try_plan<BITS, MT, 4>(pr, pl, &launched); break;
      case 6: if constexpr (MT != 32) st = try_plan<BITS, MT, 6>(pr, pl, &launched); break;
      default: st = try_plan<BITS, MT, 8>(pr, pl, &launched);
    }
    if (st != QGEMM_OK || launched) return st;
  }
  // more rows than one wave of 128-row CTAs covers: several waves, no slices
  return launch_fmt<BITS, MT, 8>(pr, 1, (pairs + 7) / 8);
}

template <int BITS>
int launch_bits(const Problem& pr, int nsm) {
  if (pr.M <= 8) return launch_rows<BITS, 8>(pr, nsm);
  if (pr.M <= 16) return launch_rows<BITS, 16>(pr, nsm);
  return launch_rows<BITS, 32>(pr, nsm);
}

}  // namespace sm

int launch_small_m(const Problem& p) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  if (p.M > kSmallMaxM) return fail(QGEMM_ERR_UNSUPPORTED, "small-M path takes M <= %d", kSmallMaxM);
  switch (p.bits) {
    case 4: return sm::launch_bits<4>(p, nsm);
    case 8: return sm::launch_bits<8>(p, nsm);
    case 1: return sm::launch_bits<1>(p, nsm);
    default: return sm::launch_bits<2>(p, nsm);
  }
}

}  // namespace qg
