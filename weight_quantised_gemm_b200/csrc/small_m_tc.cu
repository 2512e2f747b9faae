// Small-M GEMV on the 5th-generation tensor cores (M <= 16), an opt-in
// alternative to the register kernel in small_m.cu (QGEMM_SMALL_TC=1): TMA
// ring -> codes turned into exact small bf16 integers, one weight row per
// thread, in tensor memory -> tcgen05.mma (M = 128 weight rows, N = 16 tokens,
// A from tensor memory) into one fp32 accumulator per scale group -> the
// group's scale (and bias) applied to the fp32 partial sums:
//     sum_k x_k (s q_k + b) = s * sum_k x_k q_k + b * sum_k x_k.
// pictor's README ("Extreme quantization is first-class") builds its decode
// GEMVs around weights narrower than a byte; this kernel asks whether the
// Blackwell tensor core pipeline serves that case better than warp-level
// mma.sync on register fragments.
//
// Measured on B200 it does not, and it is not the library's choice: every
// weight has to reach the tensor core as 2 bytes of bf16 through tensor memory
// (or shared memory), and at M <= 16 those bytes serve at most 16 tokens.
// Ternary 12288 x 3072 at M = 1 takes 12.5 us against 7.3 us for the register
// kernel; without the tcgen05.st of the decoded weights (an instrumented copy,
// not a result) it takes 9.7. An MMA of M = 128, N = 16 from tensor memory
// issues every ~9 cycles when one converged warp issues back to back, ~56 when
// the issuing lane runs alone; the A-from-shared-memory form takes ~39.
//
// * CTA = 128 consecutive weight rows (the MMA's M); tokens are the MMA's N =
//   16, rows M..15 of every activation box read as zeros (outside the tensor).
// * Ring stage = 8 scale groups of K: one 3-D TMA box of packed codes for the
//   128 rows (viewed [row][piece][U bytes], landing [piece][row][U bytes] with
//   the U-byte swizzle: a warp's 32 rows read 16-byte chunks conflict-free),
//   the stage's activations as 64-k boxes of 16 token rows with the 128-byte
//   swizzle (the MMA's B operand, K-major), and the fp16 scales (and biases).
// * Decoders: 8 warps, two per tensor-memory lane quarter (a warp may only
//   touch its own 32 lanes); warp (q, h) turns k-half h of every group into
//   bf16 for rows 32 q .. 32 q + 31 (4-bit: 128 + q; ternary: {-2, 0, +2};
//   1-bit: {-1, +1}; 8-bit: q; all exact) and stores them into the group's
//   place in an A slot, row = lane, two k per 32-bit column. An A slot holds a
//   batch of 2 (ternary, 1-bit) or 4 (affine) groups: one barrier wait and
//   one set of commits per batch.
// * MMA warp: the whole warp runs the loop (its state stays in uniform
//   registers), one elected lane issues G / 16 MMAs per group into the
//   group's accumulator, then commits to the A slot's, the accumulator
//   batch's and (after the stage's last batch) the ring stage's barriers.
// * Drains: warp (q, h) reads the accumulators of the groups g with
//   g % 2 == h (tcgen05.ld, one row per thread) a few batches late and
//   applies the group's scale, and for the affine formats the bias times the
//   group's sum of x, which the same warp added up from the stage's
//   activation box while the stage was resident. At the end the h = 1 warps
//   hand their partial sums to the h = 0 warps through shared memory, which
//   add the bias and write bf16.
//
// Every wait is bounded: on expiry the kernel records a status code, the warps
// leave their loops, the MMA warp waits for its MMAs, and tensor memory is
// freed before the CTA exits.

#include <cuda.h>

#include "dequant.cuh"
#include "epilogue.cuh"
#include "qgemm_internal.h"
#include "small_m_layout.cuh"

namespace qg {
namespace stc {

constexpr int ROWS = 128;                 // weight rows per CTA: the MMA's M
constexpr int TOK = 16;                   // the MMA's N: tokens (M <= 16, the rest zero)
constexpr int GS = 8;                     // scale groups per ring stage
constexpr int XBOX_K = 64;                // k per activation box: one 128-byte swizzle row of bf16
constexpr int XBOX_BYTES = TOK * 128;     // 16 token rows x 128 B
constexpr int NUM_DEC_WARPS = 8;          // 2 halves x 4 tensor-memory lane quarters
constexpr int WARP_TMA = 0;
constexpr int WARP_MMA = 1;
constexpr int WARP_DEC0 = 2;
constexpr int NUM_THREADS = 32 * (WARP_DEC0 + NUM_DEC_WARPS);  // 320
constexpr int MAX_RING = 6;
constexpr int NA = 3;                     // A slots (each a batch of groups)
constexpr int ND = 8;                     // accumulators: one per group in flight
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_LIMIT = 232448;
constexpr int RING_BUDGET = 204800;
constexpr int DEC_BAR_ID = 1;             // named barrier of the 8 decoder warps
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(ROWS, TOK);

template <int BITS>
struct Fmt {
  static constexpr int G = BITS <= 2 ? 128 : 64;   // group size
  static constexpr int GB = G * BITS / 8;          // packed bytes per row and group
  static constexpr int KS = GS * G;                // k per stage
  static constexpr int ROWB = GS * GB;             // packed bytes per row and stage
  static constexpr int STEPS = G / 16;             // MMAs per group
  static constexpr int ACOLS = G / 2;              // tensor-memory columns of one group's A
  static constexpr int XBOXES = KS / XBOX_K;       // activation boxes per stage
  static constexpr bool AFFINE = BITS >= 4;
  // groups per batch: one wait, one set of commits; an A slot holds a batch (128 columns)
  static constexpr int BG = BITS <= 2 ? 2 : 4;
  static constexpr int NDB = ND / BG;              // accumulator batches
  static constexpr int LAGB = NDB - 1;             // a batch is drained after the decoders store batch + LAGB
  static constexpr uint32_t D_COL = 0;             // accumulators: 16 columns each
  static constexpr uint32_t A_COL = 16 * ND;       // A slots: BG * ACOLS columns each
  static_assert(A_COL + NA * BG * ACOLS <= TMEM_COLS, "tensor-memory budget");
  static_assert(GS % BG == 0, "batches do not straddle ring stages");
  static_assert(ND % BG == 0 && LAGB >= 1, "accumulator batches");
  static_assert(GB % 16 == 0 || BITS == 1, "k-halves of whole 8- or 16-byte pieces");
  static_assert(!AFFINE || G == XBOX_K, "an affine group is one activation box");
};

struct Params {
  const uint16_t* bias;      // bf16 [N] or null
  uint16_t* out;             // bf16 [M, N]
  int epi;                   // QGEMM_EPI_*
  const uint16_t* residual;  // bf16 [M, N] (residual update only; may equal out)
  const uint16_t* gate;      // bf16 [N] (residual update only)
  int M, N, K;
  int num_groups;            // K / G
  int num_stages;            // ceil(num_groups / GS)
  int ring;                  // ring depth
  int unit_shift;            // log2 of U, the bytes per swizzled row piece (128, 64 or 32)
  int stage_bytes;           // bytes per ring stage (multiple of 1024)
  int off_x, off_s, off_b;   // activation boxes, scales, biases inside a stage
  int off_sv;                // kept scales and biases: [ND][ROWS] float2
  int off_sx;                // per decoder warp, sums of x per group and token: [8][ND][16] float
  int off_bar;               // mbarriers and the tensor-memory slot
  uint64_t wait_limit_ns;
  unsigned int* status;
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t lim, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, lim, abort);
  return __all_sync(0xffffffffu, ok);
}

// Pair p (codes 2p and 2p + 1) of a packed 32-bit word as bf16x2: the exact
// small integer of each code (ternary doubled: {-2, 0, +2}; 4-bit: 128 + q).
template <int BITS>
__device__ __forceinline__ uint32_t decode_pair(uint32_t x, int p) {
  if constexpr (BITS == 1) {
    // codes 2p, 2p + 1 are bits p and 16 + p: {-1, +1}, the sign set where the bit is 0
    return ((~x << (15 - p)) & 0x80008000u) | 0x3F803F80u;
  } else if constexpr (BITS == 2) {
    // codes 2p, 2p + 1 are bits 2p .. 2p + 1 and 16 + 2p ..: moved to bits 14-15 and 30-31
    return (x << (14 - 2 * p)) & 0xC000C000u;
  } else if constexpr (BITS == 4) {
    // codes 2p, 2p + 1 are nibbles at bits 4p and 16 + 4p: bf16 128 + q
    return ((x >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
  } else {
    // byte j is code j: exact q through an fp32 magic number
    const float lo = __uint_as_float(ptx::prmt(x, deq::kMagic, 0x7650u + 2 * p)) - deq::kMagicF;
    const float hi = __uint_as_float(ptx::prmt(x, deq::kMagic, 0x7651u + 2 * p)) - deq::kMagicF;
    return ptx::cvt_bf16x2(lo, hi);
  }
}

template <int BITS, int TL>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    small_m_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_b,
                      const Params p) {
  using F = Fmt<BITS>;
  constexpr int BG = F::BG, NDB = F::NDB, LAGB = F::LAGB;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled boxes need it; uniform across the block
    if (threadIdx.x == 0) ptx::set_status(p.status, kStatusLayout);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * ROWS;
  const int ng = p.num_groups, ns = p.num_stages;
  const int nb = (ng + BG - 1) / BG;  // batches (the last one may be short)
  const uint64_t lim = p.wait_limit_ns;

  const uint32_t bar0 = sbase + p.off_bar;
  auto ring_full = [&](int s) { return bar0 + 8u * s; };
  auto ring_empty = [&](int s) { return bar0 + 8u * (MAX_RING + s); };
  auto a_full = [&](int i) { return bar0 + 8u * (2 * MAX_RING + i); };
  auto a_empty = [&](int i) { return bar0 + 8u * (2 * MAX_RING + NA + i); };
  auto d_full = [&](int j) { return bar0 + 8u * (2 * MAX_RING + 2 * NA + j); };
  const uint32_t drain_bar = bar0 + 8u * (2 * MAX_RING + 2 * NA + ND);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.off_bar + 8 * (2 * MAX_RING + 2 * NA + ND + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring; ++s) {
      ptx::mbar_init(ring_full(s), 1);
      ptx::mbar_init(ring_empty(s), NUM_DEC_WARPS + 1);  // every decoder warp + the MMA thread's commit
    }
    for (int i = 0; i < NA; ++i) {
      ptx::mbar_init(a_full(i), NUM_DEC_WARPS);
      ptx::mbar_init(a_empty(i), 1);
    }
    for (int j = 0; j < NDB; ++j) ptx::mbar_init(d_full(j), 1);
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == WARP_MMA) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == WARP_TMA && lane == 0) {
    ptx::tma_prefetch_desc(&tm_w);
    ptx::tma_prefetch_desc(&tm_x);
    ptx::tma_prefetch_desc(&tm_s);
    if (F::AFFINE) ptx::tma_prefetch_desc(&tm_b);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  auto give_up = [&]() {
    *abort_flag = 1;
    ptx::set_status(p.status, kStatusTimeout);
  };

  if (warp == WARP_TMA) {
    // ---------------- producer: the stage's boxes into the ring ----------------
    if (lane == 0) {
      const int units = F::ROWB >> p.unit_shift;  // row pieces per stage
      const uint32_t tx = ROWS * F::ROWB + F::XBOXES * XBOX_BYTES + GS * ROWS * 2 * (F::AFFINE ? 2 : 1);
      int t = 0;
      for (; t < ns; ++t) {
        const int s = t % p.ring;
        if (t >= p.ring && !ptx::mbar_wait(ring_empty(s), ((t / p.ring) & 1) ^ 1, lim, abort_flag)) {
          give_up();
          break;
        }
        const uint32_t st = sbase + s * p.stage_bytes;
        ptx::mbar_arrive_expect_tx(ring_full(s), tx);
        ptx::tma_load_3d(st, &tm_w, 0, n0, t * units, ring_full(s));
        for (int b = 0; b < F::XBOXES; ++b)
          ptx::tma_load_2d(st + p.off_x + b * XBOX_BYTES, &tm_x, t * F::KS + b * XBOX_K, 0, ring_full(s));
        ptx::tma_load_2d(st + p.off_s, &tm_s, n0, t * GS, ring_full(s));
        if (F::AFFINE) ptx::tma_load_2d(st + p.off_b, &tm_b, n0, t * GS, ring_full(s));
      }
      // let every copy issued above land before the block can exit
      const int first = t > p.ring ? t - p.ring : 0;
      for (int i = first; i < t; ++i) ptx::mbar_wait(ring_full(i % p.ring), (i / p.ring) & 1, lim, nullptr);
    }
  } else if (warp == WARP_MMA) {
    // ---------------- MMA issuer ----------------
    // The whole warp runs the loop and waits, so that the loop state stays in
    // uniform registers; one elected lane issues. Per batch of BG groups: one
    // wait for the decoders, BG * G / 16 MMAs (one accumulator per group),
    // two or three commits.
    const bool leader = ptx::elect_one();
    bool ok = true;
    for (int bt = 0; bt < nb; ++bt) {
      const int g0 = bt * BG, t = g0 / GS, s = t % p.ring;
      if ((g0 % GS == 0 && !warp_wait(ring_full(s), (t / p.ring) & 1, lim, abort_flag)) ||
          !warp_wait(a_full(bt % NA), (bt / NA) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      if (leader) {
        const uint32_t xst = sbase + s * p.stage_bytes + p.off_x;
        const uint32_t a = tmem_base + F::A_COL + BG * F::ACOLS * (bt % NA);
#pragma unroll
        for (int j = 0; j < BG; ++j) {
          const int g = g0 + j;
          if (g < ng) {
            const uint32_t d = tmem_base + F::D_COL + 16 * (g % ND);
#pragma unroll
            for (int kk = 0; kk < F::STEPS; ++kk) {
              const int k_in = (g % GS) * F::G + 16 * kk;  // k inside the stage
              const uint64_t bd = ptx::smem_desc_sw128_kmajor(xst + (k_in / XBOX_K) * XBOX_BYTES) +
                                  static_cast<uint64_t>(((k_in % XBOX_K) * 2) >> 4);
              ptx::tc_mma_f16_ts(d, a + F::ACOLS * j + 8 * kk, bd, IDESC, kk != 0);
            }
          }
        }
        ptx::tc_commit(a_empty(bt % NA));
        ptx::tc_commit(d_full(bt % NDB));
        if ((g0 + BG) % GS == 0 || bt == nb - 1) ptx::tc_commit(ring_empty(s));
      }
      __syncwarp();
    }
    if (!ok && leader) give_up();
    // every MMA issued above completes before tensor memory is freed
    if (leader) {
      ptx::tc_commit(drain_bar);
      ptx::mbar_wait(drain_bar, 0, lim, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------- decoders and drains ----------------
    // Warp (q, h) turns k-half h of every group into bf16 for rows 32 q ..
    // 32 q + 31 (its tensor-memory lanes), and drains the accumulators of
    // the groups g with g % 2 == h for the same rows, LAGB batches late.
    const int q = warp & 3;                  // tensor-memory lane quarter
    const int h = (warp - WARP_DEC0) >> 2;   // k-half of each group; drains groups g % 2 == h
    const int r = 32 * q + lane;             // CTA row = tensor-memory lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const int ush = p.unit_shift;
    const int key16 = sm::swizzle_key16(r & 7, ush);
    float2* sv = reinterpret_cast<float2*>(smem + p.off_sv);  // [ND][ROWS]: the group's scale, bias of each row
    float* sxw = reinterpret_cast<float*>(smem + p.off_sx) + (warp - WARP_DEC0) * ND * TOK;  // this warp's sums of x
    float acc[TL];
#pragma unroll
    for (int m = 0; m < TL; ++m) acc[m] = 0.f;

    // the accumulator of group ge: tokens 0 .. TL - 1 of row r, times the scale (and the bias term)
    auto drain_group = [&](int ge) {
      uint32_t dv[TL];
      if constexpr (TL == 16) ptx::tmem_ld_32x32b_x16(tmem_base + lane_addr + F::D_COL + 16 * (ge % ND), dv);
      else ptx::tmem_ld_32x32b_x4(tmem_base + lane_addr + F::D_COL + 16 * (ge % ND), dv);
      ptx::tmem_wait_ld();
      const float2 sb = sv[(ge % ND) * ROWS + r];
#pragma unroll
      for (int m = 0; m < TL; ++m) {
        const float dd = __uint_as_float(dv[m]);
        if constexpr (BITS == 1) {
          acc[m] = fmaf(sb.x, dd, acc[m]);
        } else if constexpr (BITS == 2) {
          acc[m] = fmaf(0.5f * sb.x, dd, acc[m]);
        } else {
          const float sx = sxw[(ge % ND) * TOK + m];
          const float dq = BITS == 4 ? fmaf(-128.f, sx, dd) : dd;
          acc[m] = fmaf(sb.x, dq, fmaf(sb.y, sx, acc[m]));
        }
      }
    };
    auto drain_batch = [&](int bd) -> bool {
      if (!warp_wait(d_full(bd % NDB), (bd / NDB) & 1, lim, abort_flag)) return false;
      ptx::tc_fence_after();
#pragma unroll
      for (int j = 0; j < BG; ++j) {
        const int ge = bd * BG + j;
        if (ge < ng && (ge & 1) == h) drain_group(ge);
      }
      return true;
    };

    bool ok = true;
    int bt = 0;
    for (int t = 0; t < ns && ok; ++t) {
      const int s = t % p.ring;
      if (!warp_wait(ring_full(s), (t / p.ring) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      const uint8_t* st = smem + s * p.stage_bytes;
      for (int b0 = 0; b0 < GS && t * GS + b0 < ng; b0 += BG, ++bt) {
        if (!warp_wait(a_empty(bt % NA), ((bt / NA) & 1) ^ 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();  // the MMAs that last read this A slot have completed
#pragma unroll
        for (int j = 0; j < BG; ++j) {
          const int gi = b0 + j, g = t * GS + gi;
          if (g >= ng) break;
          if ((g & 1) == h) {
            // the scale (and bias) of the group for this warp's drain of it, and for
            // affine formats the group's sum of x per token (tokens 0..TL-1)
            const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + p.off_s) + gi * ROWS;
            const uint16_t* bi = reinterpret_cast<const uint16_t*>(st + p.off_b) + gi * ROWS;
            sv[(g % ND) * ROWS + r] = make_float2(deq::h2f(sc[r]), F::AFFINE ? deq::h2f(bi[r]) : 0.f);
            if constexpr (F::AFFINE) {
              // box gi of the stage: token row m (m < 16) at m * 128 bytes, its 16-byte chunk c
              // at chunk c ^ (m % 8) (the 128-byte swizzle); lane = (m, part of the 64 k)
              constexpr int PARTS = 32 / TL;  // lanes per token: 8 (4 tokens) or 2 (16 tokens)
              const int m = lane / PARTS, part = lane % PARTS;
              const uint8_t* xb = st + p.off_x + gi * XBOX_BYTES + (m >> 3) * 1024 + (m & 7) * 128;
              float sum = 0.f;
#pragma unroll
              for (int c = part * (8 / PARTS); c < (part + 1) * (8 / PARTS); ++c) {
                const uint4 v = *reinterpret_cast<const uint4*>(xb + ((c ^ (m & 7)) << 4));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  sum += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xFFFF0000u);
              }
#pragma unroll
              for (int o = PARTS / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
              if (part == 0) sxw[(g % ND) * TOK + m] = sum;
            }
          }
          const uint32_t a = tmem_base + lane_addr + F::A_COL + BG * F::ACOLS * (bt % NA) + F::ACOLS * j +
                             (F::ACOLS / 2) * h;
          const int off = gi * F::GB + (F::GB / 2) * h;  // logical byte of this k-half inside the stage row
          const uint8_t* row = st + (r << ush);
          if constexpr (BITS == 1) {
            // 8 bytes = 2 words x 32 codes = 64 k: 32 columns
            const uint2 v = *reinterpret_cast<const uint2*>(row + sm::piece_offset<ROWS>(off, ush, key16));
            uint32_t o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = decode_pair<1>(e < 16 ? v.x : v.y, e % 16);
            ptx::tmem_st_32x32b_x32(a, o);
          } else if constexpr (BITS == 2) {
            // 16 bytes = 4 words x 16 codes = 64 k: 32 columns
            const uint4 v = *reinterpret_cast<const uint4*>(row + sm::piece_offset<ROWS>(off, ush, key16));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = decode_pair<2>(w[e / 8], e % 8);
            ptx::tmem_st_32x32b_x32(a, o);
          } else if constexpr (BITS == 4) {
            // 16 bytes = 4 words x 8 codes = 32 k: 16 columns
            const uint4 v = *reinterpret_cast<const uint4*>(row + sm::piece_offset<ROWS>(off, ush, key16));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = decode_pair<4>(w[e / 4], e % 4);
            ptx::tmem_st_32x32b_x16(a, o);
          } else {
            // 32 bytes = 8 words x 4 codes = 32 k: 16 columns
            const uint4 v0 = *reinterpret_cast<const uint4*>(row + sm::piece_offset<ROWS>(off, ush, key16));
            const uint4 v1 = *reinterpret_cast<const uint4*>(row + sm::piece_offset<ROWS>(off + 16, ush, key16));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = decode_pair<8>(w[e / 2], e % 2);
            ptx::tmem_st_32x32b_x16(a, o);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(a_full(bt % NA));
        // Drains come after the arrival: batch bt - LAGB is drained before
        // this warp's arrival for batch bt + 1 <= (bt - LAGB) + NDB, so the
        // MMAs that reuse its accumulators never overwrite one still being read.
        if (bt >= LAGB && !drain_batch(bt - LAGB)) {
          ok = false;
          break;
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ring_empty(s));  // this warp has read the stage
    }
    for (int bd = bt - LAGB < 0 ? 0 : bt - LAGB; ok && bd < bt; ++bd)
      if (!drain_batch(bd)) ok = false;
    if (!ok && lane == 0) give_up();

    // ---------------- the halves meet; bias, epilogue, bf16 ----------------
    // Once every decoder warp is past the first barrier every MMA has
    // completed (each accumulator was drained, or the block is giving up) and
    // no decoder reads the ring any more, so its first stage holds the
    // partial sums.
    float* red = reinterpret_cast<float*>(smem);  // [TL][ROWS]
    ptx::named_bar_sync(DEC_BAR_ID, 32 * NUM_DEC_WARPS);
    if (h == 1) {
#pragma unroll
      for (int m = 0; m < TL; ++m) red[m * ROWS + r] = acc[m];
    }
    ptx::named_bar_sync(DEC_BAR_ID, 32 * NUM_DEC_WARPS);
    if (h == 0 && !*abort_flag) {
      const int n = n0 + r;
      if (n < p.N) {
        const float bn = p.bias ? __bfloat162float(__ushort_as_bfloat16(p.bias[n])) : 0.f;
        const float gn = p.epi == QGEMM_EPI_RESIDUAL_GATE ? epi::bf16_to_f32(p.gate[n]) : 0.f;
#pragma unroll
        for (int m = 0; m < TL; ++m) {
          if (m < p.M) {
            const size_t o = static_cast<size_t>(m) * p.N + n;
            float v = acc[m] + red[m * ROWS + r] + bn;
            if (p.epi != QGEMM_EPI_NONE)
              v = epi::apply_dyn(p.epi, v, p.epi == QGEMM_EPI_RESIDUAL_GATE ? p.residual[o] : uint16_t(0), gn);
            p.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == WARP_MMA) ptx::tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------

template <int BITS>
int make_params(const Problem& pr, Params& kp, int& smem) {
  using F = Fmt<BITS>;
  kp = Params{};
  kp.bias = pr.bias;
  kp.out = static_cast<uint16_t*>(pr.out);
  kp.epi = pr.epi;
  kp.residual = pr.residual;
  kp.gate = pr.gate;
  kp.M = pr.M;
  kp.N = pr.N;
  kp.K = pr.K;
  if (pr.K % F::G) return fail(QGEMM_ERR_UNSUPPORTED, "internal: K %% group");
  kp.num_groups = pr.K / F::G;
  kp.num_stages = (kp.num_groups + GS - 1) / GS;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;  // packed bytes per weight row
  const int unit = wbytes % 128 == 0 ? 128 : wbytes % 64 == 0 ? 64 : 32;
  kp.unit_shift = unit == 128 ? 7 : unit == 64 ? 6 : 5;
  if (F::ROWB % unit || wbytes % unit)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: small-M rows are not whole %d-byte pieces", unit);
  kp.off_x = ROWS * F::ROWB;
  kp.off_s = kp.off_x + F::XBOXES * XBOX_BYTES;
  kp.off_b = kp.off_s + GS * ROWS * 2;
  kp.stage_bytes = (kp.off_b + (F::AFFINE ? GS * ROWS * 2 : 0) + 1023) & ~1023;
  int ring = RING_BUDGET / kp.stage_bytes;
  ring = ring < MAX_RING ? ring : MAX_RING;
  ring = ring < kp.num_stages ? ring : kp.num_stages;
  kp.ring = ring < 1 ? 1 : ring;
  const int red_bytes = TOK * ROWS * 4;  // at most 16 tokens
  const int data = kp.ring * kp.stage_bytes > red_bytes ? kp.ring * kp.stage_bytes : red_bytes;
  kp.off_sv = data;
  kp.off_sx = kp.off_sv + ND * ROWS * 8;
  kp.off_bar = kp.off_sx + NUM_DEC_WARPS * ND * TOK * 4;
  smem = kp.off_bar + 8 * (2 * MAX_RING + 2 * NA + ND + 1) + 16;
  if (smem > SMEM_LIMIT) return fail(QGEMM_ERR_UNSUPPORTED, "small-M stage of %d bytes does not fit", kp.stage_bytes);
  if (kp.off_x % 1024 || kp.off_s % 128 || kp.off_b % 128 || kp.stage_bytes % 1024 || kp.off_bar % 8)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: small-M stage layout misaligned");
  kp.wait_limit_ns = wait_limit_ns();
  return status_word(&kp.status);
}

template <int BITS, int TL>
int launch_fmt(const Problem& pr) {
  using F = Fmt<BITS>;
  const void* fn = reinterpret_cast<const void*>(small_m_tc_kernel<BITS, TL>);
  int st = smem_opt_in(fn, SMEM_LIMIT, "cudaFuncSetAttribute(small_m_tc_kernel)");
  if (st != QGEMM_OK) return st;
  Params kp;
  int smem = 0;
  if ((st = make_params<BITS>(pr, kp, smem)) != QGEMM_OK) return st;
  const int unit = 1 << kp.unit_shift;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;
  CUtensorMap tm_w, tm_x, tm_s, tm_b;
  // packed codes as [row][piece][U bytes]; the box is U bytes x 128 rows x a stage's pieces
  const uint64_t wdims[3] = {static_cast<uint64_t>(unit), static_cast<uint64_t>(pr.N), wbytes / unit};
  const uint64_t wstrides[2] = {wbytes, static_cast<uint64_t>(unit)};
  const uint32_t wbox[3] = {static_cast<uint32_t>(unit), static_cast<uint32_t>(ROWS),
                            static_cast<uint32_t>(F::ROWB / unit)};
  const CUtensorMapSwizzle wswz = unit == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : unit == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
  if ((st = make_tensor_map_3d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.packed, wdims, wstrides, wbox, wswz, "W")) !=
      QGEMM_OK)
    return st;
  // activations [M, K] bf16: boxes of 64 k x 16 token rows (rows past M read as zeros)
  if ((st = make_tensor_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.X, pr.K, pr.M, uint64_t(pr.K) * 2,
                               XBOX_K, TOK, CU_TENSOR_MAP_SWIZZLE_128B, "X")) != QGEMM_OK)
    return st;
  const uint64_t groups = static_cast<uint64_t>(pr.K) / F::G;
  if ((st = make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.scales, pr.N, groups,
                               uint64_t(pr.N) * 2, ROWS, GS, CU_TENSOR_MAP_SWIZZLE_NONE, "scales")) != QGEMM_OK)
    return st;
  if (F::AFFINE) {
    if ((st = make_tensor_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.biases, pr.N, groups,
                                 uint64_t(pr.N) * 2, ROWS, GS, CU_TENSOR_MAP_SWIZZLE_NONE, "biases")) != QGEMM_OK)
      return st;
  } else {
    tm_b = tm_s;  // unused for ternary and 1-bit
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((pr.N + ROWS - 1) / ROWS);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = pr.stream;
  cfg.numAttrs = 0;
  return cuda_check(cudaLaunchKernelEx(&cfg, small_m_tc_kernel<BITS, TL>, tm_w, tm_x, tm_s, tm_b, kp),
                    "small_m_tc_kernel launch");
}

}  // namespace stc

int launch_small_m_tc(const Problem& p) {
  if (p.M > stc::TOK) return fail(QGEMM_ERR_UNSUPPORTED, "the tensor-core small-M path takes M <= 16");
  if (p.floor_only || p.overlap) return fail(QGEMM_ERR_UNSUPPORTED, "internal: tensor-core small-M launch options");
  // tokens read back per accumulator: 4 (M <= 4) or 16
  const bool few = p.M <= 4;
  switch (p.bits) {
    case 4: return few ? stc::launch_fmt<4, 4>(p) : stc::launch_fmt<4, 16>(p);
    case 8: return few ? stc::launch_fmt<8, 4>(p) : stc::launch_fmt<8, 16>(p);
    case 1: return few ? stc::launch_fmt<1, 4>(p) : stc::launch_fmt<1, 16>(p);
    default: return few ? stc::launch_fmt<2, 4>(p) : stc::launch_fmt<2, 16>(p);
  }
}

}  // namespace qg
