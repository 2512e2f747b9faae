// Large-M path: TMA -> dequantisation into tensor memory -> tcgen05 MMA
// (A from TMEM, B from shared memory) -> bf16 TMA stores. One persistent CTA
// per SM.
//
// The method expands packed weights to bf16 within the GEMM kernel itself,
// tile by tile (stable-diffusion.rs README, introduction); on Blackwell that
// maps as follows. Each output tile is
// 128 weight rows x 256 tokens, computed as D[n, m] = sum_k Wdeq[n, k] X[m, k]
// by tcgen05.mma with M = 128 (weight rows), N = 256 (tokens), K = 16 per
// instruction, bf16 inputs and fp32 accumulation in tensor memory. Putting the
// weights on the MMA's M side means each dequantised weight element feeds 256
// tokens (the widest N an instruction takes) instead of 128, halving the
// dequantisation work per FLOP against the usual orientation.
//
// The dequantised weight tile never touches shared memory: the dequantising
// warps write it straight into tensor memory (one lane per weight row, two
// bf16 per 32-bit column along K) and the MMA reads its A operand from there.
//
// One pipeline stage covers 128 of K: 8 MMAs behind a single barrier wait and
// a single commit. The issuing thread's own instruction latency (on the order
// of a hundred cycles per wait, commit or MMA issue) is what limits a narrower
// stage, so the stage is as wide as shared memory allows.
//
// Rings:
//   stage ring (X in smem + A in TMEM, one index)
//                  X[256 x 128] as two 128-byte-swizzled boxes, loaded by TMA;
//                  the bf16 weight tile [128 lanes x 64 columns] written by
//                  the dequantisers. One "full" barrier (the TMA bytes plus
//                  one arrival per dequantiser) and one "empty" barrier
//                  (committed by the MMA) serve both halves.
//   W ring (smem)  packed weight tiles [128 rows x 128 k], swizzled by the TMA
//                  so that the dequantisers' row-per-lane reads are free of
//                  bank conflicts, plus the stage's fp16 scales and biases
//                  (group-major at rest, so one 256-byte TMA row per group).
// TMEM columns: the fp32 accumulator in 0..255, the A stages from 256 on.
//
// Warp roles (608 threads):
//   warp 0        TMA producer of X
//   warp 1        MMA issuer (one thread) and TMEM owner
//   warp 2        TMA producer of the W ring
//   warps 3..10   dequantisers: warp w writes TMEM lanes 32 (w % 4) ..+31 (its
//                 lane quarter), SLICES_PER_WARP 32-k slices of every stage
//   warps 11..18  epilogue: tcgen05.ld one lane quarter x 128 tokens of the
//                 accumulator 32 tokens at a time, add the bias, round to bf16
//                 into the warp's own 2 KB shared-memory slot (transposed to
//                 token-major) and TMA-store the 32 x 32 block; the
//                 accumulator goes back to the MMA after the warp's last load.
// Shared memory is laid out without slack: the kernel checks that its dynamic
// shared memory starts on a 1024-byte boundary and otherwise records a status
// code and returns.
// Every wait is bounded: on expiry the kernel records a status code, drains
// what it has in flight, frees TMEM and returns.

#include <cuda.h>

#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include "dequant.cuh"
#include "epilogue.cuh"
#include "qgemm_internal.h"

namespace qg {
namespace lm {

constexpr int TILE_N = 128;  // weight rows per tile (MMA M)
constexpr int TILE_M = 256;  // tokens per tile (MMA N)
constexpr int BK = 128;      // K per pipeline stage
constexpr int BOX_K = 64;    // K per X box: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int SLICE_K = 32;  // K per dequantiser slice: four 8-element chunks
constexpr int SLICES_PER_WARP = 2;
constexpr int NUM_DEQ_WARPS = 4 * (BK / SLICE_K) / SLICES_PER_WARP;  // a lane quarter x slices each
constexpr int NUM_EPI_WARPS = 8;                   // a lane quarter x half the tokens each
constexpr int WARP_XLOAD = 0;
constexpr int WARP_MMA = 1;
constexpr int WARP_WLOAD = 2;
constexpr int WARP_DEQ0 = 3;
constexpr int WARP_EPI0 = WARP_DEQ0 + NUM_DEQ_WARPS;
constexpr int NUM_THREADS = 32 * (WARP_EPI0 + NUM_EPI_WARPS);
constexpr int EPI_ROWS = 32;                      // tokens per tcgen05.ld
constexpr int EPI_SLOT_BYTES = EPI_ROWS * 32 * 2; // one 32 tokens x 32 features bf16 block
constexpr int EPI_TOKENS = TILE_M / (NUM_EPI_WARPS / 4);  // tokens per epilogue warp
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;                   // fp32 accumulator: columns 0..255
constexpr uint32_t A_COL = TILE_M;                // A stages: columns 256..
constexpr uint32_t A_STAGE_COLS = BK / 2;         // 128 bf16 per row = 64 columns
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(TILE_N, TILE_M);
constexpr uint32_t IDESC_PAIR = ptx::idesc_bf16_f32(2 * TILE_N, TILE_M);  // cta_group::2: M = 256 over the pair
constexpr int EPI_BAR_ID = 1;
static_assert(NUM_THREADS <= 1024, "one CTA holds at most 1024 threads");
static_assert(EPI_TOKENS % EPI_ROWS == 0, "epilogue warps cover whole tcgen05.ld chunks");

// PAIR: the CTA-pair form. Two CTAs of a cluster compute a 256-row x
// 256-token tile with tcgen05.mma.cta_group::2 (M = 256): each CTA holds
// its 128 weight rows' A stages and accumulator in its own tensor memory and
// stages 128 of the 256 tokens (the MMA reads the B operand from both CTAs'
// shared memory), so an activation stage takes 32 KB instead of 64 and four
// fit where one CTA alone holds two.
template <int BITS, bool PAIR = false, bool PLAIN = false>
struct Cfg {
  static constexpr int kTokens = PAIR ? TILE_M / 2 : TILE_M;  // tokens this CTA stages
  static constexpr int kXBoxBytes = kTokens * BOX_K * 2;
  static constexpr int kXStageBytes = 2 * kXBoxBytes;
  static constexpr int kGroup = BITS <= 2 ? 128 : 64;
  static constexpr int kGroupsPerStage = BK / kGroup;
  static constexpr int kWRowBytes = BK * BITS / 8;        // packed bytes per row per stage
  static constexpr int kSliceBytes = SLICE_K * BITS / 8;  // packed bytes per row per slice
  static constexpr int kWTileBytes = TILE_N * kWRowBytes;
  // TMA swizzle of the packed tile: one row is exactly one swizzle span (a
  // 1-bit row of 16 bytes is below the smallest span: no swizzle).
  static constexpr CUtensorMapSwizzle kWSwizzle = BITS == 8   ? CU_TENSOR_MAP_SWIZZLE_128B
                                                  : BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : BITS == 2 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                              : CU_TENSOR_MAP_SWIZZLE_NONE;
  static constexpr uint32_t kSwzMask = BITS == 8 ? 7 : BITS == 4 ? 3 : BITS == 2 ? 1 : 0;
  static constexpr int kSBytes = kGroupsPerStage * TILE_N * 2;  // one stage's scales (or biases)
  static constexpr int kSBStride = BITS <= 2 ? kSBytes : 2 * kSBytes;
  // 8-bit on one CTA with the plain epilogue (PLAIN): the epilogue stores
  // straight to global memory instead of through shared-memory slots and TMA,
  // which leaves room for a third activation stage beside the 16 KB packed
  // tiles. It reads its whole share of the accumulator and hands it back
  // before the first store, so the stores never hold the MMA. (The fused
  // epilogues store chunk by chunk before their last accumulator read; there
  // the slower 2-byte global stores held the MMA and cost 22 % on the fused
  // out projection, so they keep two stages and the slots.)
  static constexpr bool kDirect = BITS == 8 && !PAIR && PLAIN;
  static constexpr int kS = PAIR ? 4 : BITS == 8 && !kDirect ? 2 : 3;  // stage ring depth
  static constexpr int kSW = BITS == 8 ? (kDirect ? 2 : 3) : BITS == 4 ? (PAIR ? 4 : 2) : BITS == 2 ? 4 : 8;  // W ring depth
  static constexpr int kSlots = kDirect ? 0 : PAIR || BITS == 8 ? 2 : 1;  // epilogue store slots per warp
  static constexpr int kOffX = 0;
  static constexpr int kOffW = kOffX + kS * kXStageBytes;
  static constexpr int kOffOut = kOffW + kSW * kWTileBytes;
  static constexpr int kOffSB = kOffOut + NUM_EPI_WARPS * kSlots * EPI_SLOT_BYTES;
  static constexpr int kOffBar = kOffSB + kSW * kSBStride;
  static constexpr int kNumBars = 2 * kS + 2 * kSW + 3;  // stage full / empty, W ring full / empty, accumulator
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(A_COL + kS * A_STAGE_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(kOffW % 1024 == 0 && kWTileBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kOffSB % 128 == 0 && kSBStride % 128 == 0 && kSBytes % 128 == 0, "TMA rows land on 128 B");
  static_assert(kWRowBytes == 16 * (kSwzMask + 1), "one packed row is one swizzle span (or 16 bytes, unswizzled)");
};

struct Params {
  int M, N, K;
  int num_m_tiles, num_n_tiles, num_tiles, num_kb;
  int m_fastest;  // tile order: 1 = consecutive tiles walk the token dimension, 0 = the feature dimension
  const uint16_t* bias;
  uint16_t* out;             // bf16 [M, N] (written directly by the Cfg::kDirect epilogue)
  const uint16_t* residual;  // bf16 [M, N] (residual update only)
  const uint16_t* gate;      // bf16 [N] (residual update only)
  uint64_t wait_limit_ns;
  unsigned int* status;
};

// Output tile `tile` -> (feature tile, token tile) in the order the host chose.
__device__ __forceinline__ void tile_coords(const Params& p, int tile, int& n_tile, int& m_tile) {
  if (p.m_fastest) {
    n_tile = tile / p.num_m_tiles;
    m_tile = tile - n_tile * p.num_m_tiles;
  } else {
    m_tile = tile / p.num_n_tiles;
    n_tile = tile - m_tile * p.num_n_tiles;
  }
}

// Bounded wait of a whole warp: every lane waits, and the warp gives up as
// one if any lane ran out of time (so no lane is left at a warp barrier).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t lim, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, lim, abort);
  return __all_sync(0xffffffffu, ok);
}

// Byte offset inside a TMA-swizzled tile (1024-byte aligned base): the 16-byte
// unit index (address bits 4..) is XORed with the row bits from bit 7 up.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  return off ^ (((off >> 7) & MASK) << 4);
}

// Bounded waits on barriers that the other CTA of a pair may arrive on.
__device__ __forceinline__ bool warp_wait_cluster(uint32_t bar, uint32_t parity, uint64_t lim,
                                                  const volatile int* abort) {
  const bool ok = ptx::mbar_wait_cluster(bar, parity, lim, abort);
  return __all_sync(0xffffffffu, ok);
}

template <int BITS, int EPI, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    large_m_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_res,
                   const Params p) {
  using C = Cfg<BITS, PAIR, EPI == QGEMM_EPI_NONE>;
  constexpr int S = C::kS, SW = C::kSW;
  constexpr int TILE_ROWS = PAIR ? 2 * TILE_N : TILE_N;  // weight rows of one output tile
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled tiles need it; uniform across the block (and the pair)
    if (threadIdx.x == 0) ptx::set_status(p.status, kStatusLayout);
    if constexpr (PAIR) {  // the peer passes both of its cluster barriers whatever happens here
      ptx::cluster_sync();
      ptx::cluster_sync();
    }
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The pair: CTA `rank` holds weight rows rank * 128 .. +127 of each tile and
  // stages tokens rank * 128 .. +127; the even CTA issues the MMAs.
  const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
  const int unit = PAIR ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int row0 = static_cast<int>(rank) * TILE_N;     // this CTA's first row inside a tile
  const int tok0 = static_cast<int>(rank) * C::kTokens;  // this CTA's first staged token inside a tile

  auto x_stage = [&](int s) { return sbase + C::kOffX + s * C::kXStageBytes; };
  const uint32_t bar0 = sbase + C::kOffBar;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto full_w = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto empty_w = [&](int s) { return bar0 + 8u * (2 * S + SW + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * S + 2 * SW);
  const uint32_t acc_empty = acc_full + 8u;
  const uint32_t drain_bar = acc_full + 16u;
  // where this CTA's epilogue warps report the accumulator drained: the even
  // CTA's barrier (a shared::cluster address; the CTA's own one alone)
  auto acc_empty_arrive = [&]() {
    if constexpr (PAIR) ptx::mbar_arrive_remote(ptx::mapa_shared(acc_empty, 0));
    else ptx::mbar_arrive(acc_empty);
  };

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // the X producer's arrival + one per dequantiser; a pair's even CTA also
      // counts the odd CTA's one relayed arrival for the same stage
      ptx::mbar_init(full(s), PAIR && rank == 0 ? 2 + NUM_DEQ_WARPS : 1 + NUM_DEQ_WARPS);
      ptx::mbar_init(empty(s), 1);
    }
    for (int s = 0; s < SW; ++s) {
      ptx::mbar_init(full_w(s), 1);
      ptx::mbar_init(empty_w(s), NUM_DEQ_WARPS);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, PAIR ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS);
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *epi_abort = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == WARP_MMA) {
    if constexpr (PAIR) {
      ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  if (warp == WARP_XLOAD && lane == 0) {
    ptx::tma_prefetch_desc(&tm_x);
    ptx::tma_prefetch_desc(&tm_out);
  }
  if (warp == WARP_WLOAD && lane == 0) {
    ptx::tma_prefetch_desc(&tm_w);
    ptx::tma_prefetch_desc(&tm_s);
    if (BITS > 2) ptx::tma_prefetch_desc(&tm_b);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) ptx::cluster_sync();  // both CTAs' barriers and TMEM are ready before any cross-CTA use
  ptx::tc_fence_after();
  // Launched with programmatic dependent launch (QGEMM_FLAG_OVERLAP_PREVIOUS):
  // the next grid may launch now (its CTAs take SMs as this grid's leave),
  // and this grid's weight stream, dequantisation and MMAs on it do not wait
  // for the previous one; the X producer waits before its first activation
  // load and the epilogue before it reads bias, gate or residual or stores
  // out. Without the launch attribute both are no-ops.
  ptx::griddep_launch_dependents();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t lim = p.wait_limit_ns;
  const int my_tiles = (p.num_tiles - unit + units - 1) / units;
  const uint32_t total = static_cast<uint32_t>(my_tiles) * static_cast<uint32_t>(p.num_kb);

  auto give_up = [&]() {
    *abort_flag = 1;
    ptx::set_status(p.status, kStatusTimeout);
  };

  if (warp == WARP_XLOAD || warp == WARP_WLOAD) {
    // ---------------- TMA producers ----------------
    if (lane == 0) {
      const bool is_x = warp == WARP_XLOAD;
      if (is_x) ptx::griddep_wait();  // X may be the previous grid's output
      const int R = is_x ? S : SW;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < p.num_tiles; tile += units) {
        int n_tile, m_tile;
        tile_coords(p, tile, n_tile, m_tile);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int s = it % R;
          const uint32_t par = ((it / R) & 1) ^ 1;
          if (!ptx::mbar_wait(is_x ? empty(s) : empty_w(s), par, lim, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          if (is_x) {
            ptx::mbar_arrive_expect_tx(full(s), C::kXStageBytes);
            ptx::tma_load_2d(x_stage(s), &tm_x, kb * BK, m_tile * TILE_M + tok0, full(s));
            ptx::tma_load_2d(x_stage(s) + C::kXBoxBytes, &tm_x, kb * BK + BOX_K, m_tile * TILE_M + tok0, full(s));
          } else {
            const uint32_t wdst = sbase + C::kOffW + s * C::kWTileBytes;
            const uint32_t sdst = sbase + C::kOffSB + s * C::kSBStride;
            const int grp = kb * C::kGroupsPerStage;
            ptx::mbar_arrive_expect_tx(full_w(s), C::kWTileBytes + C::kSBStride);
            const int nr = n_tile * TILE_ROWS + row0;
            ptx::tma_load_2d(wdst, &tm_w, kb * C::kWRowBytes, nr, full_w(s));
            ptx::tma_load_2d(sdst, &tm_s, nr, grp, full_w(s));
            if (BITS > 2) ptx::tma_load_2d(sdst + C::kSBytes, &tm_b, nr, grp, full_w(s));
          }
        }
      }
      // Let every load this thread issued land before the block can exit. For
      // X the stage's full barrier also waits on the dequantisers, so wait on
      // the MMA having consumed it (or, after a time-out, give up quietly).
      const uint32_t first = it > static_cast<uint32_t>(R) ? it - R : 0;
      for (uint32_t i = first; i < it; ++i) {
        if (is_x)
          ptx::mbar_wait(empty(i % R), (i / R) & 1, lim, nullptr);
        else
          ptx::mbar_wait(full_w(i % R), (i / R) & 1, lim, nullptr);
      }
    }
  } else if (warp == WARP_MMA && PAIR && rank != 0) {
    // ---------------- the odd CTA of a pair: relay ----------------
    // A stage is complete here when this CTA's activation bytes have landed
    // and its dequantisers have written their A rows; then one arrival (one
    // cluster-scope release) tells the even CTA, whose MMA reads both.
    uint32_t it = 0;
    bool ok = true;
    for (int tile = unit; ok && tile < p.num_tiles; tile += units)
      for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
        const int s = it % S;
        if (!warp_wait(full(s), (it / S) & 1, lim, abort_flag)) {
          if (lane == 0) give_up();
          ok = false;
          break;
        }
        if (lane == 0) ptx::mbar_arrive_remote(ptx::mapa_shared(full(s), 0));
        __syncwarp();
      }
    // the even CTA's last commit says every MMA of the pair is done: only
    // then may this CTA's tensor memory be freed
    if (lane == 0) ptx::mbar_wait(drain_bar, 0, lim, nullptr);
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // ---------------- MMA issuer ----------------
    // The whole warp runs the loop and waits; one elected lane issues. Keeping
    // the warp converged lets the loop state stay in uniform registers, which
    // shortens the issuing thread's dependency chain per MMA.
    uint32_t it = 0, tcount = 0;
    bool ok = true;
    const bool leader = ptx::elect_one();
    auto wait_ok = [&](uint32_t bar, uint32_t par) {
      return PAIR ? warp_wait_cluster(bar, par, lim, abort_flag) : warp_wait(bar, par, lim, abort_flag);
    };
    for (int tile = unit; ok && tile < p.num_tiles; tile += units, ++tcount) {
      if (!wait_ok(acc_empty, (tcount & 1) ^ 1)) {
        if (leader) give_up();
        break;
      }
      ptx::tc_fence_after();
      for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
        const int s = it % S;
        if (!wait_ok(full(s), (it / S) & 1)) {
          if (leader) give_up();
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (leader) {
          const uint32_t a0 = tmem_base + A_COL + s * A_STAGE_COLS;
          const uint64_t d0 = ptx::smem_desc_sw128_kmajor(x_stage(s));
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint32_t xo = (kk / (BOX_K / UMMA_K)) * C::kXBoxBytes + (kk % (BOX_K / UMMA_K)) * UMMA_K * 2;
            if constexpr (PAIR)
              ptx::tc_mma_f16_ts_pair(tmem_base + ACC_COL, a0 + kk * (UMMA_K / 2), d0 + (xo >> 4), IDESC_PAIR,
                                      (kb | kk) != 0);
            else
              ptx::tc_mma_f16_ts(tmem_base + ACC_COL, a0 + kk * (UMMA_K / 2), d0 + (xo >> 4), IDESC, (kb | kk) != 0);
          }
          if constexpr (PAIR) ptx::tc_commit_pair(empty(s), 0x3);
          else ptx::tc_commit(empty(s));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) {
        if constexpr (PAIR) ptx::tc_commit_pair(acc_full, 0x3);
        else ptx::tc_commit(acc_full);
      }
      __syncwarp();
    }
    if (leader) {
      if constexpr (PAIR) {
        ptx::tc_commit_pair(drain_bar, 0x3);
        ptx::mbar_wait_cluster(drain_bar, 0, lim, nullptr);
      } else {
        ptx::tc_commit(drain_bar);
        ptx::mbar_wait(drain_bar, 0, lim, nullptr);
      }
    }
    __syncwarp();
  } else if (warp < WARP_EPI0) {
    // ---------------- dequantisers: packed smem tile -> bf16 in TMEM ----------------
    const int d = warp - WARP_DEQ0;
    const int q = warp & 3;                     // TMEM lane quarter this warp may write
    const int j0 = (d >> 2) * SLICES_PER_WARP;  // first 32-k slice of each stage
    const int r = 32 * q + lane;                // tile row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    for (uint32_t it = 0; it < total; ++it) {
      const int s = it % S, sw = it % SW;
      if (!warp_wait(full_w(sw), (it / SW) & 1, lim, abort_flag) ||
          !warp_wait(empty(s), ((it / S) & 1) ^ 1, lim, abort_flag)) {
        if (lane == 0) give_up();
        break;
      }
      ptx::tc_fence_after();  // the MMA that last read this A stage has completed
      const uint8_t* wt = smem + C::kOffW + sw * C::kWTileBytes;
      const uint16_t* sb = reinterpret_cast<const uint16_t*>(smem + C::kOffSB + sw * C::kSBStride);
      uint32_t regs[SLICES_PER_WARP][16];
#pragma unroll
      for (int u = 0; u < SLICES_PER_WARP; ++u) {
        const int j = j0 + u;
        const int g = (j * SLICE_K) / C::kGroup;  // scale group of the slice within the stage
        const uint32_t w_off = static_cast<uint32_t>(r * C::kWRowBytes + j * C::kSliceBytes);
        const float s_cur = deq::h2f(sb[g * TILE_N + r]);
        const float b_cur = BITS <= 2 ? 0.f : deq::h2f(sb[C::kSBytes / 2 + g * TILE_N + r]);
        uint4 o[4];  // 4 chunks of 8 consecutive k = the slice's 32 k
        if constexpr (BITS == 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(wt + swz<C::kSwzMask>(w_off));
          o[0] = deq::chunk_4bit(v.x, s_cur, b_cur);
          o[1] = deq::chunk_4bit(v.y, s_cur, b_cur);
          o[2] = deq::chunk_4bit(v.z, s_cur, b_cur);
          o[3] = deq::chunk_4bit(v.w, s_cur, b_cur);
        } else if constexpr (BITS == 8) {
          const uint4 v0 = *reinterpret_cast<const uint4*>(wt + swz<C::kSwzMask>(w_off));
          const uint4 v1 = *reinterpret_cast<const uint4*>(wt + swz<C::kSwzMask>(w_off + 16));
          o[0] = deq::chunk_8bit(v0.x, v0.y, s_cur, b_cur);
          o[1] = deq::chunk_8bit(v0.z, v0.w, s_cur, b_cur);
          o[2] = deq::chunk_8bit(v1.x, v1.y, s_cur, b_cur);
          o[3] = deq::chunk_8bit(v1.z, v1.w, s_cur, b_cur);
        } else if constexpr (BITS == 1) {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(wt + swz<C::kSwzMask>(w_off));
          const uint32_t s2 = deq::bf16_scale2(s_cur);
          o[0] = deq::chunk_binary<0>(v, s2);
          o[1] = deq::chunk_binary<1>(v, s2);
          o[2] = deq::chunk_binary<2>(v, s2);
          o[3] = deq::chunk_binary<3>(v, s2);
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(wt + swz<C::kSwzMask>(w_off));
          const uint32_t hs = deq::ternary_half_scale2(s_cur);
          o[0] = deq::chunk_ternary<0>(v.x, hs);
          o[1] = deq::chunk_ternary<1>(v.x, hs);
          o[2] = deq::chunk_ternary<0>(v.y, hs);
          o[3] = deq::chunk_ternary<1>(v.y, hs);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          regs[u][4 * c + 0] = o[c].x;
          regs[u][4 * c + 1] = o[c].y;
          regs[u][4 * c + 2] = o[c].z;
          regs[u][4 * c + 3] = o[c].w;
        }
      }
      // The packed stage has been read: give it back to the W producer.
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(empty_w(sw));
#pragma unroll
      for (int u = 0; u < SLICES_PER_WARP; ++u)
        ptx::tmem_st_32x32b_x16(tmem_base + lane_addr + A_COL + s * A_STAGE_COLS + (j0 + u) * (SLICE_K / 2), regs[u]);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full(s));
    }
  } else {
    // ---------------- epilogue ----------------
    ptx::griddep_wait();  // bias, gate and residual may be the previous grid's output, out may still be read by it
    const int e = warp - WARP_EPI0;
    const int q = warp & 3;                // TMEM lane quarter this warp may read
    const int t0 = (e >> 2) * EPI_TOKENS;  // first token (accumulator column) of this warp
    const int n_local = 32 * q + lane;
    uint16_t* slots = reinterpret_cast<uint16_t*>(smem + C::kOffOut + e * C::kSlots * EPI_SLOT_BYTES);
    const uint32_t slots_u32 = sbase + C::kOffOut + e * C::kSlots * EPI_SLOT_BYTES;
    uint32_t tcount = 0, nstore = 0;
    for (int tile = unit; tile < p.num_tiles; tile += units, ++tcount) {
      int n_tile, m_tile;
      tile_coords(p, tile, n_tile, m_tile);
      const int nr = n_tile * TILE_ROWS + row0;  // this CTA's first weight row of the tile
      const int n = nr + n_local;
      const int m0 = m_tile * TILE_M + t0;
      const bool n_ok = n < p.N;
      const float bias_f = (p.bias && n_ok) ? __bfloat162float(__ushort_as_bfloat16(p.bias[n])) : 0.f;
      float gate_f = 0.f;
      if constexpr (EPI == QGEMM_EPI_RESIDUAL_GATE) {
        if (n_ok) gate_f = epi::bf16_to_f32(p.gate[n]);
        // while the tile's MMAs run, bring its residual block into L2
        if (e == 0 && lane == 0) ptx::tma_prefetch_l2_2d(&tm_res, nr, m_tile * TILE_M);
      }
      const bool got = warp_wait(acc_full, tcount & 1, lim, abort_flag);
      if (!got && lane == 0) {
        *epi_abort = 1;
        give_up();
      }
      ptx::named_bar_sync(EPI_BAR_ID, 32 * NUM_EPI_WARPS);  // all epilogue warps agree before going on
      if (*epi_abort) break;
      ptx::tc_fence_after();
      const int rows_left = p.M - m0;  // tokens of this warp's half still inside X
      const int chunks = rows_left >= EPI_TOKENS ? EPI_TOKENS / EPI_ROWS
                                                 : (rows_left > 0 ? (rows_left + EPI_ROWS - 1) / EPI_ROWS : 0);
      if constexpr (EPI == QGEMM_EPI_NONE) {
        // Read this warp's share of the accumulator 16 tokens at a time, add
        // the bias and round to bf16 pairs in registers, then hand the
        // accumulator back to the MMA before any shared-memory or TMA store:
        // the next tile's MMAs wait only for the tensor-memory reads. (The
        // fused epilogues keep the per-chunk order below: their arithmetic
        // and residual loads would not fit beside 64 held pairs.)
        constexpr int LD = 16;        // tokens per tcgen05.ld
        uint32_t pk[EPI_TOKENS / 2];  // tokens 2i and 2i + 1 as a bf16 pair
#pragma unroll
        for (int c = 0; c < EPI_TOKENS / LD; ++c) {
          uint32_t v[LD];
          if (c * LD < rows_left) {
            ptx::tmem_ld_32x32b_x16(tmem_base + ACC_COL + t0 + c * LD + (static_cast<uint32_t>(32 * q) << 16), v);
            ptx::tmem_wait_ld();
          }
#pragma unroll
          for (int i = 0; i < LD / 2; ++i)
            pk[c * (LD / 2) + i] = ptx::cvt_bf16x2(__uint_as_float(v[2 * i]) + bias_f,
                                                   __uint_as_float(v[2 * i + 1]) + bias_f);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) acc_empty_arrive();
        if constexpr (C::kDirect) {
          // token m of this warp's rows: 32 lanes write 32 consecutive features (64 bytes)
          if (n_ok) {
#pragma unroll
            for (int t = 0; t < EPI_TOKENS; ++t)
              if (t < rows_left)
                p.out[static_cast<size_t>(m0 + t) * p.N + n] = static_cast<uint16_t>(pk[t / 2] >> (16 * (t & 1)));
          }
          continue;
        } else {
#pragma unroll
        for (int c = 0; c < EPI_TOKENS / EPI_ROWS; ++c) {
          if (c < chunks && nr + 32 * q < p.N) {
            const uint32_t slot = nstore % C::kSlots;
            // the TMA store that last used this slot has finished reading it
            if (lane == 0) ptx::bulk_wait_group_read<C::kSlots - 1>();
            __syncwarp();
            uint16_t* sl = slots + slot * (EPI_SLOT_BYTES / 2);
#pragma unroll
            for (int t = 0; t < EPI_ROWS; ++t)
              sl[t * 32 + lane] = static_cast<uint16_t>(pk[c * (EPI_ROWS / 2) + t / 2] >> (16 * (t & 1)));
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              // rows past M and columns past N fall outside the tensor map and are dropped
              ptx::tma_store_2d(&tm_out, slots_u32 + slot * EPI_SLOT_BYTES, nr + 32 * q, m0 + c * EPI_ROWS);
              ptx::bulk_commit_group();
            }
            ++nstore;
          }
        }
        continue;
        }
      }
      for (int c = 0; c < EPI_TOKENS / EPI_ROWS; ++c) {
        uint32_t v[32];
        // the residual update's 32 residual values of this chunk, two tokens per
        // register (a warp reads 64 contiguous bytes per token)
        uint32_t res2[EPI == QGEMM_EPI_RESIDUAL_GATE ? EPI_ROWS / 2 : 1];
        if constexpr (EPI == QGEMM_EPI_RESIDUAL_GATE) {
#pragma unroll
          for (int t = 0; t < EPI_ROWS; t += 2) {
            const int m = m0 + c * EPI_ROWS + t;
            const bool ok = c < chunks && n_ok;
            const uint32_t lo = (ok && m < p.M) ? p.residual[static_cast<size_t>(m) * p.N + n] : 0u;
            const uint32_t hi = (ok && m + 1 < p.M) ? p.residual[static_cast<size_t>(m + 1) * p.N + n] : 0u;
            res2[t / 2] = lo | (hi << 16);
          }
        }
        if (c < chunks) {
          ptx::tmem_ld_32x32b_x32(tmem_base + ACC_COL + t0 + c * EPI_ROWS + (static_cast<uint32_t>(32 * q) << 16), v);
          ptx::tmem_wait_ld();
        }
        if (c == EPI_TOKENS / EPI_ROWS - 1) {
          // this warp's last read of the accumulator: hand it back before storing
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) acc_empty_arrive();
        }
        if constexpr (C::kDirect) {
          if (c < chunks && n_ok) {
#pragma unroll
            for (int t = 0; t < EPI_ROWS; ++t) {
              const int m = m0 + c * EPI_ROWS + t;
              const uint16_t r = EPI == QGEMM_EPI_RESIDUAL_GATE ? static_cast<uint16_t>(res2[EPI == QGEMM_EPI_RESIDUAL_GATE ? t / 2 : 0] >> (16 * (t & 1))) : 0;
              const float f = epi::apply<EPI>(__uint_as_float(v[t]) + bias_f, r, gate_f);
              if (m < p.M) p.out[static_cast<size_t>(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
            }
          }
        } else if (c < chunks && nr + 32 * q < p.N) {
          const uint32_t slot = nstore % C::kSlots;
          // the TMA store that last used this slot has finished reading it
          if (lane == 0) ptx::bulk_wait_group_read<C::kSlots - 1>();
          __syncwarp();
          uint16_t* sl = slots + slot * (EPI_SLOT_BYTES / 2);
#pragma unroll
          for (int t = 0; t < EPI_ROWS; ++t) {
            const uint16_t r =
                EPI == QGEMM_EPI_RESIDUAL_GATE ? static_cast<uint16_t>(res2[EPI == QGEMM_EPI_RESIDUAL_GATE ? t / 2 : 0] >> (16 * (t & 1))) : 0;
            const float f = epi::apply<EPI>(__uint_as_float(v[t]) + bias_f, r, gate_f);
            sl[t * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past M and columns past N fall outside the tensor map and are dropped
            ptx::tma_store_2d(&tm_out, slots_u32 + slot * EPI_SLOT_BYTES, nr + 32 * q, m0 + c * EPI_ROWS);
            ptx::bulk_commit_group();
          }
          ++nstore;
        }
      }
    }
    if (lane == 0) ptx::bulk_wait_group<0>();
  }

  ptx::tc_fence_before();
  __syncthreads();
  // a pair: neither CTA leaves (or frees its tensor memory) while the other
  // may still arrive on its barriers or the MMAs read its operands
  if constexpr (PAIR) ptx::cluster_sync();
  if (warp == WARP_MMA) {
    ptx::tc_fence_after();
    if constexpr (PAIR) ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// How many CTA pairs of this kernel can be resident at once (queried once
// per device and kernel): the grid of a pair launch takes no more, so that
// every pair starts at once and the static tile order stays balanced.
inline int max_pairs(const void* fn, int smem, int nsm) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nsm / 2;
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> cache;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find({dev, fn});
    if (it != cache.end()) return it->second;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (nsm / 2));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) n = nsm / 2;
  n = n < nsm / 2 ? n : nsm / 2;
  std::lock_guard<std::mutex> lk(mu);
  cache[{dev, fn}] = n;
  return n;
}

template <int BITS, int EPI, bool PAIR>
int launch_fmt(const Problem& pr, int nsm) {
  using C = Cfg<BITS, PAIR, EPI == QGEMM_EPI_NONE>;
  constexpr int TILE_ROWS = PAIR ? 2 * TILE_N : TILE_N;
  const void* fn = reinterpret_cast<const void*>(large_m_kernel<BITS, EPI, PAIR>);
  int st = smem_opt_in(fn, C::kSmemBytes, "cudaFuncSetAttribute(large_m_kernel)");
  if (st != QGEMM_OK) return st;
  CUtensorMap tm_x, tm_w, tm_s, tm_b;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;
  const uint64_t groups = static_cast<uint64_t>(pr.K) / C::kGroup;
  const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
  if ((st = make_tensor_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.X, pr.K, pr.M, uint64_t(pr.K) * 2, BOX_K,
                               C::kTokens, CU_TENSOR_MAP_SWIZZLE_128B, "X")) != QGEMM_OK)
    return st;
  if ((st = make_tensor_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.packed, wbytes, pr.N, wbytes, C::kWRowBytes,
                               TILE_N, C::kWSwizzle, "W")) != QGEMM_OK)
    return st;
  if ((st = make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.scales, pr.N, groups, uint64_t(pr.N) * 2,
                               TILE_N, C::kGroupsPerStage, none, "scales")) != QGEMM_OK)
    return st;
  if (BITS > 2) {
    if ((st = make_tensor_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.biases, pr.N, groups, uint64_t(pr.N) * 2,
                                 TILE_N, C::kGroupsPerStage, none, "biases")) != QGEMM_OK)
      return st;
  } else {
    tm_b = tm_s;  // unused for ternary
  }
  CUtensorMap tm_out;
  if ((st = make_tensor_map_2d(&tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.out, pr.N, pr.M, uint64_t(pr.N) * 2, 32,
                               EPI_ROWS, none, "out")) != QGEMM_OK)
    return st;
  unsigned int* status;
  if ((st = status_word(&status)) != QGEMM_OK) return st;
  Params kp;
  kp.M = pr.M;
  kp.N = pr.N;
  kp.K = pr.K;
  kp.num_m_tiles = (pr.M + TILE_M - 1) / TILE_M;
  kp.num_n_tiles = (pr.N + TILE_ROWS - 1) / TILE_ROWS;
  if (static_cast<int64_t>(kp.num_m_tiles) * kp.num_n_tiles > INT32_MAX)
    return fail(QGEMM_ERR_UNSUPPORTED, "M=%d x N=%d: more output tiles than one launch indexes", pr.M, pr.N);
  kp.num_tiles = kp.num_m_tiles * kp.num_n_tiles;
  kp.num_kb = pr.K / BK;
  // one CTA per SM, or one pair per two SMs; `units` tiles are in flight at once
  const int cap = PAIR ? max_pairs(fn, C::kSmemBytes, nsm) : nsm;
  const int units = kp.num_tiles < cap ? kp.num_tiles : cap;
  const int grid = PAIR ? 2 * units : units;
  // The grid works on `units` consecutive tiles at a time. Walk the dimension
  // that keeps fewer bytes of activation panels (256 tokens x K) and weight
  // panels (TILE_ROWS rows x K, packed) live in L2 at once.
  {
    const double x_panel = double(TILE_M) * pr.K * 2;
    const double w_panel = double(TILE_ROWS) * pr.K * BITS / 8;
    auto live = [&](int fast, double fast_panel, double slow_panel) {
      const int f = fast < units ? fast : units;
      return f * fast_panel + double((units + fast - 1) / fast) * slow_panel;
    };
    kp.m_fastest = live(kp.num_m_tiles, x_panel, w_panel) <= live(kp.num_n_tiles, w_panel, x_panel);
  }
  kp.bias = pr.bias;
  kp.out = static_cast<uint16_t*>(pr.out);
  kp.residual = pr.residual;
  kp.gate = pr.gate;
  CUtensorMap tm_res = tm_out;  // the residual update's L2 prefetch box: this CTA's part of a tile
  if (EPI == QGEMM_EPI_RESIDUAL_GATE &&
      (st = make_tensor_map_2d(&tm_res, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.residual, pr.N, pr.M,
                               uint64_t(pr.N) * 2, TILE_N, TILE_M, CU_TENSOR_MAP_SWIZZLE_NONE, "residual")) != QGEMM_OK)
    return st;
  kp.wait_limit_ns = wait_limit_ns();
  kp.status = status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = pr.stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (PAIR) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
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
  return cuda_check(cudaLaunchKernelEx(&cfg, large_m_kernel<BITS, EPI, PAIR>, tm_x, tm_w, tm_s, tm_b, tm_out, tm_res,
                                       kp),
                    "large_m_kernel launch");
}

}  // namespace lm

int launch_large_m(const Problem& p) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  // The CTA-pair form only when asked for (QGEMM_LARGE_PAIR=1): measured on
  // B200 it is slower than one CTA per tile in every format (8-bit FLUX
  // linears 22-31 % slower, 4-bit QKV 34 %), so the library's choice is the
  // one-CTA form.
  const int mode = large_pair_mode();
  const bool pair = nsm >= 2 && mode == 1;
  auto go = [&](auto bits_tag, auto pair_tag) {
    constexpr int B = decltype(bits_tag)::value;
    constexpr bool P = decltype(pair_tag)::value;
    switch (p.epi) {
      case QGEMM_EPI_GELU_TANH: return lm::launch_fmt<B, QGEMM_EPI_GELU_TANH, P>(p, nsm);
      case QGEMM_EPI_RESIDUAL_GATE: return lm::launch_fmt<B, QGEMM_EPI_RESIDUAL_GATE, P>(p, nsm);
      default: return lm::launch_fmt<B, QGEMM_EPI_NONE, P>(p, nsm);
    }
  };
  auto go_bits = [&](auto bits_tag) {
    return pair ? go(bits_tag, std::true_type{}) : go(bits_tag, std::false_type{});
  };
  switch (p.bits) {
    case 4: return go_bits(std::integral_constant<int, 4>{});
    case 8: return go_bits(std::integral_constant<int, 8>{});
    case 1: return go_bits(std::integral_constant<int, 1>{});
    default: return go_bits(std::integral_constant<int, 2>{});
  }
}

}  // namespace qg
