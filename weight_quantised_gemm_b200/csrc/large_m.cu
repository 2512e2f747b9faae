// Large-M path: TMA -> dequantisation into tensor memory -> tcgen05 MMA
// (A from TMEM, B from shared memory) -> TMA-store epilogue. One persistent
// CTA per SM.
//
// "Dequantised inside the matmul kernel a tile at a time" (stable-diffusion.rs
// README, introduction) maps onto Blackwell as follows. Each output tile is
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
// Shared memory then carries only the TMA-loaded activation and packed-weight
// tiles and the MMA's activation reads, which keeps the tensor pipe ahead of
// the shared-memory port.
//
// Rings, each with its own full/empty mbarriers:
//   X ring (smem)  activation tiles X[256 x 64], 128-byte swizzle; TMA in,
//                  emptied by the MMA;
//   W ring (smem)  packed weight tiles [128 rows x 64 k] plus the tile's 128
//                  fp16 scales and biases (group-major at rest, so one 256-byte
//                  TMA box each); TMA in, emptied by the dequantisers;
//   A ring (TMEM)  dequantised bf16 weight tiles [128 lanes x 32 columns];
//                  written by the dequantisers, emptied by the MMA.
// TMEM columns: the fp32 accumulator in 0..255, the A ring in 256..383.
//
// Warp roles (480 threads):
//   warp 0        TMA producer of the X ring
//   warp 1        MMA issuer (one thread) and TMEM owner
//   warp 2        TMA producer of the W ring
//   warps 3..10   dequantisers: warp w writes TMEM lanes 32 (w % 4) ..+31
//                 (its lane quarter), one 32-k half of each 64-k block
//   warps 11..14  epilogue: tcgen05.ld the accumulator (each warp one lane
//                 quarter = 32 weight rows), add the bias, round to bf16 into a
//                 shared-memory copy of the whole tile, hand the accumulator
//                 back, then one TMA store of [256 tokens x 128 features].
// Every wait is bounded: on expiry the kernel records a status code, drains
// what it has in flight, frees TMEM and returns.

#include <cuda.h>

#include <mutex>

#include "dequant.cuh"
#include "qgemm_internal.h"

namespace qg {
namespace lm {

constexpr int TILE_N = 128;  // weight rows per tile (MMA M)
constexpr int TILE_M = 256;  // tokens per tile (MMA N)
constexpr int BK = 64;       // K per pipeline stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int DEQ_SETS = 2;                    // dequantiser sets, taking K blocks in turn
constexpr int DEQ_WARPS_PER_SET = 8;           // one set covers a 128 x 64 block
constexpr int NUM_DEQ_WARPS = DEQ_SETS * DEQ_WARPS_PER_SET;
constexpr int NUM_EPI_WARPS = 4;
constexpr int WARP_XLOAD = 0;
constexpr int WARP_MMA = 1;
constexpr int WARP_WLOAD = 2;
constexpr int WARP_DEQ0 = 3;
constexpr int WARP_EPI0 = WARP_DEQ0 + NUM_DEQ_WARPS;
constexpr int NUM_THREADS = 32 * (WARP_EPI0 + NUM_EPI_WARPS);
constexpr int X_STAGE_BYTES = TILE_M * BK * 2;  // 32 KB
constexpr int SB_BYTES = TILE_N * 2;            // one group's scales (or biases) for the tile's rows
constexpr int OUT_BYTES = TILE_M * TILE_N * 2;  // the whole bf16 output tile
constexpr int OUT_ROWS = 32;                    // tokens per accumulator chunk read back
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;                 // fp32 accumulator: columns 0..255
constexpr uint32_t A_COL = TILE_M;              // A ring: columns 256..
constexpr uint32_t A_STAGE_COLS = BK / 2;       // 64 bf16 per row = 32 columns
constexpr int SA = 4;                           // A ring depth
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(TILE_N, TILE_M);
constexpr int EPI_BAR_ID = 1;
static_assert(A_COL + SA * A_STAGE_COLS <= TMEM_COLS, "TMEM budget");
static_assert(NUM_THREADS <= 1024, "one CTA holds at most 1024 threads");

template <int BITS>
struct Cfg {
  static constexpr int kGroup = BITS == 2 ? 128 : 64;
  static constexpr int kWRowBytes = BK * BITS / 8;  // packed bytes per row per stage
  static constexpr int kWTileBytes = TILE_N * kWRowBytes;
  static constexpr int kSBBytes = BITS == 2 ? SB_BYTES : 2 * SB_BYTES;  // scales (+ biases)
  static constexpr int kWStride = kWTileBytes + kSBBytes;             // one W-ring stage
  static constexpr int kSX = 4;                                       // X ring depth
  static constexpr int kSW = BITS == 8 ? 3 : BITS == 4 ? 6 : 8;       // W ring depth
  static constexpr int kOffX = 0;
  static constexpr int kOffW = kOffX + kSX * X_STAGE_BYTES;
  static constexpr int kOffOut = (kOffW + kSW * kWStride + 1023) & ~1023;
  static constexpr int kOffBar = kOffOut + OUT_BYTES;
  static constexpr int kNumBars = 2 * kSX + 2 * kSW + 2 * SA + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base to 1024 B
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kOffW % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(kWStride % 128 == 0 && kOffOut % 128 == 0, "TMA boxes land on 128-byte boundaries");
};

struct Params {
  int M, N, K;
  int num_m_tiles, num_n_tiles, num_tiles, num_kb;
  int m_fastest;  // tile order: 1 = consecutive tiles walk the token dimension, 0 = the feature dimension
  const uint16_t* bias;
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

template <int BITS>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    large_m_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_out, const Params p) {
  using C = Cfg<BITS>;
  constexpr int SX = C::kSX, SW = C::kSW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto x_stage = [&](int s) { return sbase + C::kOffX + s * X_STAGE_BYTES; };
  auto w_stage = [&](int s) { return C::kOffW + s * C::kWStride; };  // byte offset into smem
  const uint32_t bar0 = sbase + C::kOffBar;
  auto full_x = [&](int s) { return bar0 + 8u * s; };
  auto empty_x = [&](int s) { return bar0 + 8u * (SX + s); };
  auto full_w = [&](int s) { return bar0 + 8u * (2 * SX + s); };
  auto empty_w = [&](int s) { return bar0 + 8u * (2 * SX + SW + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + s); };
  auto empty_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + SA + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * SX + 2 * SW + 2 * SA);
  const uint32_t acc_empty = acc_full + 8u;
  const uint32_t drain_bar = acc_full + 16u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      ptx::mbar_init(full_x(s), 1);
      ptx::mbar_init(empty_x(s), 1);
    }
    for (int s = 0; s < SW; ++s) {
      ptx::mbar_init(full_w(s), 1);
      ptx::mbar_init(empty_w(s), DEQ_WARPS_PER_SET);
    }
    for (int s = 0; s < SA; ++s) {
      ptx::mbar_init(full_a(s), DEQ_WARPS_PER_SET);
      ptx::mbar_init(empty_a(s), 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, NUM_EPI_WARPS);
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *epi_abort = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == WARP_MMA) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == WARP_XLOAD && lane == 0) {
    ptx::tma_prefetch_desc(&tm_x);
    ptx::tma_prefetch_desc(&tm_out);
  }
  if (warp == WARP_WLOAD && lane == 0) {
    ptx::tma_prefetch_desc(&tm_w);
    ptx::tma_prefetch_desc(&tm_s);
    if (BITS != 2) ptx::tma_prefetch_desc(&tm_b);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t lim = p.wait_limit_ns;

  auto give_up = [&]() {
    *abort_flag = 1;
    ptx::set_status(p.status, kStatusTimeout);
  };

  if (warp == WARP_XLOAD || warp == WARP_WLOAD) {
    // ---------------- TMA producers ----------------
    if (lane == 0) {
      const bool is_x = warp == WARP_XLOAD;
      const int S = is_x ? SX : SW;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int n_tile, m_tile;
        tile_coords(p, tile, n_tile, m_tile);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t par = ((it / S) & 1) ^ 1;
          if (!ptx::mbar_wait(is_x ? empty_x(s) : empty_w(s), par, lim, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          if (is_x) {
            ptx::mbar_arrive_expect_tx(full_x(s), X_STAGE_BYTES);
            ptx::tma_load_2d(x_stage(s), &tm_x, kb * BK, m_tile * TILE_M, full_x(s));
          } else {
            const uint32_t dst = sbase + w_stage(s);
            const int grp = (kb * BK) / C::kGroup;
            ptx::mbar_arrive_expect_tx(full_w(s), C::kWStride);
            ptx::tma_load_2d(dst, &tm_w, kb * C::kWRowBytes, n_tile * TILE_N, full_w(s));
            ptx::tma_load_2d(dst + C::kWTileBytes, &tm_s, n_tile * TILE_N, grp, full_w(s));
            if (BITS != 2) ptx::tma_load_2d(dst + C::kWTileBytes + SB_BYTES, &tm_b, n_tile * TILE_N, grp, full_w(s));
          }
        }
      }
      // Let every load this thread issued land before the block can exit.
      const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0;
      for (uint32_t i = first; i < it; ++i)
        ptx::mbar_wait(is_x ? full_x(i % S) : full_w(i % S), (i / S) & 1, lim, nullptr);
    }
  } else if (warp == WARP_MMA) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tcount) {
        // the epilogue has read the previous tile's accumulator out
        if (!ptx::mbar_wait(acc_empty, (tcount & 1) ^ 1, lim, abort_flag)) {
          give_up();
          break;
        }
        ptx::tc_fence_after();
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int sx = it % SX, sa = it % SA;
          if (!ptx::mbar_wait(full_x(sx), (it / SX) & 1, lim, abort_flag) ||
              !ptx::mbar_wait(full_a(sa), (it / SA) & 1, lim, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint32_t a_tmem = tmem_base + A_COL + sa * A_STAGE_COLS + kk * (UMMA_K / 2);
            const uint64_t bdesc = ptx::smem_desc_sw128_kmajor(x_stage(sx) + kk * UMMA_K * 2);
            ptx::tc_mma_f16_ts(tmem_base + ACC_COL, a_tmem, bdesc, IDESC, (kb | kk) != 0);
          }
          ptx::tc_commit(empty_x(sx));
          ptx::tc_commit(empty_a(sa));
        }
        if (!ok) break;
        ptx::tc_commit(acc_full);
      }
      // All MMAs issued above complete before TMEM is released.
      ptx::tc_commit(drain_bar);
      ptx::mbar_wait(drain_bar, 0, lim, nullptr);
    }
  } else if (warp < WARP_EPI0) {
    // ---------------- dequantisers: packed smem tile -> bf16 in TMEM ----------------
    // Set `set` takes the CTA's K blocks it = set, set + DEQ_SETS, ... (counted
    // over all its tiles), so DEQ_SETS blocks are in flight per weight row.
    const int d = warp - WARP_DEQ0;
    const int set = d / DEQ_WARPS_PER_SET;
    const int q = warp & 3;                      // TMEM lane quarter this warp may write
    const int h = (d >> 2) & 1;                  // which 32-k half of each 64-k block
    const int r = 32 * q + lane;                 // tile row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const int my_tiles = (p.num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                         static_cast<int>(gridDim.x);
    const uint32_t total = static_cast<uint32_t>(my_tiles) * static_cast<uint32_t>(p.num_kb);
    for (uint32_t it = set; it < total; it += DEQ_SETS) {
      {
        const int sw = it % SW, sa = it % SA;
        if (!warp_wait(full_w(sw), (it / SW) & 1, lim, abort_flag) ||
            !warp_wait(empty_a(sa), ((it / SA) & 1) ^ 1, lim, abort_flag)) {
          if (lane == 0) give_up();
          break;
        }
        ptx::tc_fence_after();  // the MMA that last read this A stage has completed
        const uint8_t* wst = smem + w_stage(sw);
        const float s_cur = deq::h2f(reinterpret_cast<const uint16_t*>(wst + C::kWTileBytes)[r]);
        const float b_cur =
            BITS == 2 ? 0.f : deq::h2f(reinterpret_cast<const uint16_t*>(wst + C::kWTileBytes + SB_BYTES)[r]);
        const uint8_t* wsrc = wst + r * C::kWRowBytes + h * (C::kWRowBytes / 2);
        uint4 o[4];  // 4 chunks of 8 consecutive k = this thread's 32 k
        if constexpr (BITS == 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(wsrc);
          o[0] = deq::chunk_4bit(v.x, s_cur, b_cur);
          o[1] = deq::chunk_4bit(v.y, s_cur, b_cur);
          o[2] = deq::chunk_4bit(v.z, s_cur, b_cur);
          o[3] = deq::chunk_4bit(v.w, s_cur, b_cur);
        } else if constexpr (BITS == 8) {
          const uint4 v0 = *reinterpret_cast<const uint4*>(wsrc);
          const uint4 v1 = *reinterpret_cast<const uint4*>(wsrc + 16);
          o[0] = deq::chunk_8bit(v0.x, v0.y, s_cur, b_cur);
          o[1] = deq::chunk_8bit(v0.z, v0.w, s_cur, b_cur);
          o[2] = deq::chunk_8bit(v1.x, v1.y, s_cur, b_cur);
          o[3] = deq::chunk_8bit(v1.z, v1.w, s_cur, b_cur);
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(wsrc);
          const uint32_t hs = deq::ternary_half_scale2(s_cur);
          o[0] = deq::chunk_ternary<0>(v.x, hs);
          o[1] = deq::chunk_ternary<1>(v.x, hs);
          o[2] = deq::chunk_ternary<0>(v.y, hs);
          o[3] = deq::chunk_ternary<1>(v.y, hs);
        }
        // The packed stage has been read: give it back to the W producer.
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(empty_w(sw));
        const uint32_t regs[16] = {o[0].x, o[0].y, o[0].z, o[0].w, o[1].x, o[1].y, o[1].z, o[1].w,
                                   o[2].x, o[2].y, o[2].z, o[2].w, o[3].x, o[3].y, o[3].z, o[3].w};
        ptx::tmem_st_32x32b_x16(tmem_base + lane_addr + A_COL + sa * A_STAGE_COLS + h * 16, regs);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(full_a(sa));
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;                        // TMEM lane quarter this warp may access
    const int ep = threadIdx.x - 32 * WARP_EPI0;   // 0..127
    const int n_local = 32 * q + lane;
    uint16_t* stg = reinterpret_cast<uint16_t*>(smem + C::kOffOut);
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      int n_tile, m_tile;
      tile_coords(p, tile, n_tile, m_tile);
      const int n0 = n_tile * TILE_N;
      const int m0 = m_tile * TILE_M;
      const int n = n0 + n_local;
      const float bias_f =
          (p.bias && n < p.N) ? __bfloat162float(__ushort_as_bfloat16(p.bias[n])) : 0.f;
      const bool got = warp_wait(acc_full, tcount & 1, lim, abort_flag);
      if (!got && lane == 0) {
        *epi_abort = 1;
        give_up();
      }
      // the staging copy of the previous tile has been read by its TMA store
      if (ep == 0) ptx::bulk_wait_group_read<0>();
      ptx::named_bar_sync(EPI_BAR_ID, 32 * NUM_EPI_WARPS);  // all four warps agree before going on
      if (*epi_abort) break;
      ptx::tc_fence_after();
      const int rows_left = p.M - m0;
      const int chunks = rows_left >= TILE_M ? TILE_M / OUT_ROWS : (rows_left + OUT_ROWS - 1) / OUT_ROWS;
      for (int cch = 0; cch < chunks; ++cch) {
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(tmem_base + ACC_COL + cch * OUT_ROWS + (static_cast<uint32_t>(32 * q) << 16), v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < OUT_ROWS; ++j) {
          const float f = __uint_as_float(v[j]) + bias_f;
          stg[(cch * OUT_ROWS + j) * TILE_N + n_local] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
        }
      }
      // this warp has read its whole accumulator quarter: hand it back
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty);
      ptx::fence_proxy_async_smem();
      ptx::named_bar_sync(EPI_BAR_ID, 32 * NUM_EPI_WARPS);
      if (ep == 0) {
        ptx::tma_store_2d(&tm_out, sbase + C::kOffOut, n0, m0);
        ptx::bulk_commit_group();
      }
    }
    if (ep == 0) ptx::bulk_wait_group<0>();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int BITS>
int launch_fmt(const Problem& pr, int nsm) {
  using C = Cfg<BITS>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(large_m_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  int st = cuda_check(attr_err, "cudaFuncSetAttribute(large_m_kernel)");
  if (st != QGEMM_OK) return st;
  CUtensorMap tm_x, tm_w, tm_s, tm_b, tm_out;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;
  const uint64_t groups = static_cast<uint64_t>(pr.K) / C::kGroup;
  const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
  if ((st = make_tensor_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.X, pr.K, pr.M, uint64_t(pr.K) * 2, BK,
                        TILE_M, CU_TENSOR_MAP_SWIZZLE_128B, "X")) != QGEMM_OK)
    return st;
  if ((st = make_tensor_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.packed, wbytes, pr.N, wbytes,
                        C::kWRowBytes, TILE_N, none, "W")) != QGEMM_OK)
    return st;
  if ((st = make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.scales, pr.N, groups, uint64_t(pr.N) * 2,
                        TILE_N, 1, none, "scales")) != QGEMM_OK)
    return st;
  if (BITS != 2) {
    if ((st = make_tensor_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.biases, pr.N, groups, uint64_t(pr.N) * 2,
                          TILE_N, 1, none, "biases")) != QGEMM_OK)
      return st;
  } else {
    tm_b = tm_s;  // unused for ternary
  }
  if ((st = make_tensor_map_2d(&tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.out, pr.N, pr.M, uint64_t(pr.N) * 2,
                        TILE_N, TILE_M, none, "out")) != QGEMM_OK)
    return st;
  unsigned int* status;
  if ((st = status_word(&status)) != QGEMM_OK) return st;
  Params kp;
  kp.M = pr.M;
  kp.N = pr.N;
  kp.K = pr.K;
  kp.num_m_tiles = (pr.M + TILE_M - 1) / TILE_M;
  kp.num_n_tiles = (pr.N + TILE_N - 1) / TILE_N;
  kp.num_tiles = kp.num_m_tiles * kp.num_n_tiles;
  const int grid = kp.num_tiles < nsm ? kp.num_tiles : nsm;
  // The grid works on `grid` consecutive tiles at a time. Walk the dimension
  // that keeps fewer bytes of activation panels (256 tokens x K) and weight
  // panels (128 rows x K, packed) live in L2 at once.
  {
    const double x_panel = double(TILE_M) * pr.K * 2;
    const double w_panel = double(TILE_N) * pr.K * BITS / 8;
    auto live = [&](int fast, int slow, double fast_panel, double slow_panel) {
      const int f = fast < grid ? fast : grid;
      return f * fast_panel + double((grid + fast - 1) / fast) * slow_panel;
    };
    kp.m_fastest = live(kp.num_m_tiles, kp.num_n_tiles, x_panel, w_panel) <=
                   live(kp.num_n_tiles, kp.num_m_tiles, w_panel, x_panel);
  }
  kp.num_kb = pr.K / BK;
  kp.bias = pr.bias;
  kp.wait_limit_ns = wait_limit_ns();
  kp.status = status;
  large_m_kernel<BITS><<<grid, NUM_THREADS, C::kSmemBytes, pr.stream>>>(tm_x, tm_w, tm_s, tm_b, tm_out, kp);
  return cuda_check(cudaGetLastError(), "large_m_kernel launch");
}

}  // namespace lm

int launch_large_m(const Problem& p) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  switch (p.bits) {
    case 4: return lm::launch_fmt<4>(p, nsm);
    case 8: return lm::launch_fmt<8>(p, nsm);
    default: return lm::launch_fmt<2>(p, nsm);
  }
}

}  // namespace qg
