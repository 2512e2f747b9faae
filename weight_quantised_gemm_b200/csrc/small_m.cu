// Small-M path (M <= 16): a memory-bound kernel that streams the packed
// weights once.
//
// pictor's README ("Extreme quantization is first-class") names GEMV paths
// built for sub-byte weights; at decode-sized M the packed bytes set the time,
// so this kernel is built around keeping HBM busy:
//
// * One CTA per SM owns a contiguous range of weight rows (whole n8 blocks).
//   A producer warp streams that range through a shared-memory ring with TMA:
//   per stage, the packed codes of 128 bytes of K for every row (128-byte
//   swizzle), the stage's fp16 scales (and biases) as one box, and the
//   matching slice of the activations, copied row by row with bulk copies
//   into a padded layout. The ring holds up to eight stages, so at the
//   workloads' K every load of the CTA is in flight from the start.
// * Eight consumer warps turn codes into bf16 in registers and feed warp-level
//   mma.sync (m16n8k16, bf16 in, fp32 accumulate): the activations are the
//   16-row A operand (rows past M are zero), the weights the 8-column B.
//   The warps split each stage by whole groups and meet once, at the end, in
//   shared memory.
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
#include "qgemm_internal.h"

namespace qg {
namespace sm {

constexpr int NBMAX = 12;             // n8 blocks (of 8 weight rows) per CTA, at most
constexpr int NPMAX = NBMAX / 2;      // n16 pairs of blocks: the weight rows of one mma
constexpr int PPW = NPMAX;            // pairs per consumer warp
constexpr int NUM_CONSUMER_WARPS = 8;
constexpr int WARP_PRODUCER = NUM_CONSUMER_WARPS;
constexpr int NUM_THREADS = 32 * (NUM_CONSUMER_WARPS + 1);  // 288
constexpr int MAX_STAGES = 8;
constexpr int ROW_BYTES_PER_STAGE = 128;  // one 128-byte swizzle row of packed codes
constexpr int RING_BUDGET = 196608;       // bytes of shared memory for the ring

template <int BITS>
struct Fmt {
  static constexpr int G = BITS == 2 ? 128 : 64;          // group size
  static constexpr int KS = ROW_BYTES_PER_STAGE * 8 / BITS;  // k per stage: 512, 256 or 128
  static constexpr int GS = KS / G;                        // groups per stage: 4, 4, 2
  static constexpr int STEPS = G / 16;                     // mma k-steps per group
  static constexpr int NSETS = NUM_CONSUMER_WARPS / GS;  // warp sets sharing out the stages
  static constexpr int GBYTES = G * BITS / 8;              // packed bytes per row and group
};

struct Params {
  const uint16_t* X;     // bf16 [M, K]
  const uint16_t* bias;  // bf16 [N] or null
  uint16_t* out;         // bf16 [M, N]
  int M, N, K;
  int bpc;               // n8 blocks per CTA
  int num_stages;        // K / KS, rounded up
  int ring;              // ring depth
  int stage_bytes;       // bytes per ring stage (multiple of 1024)
  int off_s, off_b, off_x, x_stride;  // offsets inside a stage; X row stride in bytes
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

// Byte offset, inside a stage row, of the 32-bit word that holds quad thread
// c's 4 codes (k = 4c .. 4c+3) of step k of group gs. Rows carry the 128-byte
// swizzle: logical 16-byte chunk j of row r sits at physical chunk j ^ (r % 8).
//   ternary: one word per 16-k step (quad threads share it);
//   4-bit:   two words per step, thread c reads word c / 2;
//   8-bit:   four words per step, thread c reads word c.
template <int BITS>
__device__ __forceinline__ int word_offset(int gs, int k, int c, int r7) {
  int chunk, wic;
  if constexpr (BITS == 2) {
    chunk = 2 * gs + (k >> 2);
    wic = k & 3;
  } else if constexpr (BITS == 4) {
    chunk = 2 * gs + (k >> 1);
    wic = 2 * (k & 1) + (c >> 1);
  } else {
    chunk = 4 * gs + k;
    wic = c;
  }
  return ((chunk ^ r7) << 4) + 4 * wic;
}

// B operand of one step for quad thread c from its word: codes 4c .. 4c+3 as
// two bf16x2 registers (k pairs (4c, 4c+1) and (4c+2, 4c+3)).
template <int BITS>
__device__ __forceinline__ void decode_word(uint32_t x, int c, uint32_t& b0, uint32_t& b1) {
  if constexpr (BITS == 2) {
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

template <int BITS, int MT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    small_m_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_b, const Params p) {
  using F = Fmt<BITS>;
  constexpr int STEPS = F::STEPS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  const int nblocks_total = p.N / 8;
  const int blk0 = blockIdx.x * p.bpc;
  const int nb = min(p.bpc, nblocks_total - blk0);
  const int n0 = 8 * blk0;
  const int R = 8 * p.bpc;  // rows per TMA box (rows past N read as zeros)
  const int data_bytes = max(p.ring * p.stage_bytes, NUM_CONSUMER_WARPS * PPW * 2 * 32 * 16);
  const uint32_t bar0 = sbase + data_bytes;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (MAX_STAGES + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + data_bytes + 16 * MAX_STAGES);
  const uint64_t lim = p.wait_limit_ns;
  // Each CTA walks the K slices starting at its own offset: every CTA reads
  // the same activations, and rotating the order spreads those reads over
  // the L2 instead of sending all CTAs to the same lines at once.
  const int rot = blockIdx.x % p.num_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), F::GS);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  auto give_up = [&]() {
    *abort_flag = 1;
    ptx::set_status(p.status, kStatusTimeout);
  };

  // acc[p][h][j]: weight rows 16p + g (j < 2) and 16p + g + 8 (j >= 2), tokens
  // 8h + 2c + (j & 1)
  constexpr int TH = MT > 8 ? 2 : 1;
  float acc[PPW][TH][4];
#pragma unroll
  for (int q = 0; q < PPW; ++q)
#pragma unroll
    for (int h = 0; h < TH; ++h)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[q][h][j] = 0.f;
  // Every CTA runs NPMAX n16 pairs with no per-pair branch, so the compiler can
  // interleave the pairs' loads, decodes and mma. Rows past the CTA's own
  // (past 8 * nb) are computed from whatever the stage holds there and are
  // never written out; the stage reserves room for all 16 * NPMAX rows.

  if (warp == WARP_PRODUCER) {
    // ---------------- producer: TMA boxes and bulk copies into the ring ----------------
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tm_w);
      ptx::tma_prefetch_desc(&tm_s);
      const int sb_bytes = F::GS * R * 2;
      int t = 0;
      for (; t < p.num_stages; ++t) {
        const int s = t % p.ring;
        if (!ptx::mbar_wait(empty(s), ((t / p.ring) & 1) ^ 1, lim, abort_flag)) {
          give_up();
          break;
        }
        const int kt = (t + rot) % p.num_stages;  // which K slice this ring slot carries
        const int valid = min(F::KS, p.K - kt * F::KS);
        const uint32_t st = sbase + s * p.stage_bytes;
        ptx::mbar_arrive_expect_tx(full(s), R * ROW_BYTES_PER_STAGE + sb_bytes * (BITS == 2 ? 1 : 2) +
                                                p.M * valid * 2);
        ptx::tma_load_2d(st, &tm_w, kt * ROW_BYTES_PER_STAGE, n0, full(s));
        ptx::tma_load_2d(st + p.off_s, &tm_s, n0, kt * F::GS, full(s));
        if (BITS != 2) ptx::tma_load_2d(st + p.off_b, &tm_b, n0, kt * F::GS, full(s));
        for (int m = 0; m < p.M; ++m)
          bulk_copy_g2s(st + p.off_x + m * p.x_stride, p.X + static_cast<size_t>(m) * p.K + kt * F::KS, valid * 2,
                        full(s));
      }
      // Let every copy this thread issued land before the ring is reused.
      const int first = t > p.ring ? t - p.ring : 0;
      for (int i = first; i < t; ++i) ptx::mbar_wait(full(i % p.ring), (i / p.ring) & 1, lim, nullptr);
    }
  } else {
    // ---------------- consumers ----------------
    const int gs = warp % F::GS;                   // group of the stage this warp takes
    const int half = 0;                            // every warp takes all of the CTA's pairs
    for (int t = (warp / F::GS) % F::NSETS; t < p.num_stages; t += F::NSETS) {
      const int s = t % p.ring;
      if (!warp_wait(full(s), (t / p.ring) & 1, lim, abort_flag)) {
        if (lane == 0) give_up();
        break;
      }
      const uint8_t* st = smem + s * p.stage_bytes;
      const int kt = (t + rot) % p.num_stages;
      if (kt * F::KS + gs * F::G < p.K) {
        // activations of this group (the B operand): tokens g and g + 8,
        // k = gs*G + 16*step + 4c .. +3
        const uint8_t* xg = st + p.off_x + g * p.x_stride + (gs * F::G + 4 * c) * 2;
        const bool ga = g < p.M, gb = MT > 8 && g + 8 < p.M;
        float xs[TH][4];  // sum of x over the group per token (affine)
        float tmp[PPW][TH][4];
#pragma unroll
        for (int h = 0; h < TH; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) xs[h][j] = 0.f;
#pragma unroll
        for (int q = 0; q < PPW; ++q)
#pragma unroll
          for (int h = 0; h < TH; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) tmp[q][h][j] = 0.f;
        // weight row 16 * (half * PPW + q) + g of this warp's pair q
        const uint8_t* rowg = st + (16 * half * PPW + g) * ROW_BYTES_PER_STAGE;
#pragma unroll
        for (int k = 0; k < STEPS; ++k) {
          const uint2 x0 = ga ? *reinterpret_cast<const uint2*>(xg + 32 * k) : make_uint2(0u, 0u);
          const uint2 x1 = gb ? *reinterpret_cast<const uint2*>(xg + 8 * p.x_stride + 32 * k) : make_uint2(0u, 0u);
          if constexpr (BITS != 2) {
            const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
            mma_bf16_16816(xs[0], ones, x0.x, x0.y);
            if constexpr (TH > 1) mma_bf16_16816(xs[TH - 1], ones, x1.x, x1.y);
          }
          const int wo = word_offset<BITS>(gs, k, c, g);  // rows g and g + 8 share the swizzle
#pragma unroll
          for (int q = 0; q < PPW; ++q) {
            const uint8_t* r0 = rowg + q * 16 * ROW_BYTES_PER_STAGE;
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(r0 + wo);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(r0 + 8 * ROW_BYTES_PER_STAGE + wo);
            uint32_t a[4];
            decode_word<BITS>(w0, c, a[0], a[2]);  // row g: k pairs (4c, 4c+1), (4c+2, 4c+3)
            decode_word<BITS>(w1, c, a[1], a[3]);  // row g + 8
            mma_bf16_16816(tmp[q][0], a, x0.x, x0.y);
            if constexpr (TH > 1) mma_bf16_16816(tmp[q][TH - 1], a, x1.x, x1.y);
          }
        }
        // apply the group's scale (and bias) of rows 16q + g and 16q + g + 8
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + p.off_s) + gs * R;
        const uint16_t* bi = reinterpret_cast<const uint16_t*>(st + p.off_b) + gs * R;
#pragma unroll
        for (int q = 0; q < PPW; ++q) {
          {
            const int r0 = 16 * (half * PPW + q) + g;
            const float s2[2] = {deq::h2f(sc[r0]), deq::h2f(sc[r0 + 8])};
            float b2[2] = {0.f, 0.f};
            if constexpr (BITS != 2) {
              b2[0] = deq::h2f(bi[r0]);
              b2[1] = deq::h2f(bi[r0 + 8]);
            }
#pragma unroll
            for (int h = 0; h < TH; ++h)
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float sj = s2[j >> 1];
                if constexpr (BITS == 2) {
                  acc[q][h][j] = fmaf(0.5f * sj, tmp[q][h][j], acc[q][h][j]);
                } else {
                  const float d = BITS == 4 ? fmaf(-128.f, xs[h][j], tmp[q][h][j]) : tmp[q][h][j];
                  const float e = fmaf(b2[j >> 1], xs[h][j], acc[q][h][j]);
                  acc[q][h][j] = fmaf(sj, d, e);
                }
              }
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(empty(s));
    }
  }

  // ---------------- the warps' partial sums meet in shared memory ----------------
  __syncthreads();  // the ring is drained: reuse it
  float4* red = reinterpret_cast<float4*>(smem);  // [warp][pair of the warp][token half][lane]
  if (warp < NUM_CONSUMER_WARPS) {
#pragma unroll
    for (int q = 0; q < PPW; ++q)
#pragma unroll
        for (int h = 0; h < TH; ++h)
          red[((warp * PPW + q) * TH + h) * 32 + lane] =
              make_float4(acc[q][h][0], acc[q][h][1], acc[q][h][2], acc[q][h][3]);
  }
  __syncthreads();
  const int rows = 8 * nb;
  for (int i = threadIdx.x; i < p.M * rows; i += NUM_THREADS) {
    const int m = i / rows, nl = i % rows;
    const int q = nl >> 4, hrow = (nl >> 3) & 1, gg = nl & 7;
    const int h = m >> 3, cc = (m & 7) >> 1;
    const int j = 2 * hrow + (m & 1);
    const int ln = 4 * gg + cc;
    float v = 0.f;
    const int wh = q / PPW, ql = q % PPW;  // the warps holding pair q: those of half wh
    constexpr int WPH = NUM_CONSUMER_WARPS;
#pragma unroll
    for (int w = wh * WPH; w < (wh + 1) * WPH; ++w) {
      const float4 f = red[((w * PPW + ql) * TH + h) * 32 + ln];
      v += j == 0 ? f.x : j == 1 ? f.y : j == 2 ? f.z : f.w;
    }
    const int n = n0 + nl;
    if (p.bias) v += __bfloat162float(__ushort_as_bfloat16(p.bias[n]));
    p.out[static_cast<size_t>(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
constexpr int kMaxSmem = 232448;

template <int BITS, int MT>
int launch_fmt(const Problem& pr, int nsm) {
  using F = Fmt<BITS>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(small_m_kernel<BITS, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  });
  int st = cuda_check(attr_err, "cudaFuncSetAttribute(small_m_kernel)");
  if (st != QGEMM_OK) return st;

  Params kp;
  kp.X = static_cast<const uint16_t*>(pr.X);
  kp.bias = pr.bias;
  kp.out = static_cast<uint16_t*>(pr.out);
  kp.M = pr.M;
  kp.N = pr.N;
  kp.K = pr.K;
  const int nblocks = pr.N / 8;
  int bpc = (nblocks + nsm - 1) / nsm;
  bpc = bpc < NBMAX ? bpc : NBMAX;
  const int grid = (nblocks + bpc - 1) / bpc;
  const int R = 8 * bpc;
  kp.bpc = bpc;
  kp.num_stages = (pr.K + F::KS - 1) / F::KS;
  const int sb = F::GS * R * 2;
  // TMA tile destinations start on 128-byte boundaries (the packed box on a
  // 1024-byte one, for its 128-byte swizzle); bulk copies need 16 bytes.
  const int rows_read = R > 16 * NPMAX ? R : 16 * NPMAX;  // rows the consumers touch
  kp.off_s = rows_read * ROW_BYTES_PER_STAGE;
  kp.off_b = (kp.off_s + sb + 127) & ~127;
  kp.off_x = (kp.off_b + (BITS == 2 ? 0 : sb) + 127) & ~127;
  kp.x_stride = F::KS * 2 + 16;  // +16 B staggers rows across banks
  kp.stage_bytes = (kp.off_x + pr.M * kp.x_stride + 1023) & ~1023;
  int ring = RING_BUDGET / kp.stage_bytes;
  ring = ring < MAX_STAGES ? ring : MAX_STAGES;
  ring = ring < kp.num_stages ? ring : kp.num_stages;
  kp.ring = ring < 1 ? 1 : ring;
  const int red_bytes = NUM_CONSUMER_WARPS * PPW * 2 * 32 * 16;
  const int data_bytes = kp.ring * kp.stage_bytes > red_bytes ? kp.ring * kp.stage_bytes : red_bytes;
  const int smem = data_bytes + 16 * MAX_STAGES + 16 + 1024;
  if (smem > kMaxSmem) return fail(QGEMM_ERR_UNSUPPORTED, "small-M stage of %d bytes does not fit", kp.stage_bytes);
  if (kp.off_s % 128 || kp.off_b % 128 || kp.off_x % 16 || kp.x_stride % 16 || kp.stage_bytes % 1024)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: small-M stage layout misaligned");
  kp.wait_limit_ns = wait_limit_ns();
  if ((st = status_word(&kp.status)) != QGEMM_OK) return st;

  CUtensorMap tm_w, tm_s, tm_b;
  const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;
  const uint64_t groups = static_cast<uint64_t>(pr.K) / F::G;
  if ((st = make_tensor_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.packed, wbytes, pr.N, wbytes,
                               ROW_BYTES_PER_STAGE, R, CU_TENSOR_MAP_SWIZZLE_128B, "W")) != QGEMM_OK)
    return st;
  if ((st = make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.scales, pr.N, groups,
                               uint64_t(pr.N) * 2, R, F::GS, CU_TENSOR_MAP_SWIZZLE_NONE, "scales")) != QGEMM_OK)
    return st;
  if (BITS != 2) {
    if ((st = make_tensor_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.biases, pr.N, groups,
                                 uint64_t(pr.N) * 2, R, F::GS, CU_TENSOR_MAP_SWIZZLE_NONE, "biases")) != QGEMM_OK)
      return st;
  } else {
    tm_b = tm_s;  // unused for ternary
  }
  small_m_kernel<BITS, MT><<<grid, NUM_THREADS, smem, pr.stream>>>(tm_w, tm_s, tm_b, kp);
  return cuda_check(cudaGetLastError(), "small_m_kernel launch");
}

template <int BITS>
int launch_bits(const Problem& pr, int nsm) {
  return pr.M <= 8 ? launch_fmt<BITS, 8>(pr, nsm) : launch_fmt<BITS, 16>(pr, nsm);
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
    default: return sm::launch_bits<2>(p, nsm);
  }
}

}  // namespace qg
