// Grouped small-M launch: several independent GEMVs (M <= 16 each, one
// weight format) in one persistent kernel, so that the launch and the first
// bytes' latency are paid once for all of them and HBM streams their weights
// back to back.
//
// At decode-sized M a GEMV is a read of its packed weights, and a single
// 10-40 MB read is dominated by the launch and the time before the first
// bytes arrive rather than by bandwidth. pictor's README ("Extreme
// quantization is first-class") builds GEMV paths for sub-byte weights; the
// linears of one transformer block that take the same input (the image and
// text streams' projections of a double-stream block, the modulation
// vectors) are independent, and one launch can serve them all.
//
// Work items are (problem, block of 32 weight rows) with the whole K of that
// problem. The host assigns items to CTAs longest first, each to the least
// loaded CTA (load = the item's K stages), and passes each CTA its list. One
// CTA per SM; a producer warp streams every item's stages through one
// shared-memory ring without a break between items, and eight consumer
// warps (warp w: scale group w of every stage) turn codes into bf16 and feed
// mma.sync as in the one-problem kernel. At the end of an item the
// consumers' partial sums meet in a reduction area of their own (the ring
// keeps filling meanwhile), and they write the item's outputs with the bias.

#include <cuda.h>

#include <algorithm>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "qgemm_internal.h"
#include "small_m_common.cuh"
#include "small_m_layout.cuh"

namespace qg {
namespace smg {

using sm::Fmt;
using sm::GS;

constexpr int NUM_CONSUMER_WARPS = 8;
constexpr int WARP_PRODUCER = NUM_CONSUMER_WARPS;
constexpr int NUM_THREADS = 32 * (NUM_CONSUMER_WARPS + 1);
constexpr int CONSUMER_THREADS = 32 * NUM_CONSUMER_WARPS;
constexpr int NP = 2;              // 16-row pairs per item
constexpr int R = 16 * NP;         // weight rows per item
constexpr int MAX_STAGES = 24;     // ring slots: 32-row stages are small (5-18 KB)
constexpr int SMEM_LIMIT = 232448;
constexpr int CONSUMER_BAR = 1;    // named barrier of the consumer warps

struct GProblem {
  const uint16_t* X;     // bf16 [M, K]
  const uint16_t* bias;  // bf16 [N] or null
  uint16_t* out;         // bf16 [M, N]
  int M, N, K;
  int num_stages;        // ceil(K / KS)
  int unit_shift;        // log2 of U, the bytes per swizzled row piece
};

struct GParams {
  GProblem prob[kGroupedMaxProblems];
  int ring;              // ring depth
  int stage_bytes;       // bytes per ring stage (multiple of 1024)
  int off_s, off_b;      // scales and biases inside a stage
  int red_off;           // the consumers' reduction area
  int bar_off;           // mbarriers and the abort flag
  uint64_t wait_limit_ns;
  unsigned int* status;
  uint16_t cta_begin[kGroupedMaxCtas + 1];  // CTA c works on items[cta_begin[c] .. cta_begin[c + 1])
  uint16_t items[kGroupedMaxItems];         // problem << 12 | row block
};

struct GMaps {
  CUtensorMap w[kGroupedMaxProblems];
  CUtensorMap s[kGroupedMaxProblems];
  CUtensorMap b[kGroupedMaxProblems];
};

// Named barrier of `n` threads that also returns whether any of them passed
// `pred` true.
__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

template <int BITS, int MT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_kernel(const __grid_constant__ GMaps maps, const __grid_constant__ GParams p) {
  using F = Fmt<BITS>;
  constexpr int STEPS = F::STEPS;
  constexpr int TH = MT > 8 ? 2 : 1;  // 8-token halves
  constexpr int NLP = R + 4;          // row pitch of the partial sums
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) ptx::set_status(p.status, kStatusLayout);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t bar0 = sbase + p.bar_off;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (MAX_STAGES + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.bar_off + 16 * MAX_STAGES);
  const uint64_t lim = p.wait_limit_ns;
  const int ib = p.cta_begin[blockIdx.x], ie = p.cta_begin[blockIdx.x + 1];

  // Stage t of item `it` (the CTA's gs-th stage overall) into ring slot gs % ring.
  auto issue_stage = [&](int it, int t, uint32_t gs) {
    constexpr int sb_bytes = GS * R * 2;
    const int pi = p.items[it] >> 12, rb = p.items[it] & 0xFFF;
    const GProblem& P = p.prob[pi];
    const int n0 = rb * R, nst = P.num_stages, rot = rb % nst;
    const int units = F::ROWB >> P.unit_shift;
    const int s = gs % p.ring, kt = (t + rot) % nst;
    const uint32_t st = sbase + s * p.stage_bytes;
    ptx::mbar_arrive_expect_tx(full(s), R * F::ROWB + sb_bytes * (BITS <= 2 ? 1 : 2));
    ptx::tma_load_3d(st, &maps.w[pi], 0, n0, kt * units, full(s));
    ptx::tma_load_2d(st + p.off_s, &maps.s[pi], n0, kt * GS, full(s));
    if (BITS > 2) ptx::tma_load_2d(st + p.off_b, &maps.b[pi], n0, kt * GS, full(s));
  };
  // The producer's lane 0 sets up the ring and puts the first stage in flight
  // before the block-wide barrier (as in the one-problem kernel).
  if (threadIdx.x == 32 * WARP_PRODUCER) {
    for (int s = 0; s < p.ring; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), NUM_CONSUMER_WARPS);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
    if (ib < ie) issue_stage(ib, 0, 0);
  }
  __syncthreads();
  auto give_up = [&]() {
    *abort_flag = 1;
    ptx::set_status(p.status, kStatusTimeout);
  };

  if (warp == WARP_PRODUCER) {
    // ---------------- producer: every item's stages, back to back ----------------
    // The weights do not depend on the previous grid: stream at once, and let
    // the next grid launch (both no-ops without the launch attribute).
    sm::griddep_launch_dependents();
    if (lane == 0) {
      uint32_t gs = 0;  // stages issued so far, over all items
      bool ok = true;
      for (int it = ib; ok && it < ie; ++it) {
        const int nst = p.prob[p.items[it] >> 12].num_stages;
        for (int t = 0; t < nst; ++t, ++gs) {
          if (gs == 0) continue;  // issued before the block-wide barrier
          const int s = gs % p.ring;
          if (gs >= static_cast<uint32_t>(p.ring) &&
              !ptx::mbar_wait(empty(s), ((gs / p.ring) & 1) ^ 1, lim, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          issue_stage(it, t, gs);
        }
      }
      // let every copy issued above land before the block can exit
      const uint32_t first = gs > static_cast<uint32_t>(p.ring) ? gs - p.ring : 0;
      for (uint32_t i = first; i < gs; ++i) ptx::mbar_wait(full(i % p.ring), (i / p.ring) & 1, lim, nullptr);
    }
  } else {
    // ---------------- consumers ----------------
    sm::griddep_launch_dependents();
    sm::griddep_wait();  // X may be the previous grid's output, and out may still be read by it
    const int gl = warp;  // scale group gl of every stage
    float* red = reinterpret_cast<float*>(smem + p.red_off);  // [group lane][token][NLP]
    uint32_t gs = 0;
    for (int it = ib; it < ie; ++it) {
      const int pi = p.items[it] >> 12, rb = p.items[it] & 0xFFF;
      const GProblem& P = p.prob[pi];
      const int n0 = rb * R, nst = P.num_stages, rot = rb % nst;
      const int ush = P.unit_shift;
      const int key16 = sm::swizzle_key16(g, ush);
      const bool ga = g < P.M, gb = MT > 8 && g + 8 < P.M;  // tokens g and g + 8 exist
      // acc[q][h][j]: weight rows 16q + g (j < 2) and 16q + g + 8 (j >= 2), tokens 8h + 2c + (j & 1)
      float acc[NP][TH][4];
#pragma unroll
      for (int q = 0; q < NP; ++q)
#pragma unroll
        for (int h = 0; h < TH; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[q][h][j] = 0.f;
      bool ok = true;
      for (int t = 0; t < nst; ++t, ++gs) {
        const int s = gs % p.ring;
        const int kt = (t + rot) % nst;
        const int k0 = kt * F::KS + gl * F::G;
        const bool in = k0 < P.K;
        // the B fragments (tokens g and g + 8, thread c's chunk of the group)
        // straight from global memory, issued before the wait so that the two
        // latencies overlap
        constexpr int XV = F::G / 32;
        uint4 xr[TH][XV];
        const uint4* x0p = reinterpret_cast<const uint4*>(P.X + static_cast<size_t>(g) * P.K + k0 + c * (F::G / 4));
        const uint4* x1p =
            reinterpret_cast<const uint4*>(P.X + static_cast<size_t>(g + 8) * P.K + k0 + c * (F::G / 4));
#pragma unroll
        for (int v = 0; v < XV; ++v) {
          xr[0][v] = (in && ga) ? __ldg(x0p + v) : make_uint4(0u, 0u, 0u, 0u);
          if constexpr (TH > 1) xr[TH - 1][v] = (in && gb) ? __ldg(x1p + v) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (!sm::warp_wait(full(s), (gs / p.ring) & 1, lim, abort_flag)) {
          if (lane == 0) give_up();
          ok = false;
          break;
        }
        const uint8_t* st = smem + s * p.stage_bytes;
        if (in) {
          float xs[TH][4];  // sum of x over the group per token (affine)
          float tmp[NP][TH][4];
#pragma unroll
          for (int h = 0; h < TH; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) xs[h][j] = 0.f;
#pragma unroll
          for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int h = 0; h < TH; ++h)
#pragma unroll
              for (int j = 0; j < 4; ++j) tmp[q][h][j] = 0.f;
          // this thread's packed chunks of the group, rows 16q + g and 16q + g + 8
          // (the two rows share the swizzle key), one load per row
          constexpr int CW = sm::Chunk<BITS>::WORDS;
          uint32_t w0[NP][CW], w1[NP][CW];
          {
            const uint8_t* wc = st + sm::piece_offset<R>(sm::chunk_offset<BITS>(gl, c), ush, key16);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
              const int r0 = 16 * q + g;
              sm::load_chunk<BITS>(wc + (r0 << ush), w0[q]);
              sm::load_chunk<BITS>(wc + ((r0 + 8) << ush), w1[q]);
            }
          }
#pragma unroll
          for (int k = 0; k < STEPS; ++k) {
            const uint2 x0 = sm::x_step(xr[0], k), x1 = sm::x_step(xr[TH - 1], k);
            if constexpr (BITS > 2) {
              const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
              sm::mma_bf16_16816(xs[0], ones, x0.x, x0.y);
              if constexpr (TH > 1) sm::mma_bf16_16816(xs[TH - 1], ones, x1.x, x1.y);
            }
#pragma unroll
            for (int q = 0; q < NP; ++q) {
              uint32_t a[4];
              sm::decode_quad<BITS>(w0[q][sm::step_word<BITS>(k)], sm::step_quad<BITS>(k), a[0], a[2]);
              sm::decode_quad<BITS>(w1[q][sm::step_word<BITS>(k)], sm::step_quad<BITS>(k), a[1], a[3]);
              sm::mma_bf16_16816(tmp[q][0], a, x0.x, x0.y);
              if constexpr (TH > 1) sm::mma_bf16_16816(tmp[q][TH - 1], a, x1.x, x1.y);
            }
          }
          // the group's scale (and bias) of rows 16q + g and 16q + g + 8
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + p.off_s) + gl * R;
          const uint16_t* bi = reinterpret_cast<const uint16_t*>(st + p.off_b) + gl * R;
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            const int r0 = 16 * q + g;
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
      // Every consumer warp reaches this barrier once per item, whether or
      // not its waits succeeded; if any gave up, all leave together.
      if (bar_any(CONSUMER_BAR, CONSUMER_THREADS, !ok)) break;
#pragma unroll
      for (int q = 0; q < NP; ++q)
#pragma unroll
        for (int h = 0; h < TH; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = 8 * h + 2 * c + (j & 1), nl = 16 * q + g + 8 * (j >> 1);
            red[(gl * MT + m) * NLP + nl] = acc[q][h][j];
          }
      ptx::named_bar_sync(CONSUMER_BAR, CONSUMER_THREADS);
      for (int i = threadIdx.x; i < P.M * R; i += CONSUMER_THREADS) {
        const int m = i / R, nl = i - m * R;
        const int n = n0 + nl;
        if (n >= P.N) continue;
        float v = 0.f;
#pragma unroll
        for (int l = 0; l < NUM_CONSUMER_WARPS; ++l) v += red[(l * MT + m) * NLP + nl];
        if (P.bias) v += __bfloat162float(__ushort_as_bfloat16(P.bias[n]));
        P.out[static_cast<size_t>(m) * P.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
      ptx::named_bar_sync(CONSUMER_BAR, CONSUMER_THREADS);  // the reduction area is free again
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int BITS, int MT>
int launch(const Problem* probs, int count, bool overlap, cudaStream_t stream, int nsm) {
  using F = Fmt<BITS>;
  const void* fn = reinterpret_cast<const void*>(grouped_kernel<BITS, MT>);
  int st = smem_opt_in(fn, SMEM_LIMIT, "cudaFuncSetAttribute(grouped small-M kernel)");
  if (st != QGEMM_OK) return st;
  static GParams kp;  // large: built in static storage under the launch lock
  static GMaps maps;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  kp = GParams{};
  // work items, longest first (stable), then each to the least loaded CTA
  std::vector<std::pair<int, int>> items;  // (stages, problem << 12 | row block)
  for (int i = 0; i < count; ++i) {
    const Problem& pr = probs[i];
    if (pr.M == 0) continue;
    const int blocks = (pr.N + R - 1) / R;
    if (blocks > 4096) return fail(QGEMM_ERR_UNSUPPORTED, "grouped: N=%d is above %d rows", pr.N, 4096 * R);
    const int nst = (pr.K + F::KS - 1) / F::KS;
    for (int b = 0; b < blocks; ++b) items.emplace_back(nst, (i << 12) | b);
  }
  if (items.empty()) return QGEMM_OK;
  if (static_cast<int>(items.size()) > kGroupedMaxItems)
    return fail(QGEMM_ERR_UNSUPPORTED, "grouped: %d row blocks of %d rows, at most %d", int(items.size()), R,
                kGroupedMaxItems);
  std::stable_sort(items.begin(), items.end(), [](const auto& a, const auto& b) { return a.first > b.first; });
  const int grid = std::min<int>({nsm, kGroupedMaxCtas, static_cast<int>(items.size())});
  std::vector<std::vector<int>> lists(grid);
  std::priority_queue<std::pair<long, int>, std::vector<std::pair<long, int>>, std::greater<>> load;
  for (int c = 0; c < grid; ++c) load.emplace(0L, c);
  for (const auto& it : items) {
    auto [l, c] = load.top();
    load.pop();
    lists[c].push_back(it.second);
    load.emplace(l + it.first, c);
  }
  int pos = 0;
  for (int c = 0; c < grid; ++c) {
    kp.cta_begin[c] = static_cast<uint16_t>(pos);
    for (int v : lists[c]) kp.items[pos++] = static_cast<uint16_t>(v);
  }
  kp.cta_begin[grid] = static_cast<uint16_t>(pos);

  // stage layout: R rows of packed codes, then the stage's scales (and biases)
  const int sb = GS * R * 2;
  kp.off_s = R * F::ROWB;
  kp.off_b = (kp.off_s + sb + 127) & ~127;
  kp.stage_bytes = (kp.off_b + (BITS <= 2 ? 0 : sb) + 1023) & ~1023;
  const int red_bytes = NUM_CONSUMER_WARPS * MT * (R + 4) * 4;
  const int tail = red_bytes + 16 * MAX_STAGES + 16;
  int ring = (SMEM_LIMIT - tail) / kp.stage_bytes;
  ring = ring < MAX_STAGES ? ring : MAX_STAGES;
  if (ring < 2) return fail(QGEMM_ERR_UNSUPPORTED, "internal: grouped stage of %d bytes", kp.stage_bytes);
  kp.ring = ring;
  kp.red_off = ring * kp.stage_bytes;
  kp.bar_off = (kp.red_off + red_bytes + 7) & ~7;
  const int smem = kp.bar_off + 16 * MAX_STAGES + 16;
  if (smem > SMEM_LIMIT || kp.off_s % 1024 || kp.off_b % 128 || kp.stage_bytes % 1024 || kp.red_off % 16)
    return fail(QGEMM_ERR_UNSUPPORTED, "internal: grouped small-M layout");
  kp.wait_limit_ns = wait_limit_ns();
  if ((st = status_word(&kp.status)) != QGEMM_OK) return st;

  for (int i = 0; i < count; ++i) {
    const Problem& pr = probs[i];
    GProblem& gp = kp.prob[i];
    gp.X = static_cast<const uint16_t*>(pr.X);
    gp.bias = pr.bias;
    gp.out = static_cast<uint16_t*>(pr.out);
    gp.M = pr.M;
    gp.N = pr.N;
    gp.K = pr.K;
    gp.num_stages = (pr.K + F::KS - 1) / F::KS;
    const uint64_t wbytes = static_cast<uint64_t>(pr.K) * BITS / 8;
    const int unit = wbytes % 128 == 0 ? 128 : wbytes % 64 == 0 ? 64 : 32;
    gp.unit_shift = unit == 128 ? 7 : unit == 64 ? 6 : 5;
    if (F::ROWB % unit || wbytes % unit)
      return fail(QGEMM_ERR_UNSUPPORTED, "internal: grouped rows are not whole %d-byte pieces", unit);
    if (pr.M == 0) {
      maps.w[i] = maps.s[i] = maps.b[i] = CUtensorMap{};
      continue;
    }
    const uint64_t groups = static_cast<uint64_t>(pr.K) / F::G;
    const uint64_t wdims[3] = {static_cast<uint64_t>(unit), static_cast<uint64_t>(pr.N), wbytes / unit};
    const uint64_t wstrides[2] = {wbytes, static_cast<uint64_t>(unit)};
    const uint32_t wbox[3] = {static_cast<uint32_t>(unit), static_cast<uint32_t>(R),
                              static_cast<uint32_t>(F::ROWB / unit)};
    const CUtensorMapSwizzle wswz = unit == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                    : unit == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_32B;
    if ((st = make_tensor_map_3d(&maps.w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.packed, wdims, wstrides, wbox, wswz,
                                 "grouped W")) != QGEMM_OK)
      return st;
    if ((st = make_tensor_map_2d(&maps.s[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.scales, pr.N, groups,
                                 uint64_t(pr.N) * 2, R, GS, CU_TENSOR_MAP_SWIZZLE_NONE, "grouped scales")) !=
        QGEMM_OK)
      return st;
    if (BITS > 2) {
      if ((st = make_tensor_map_2d(&maps.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.biases, pr.N, groups,
                                   uint64_t(pr.N) * 2, R, GS, CU_TENSOR_MAP_SWIZZLE_NONE, "grouped biases")) !=
          QGEMM_OK)
        return st;
    } else {
      maps.b[i] = maps.s[i];
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cuda_check(cudaLaunchKernelEx(&cfg, grouped_kernel<BITS, MT>, maps, kp), "grouped small-M kernel launch");
}

template <int BITS>
int launch_bits(const Problem* probs, int count, bool overlap, cudaStream_t stream, int nsm) {
  int mt = 0;
  for (int i = 0; i < count; ++i) mt = probs[i].M > mt ? probs[i].M : mt;
  return mt <= 8 ? launch<BITS, 8>(probs, count, overlap, stream, nsm)
                 : launch<BITS, 16>(probs, count, overlap, stream, nsm);
}

}  // namespace smg

int launch_small_m_grouped(const Problem* probs, int count, bool overlap, cudaStream_t stream) {
  int nsm;
  int st = sm_count(&nsm);
  if (st != QGEMM_OK) return st;
  if (count < 1 || count > kGroupedMaxProblems) return fail(QGEMM_ERR_INVALID_ARG, "grouped: %d problems", count);
  switch (probs[0].bits) {
    case 4: return smg::launch_bits<4>(probs, count, overlap, stream, nsm);
    case 8: return smg::launch_bits<8>(probs, count, overlap, stream, nsm);
    case 1: return smg::launch_bits<1>(probs, count, overlap, stream, nsm);
    default: return smg::launch_bits<2>(probs, count, overlap, stream, nsm);
  }
}

}  // namespace qg
