// Host packer: round-to-nearest group quantisation of fp32 weights into the
// at-rest format described in include/qgemm.h.
//
// The method stores its weights packed (stable-diffusion.rs README,
// introduction); this is the offline step that produces those bits.
// All decisions are taken in fp64 with ties to even (the 1-bit scale from an
// exact sum), and the fp64 -> fp16 rounding is written here from the IEEE 754
// binary16 definition.

#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "exact_abs_sum.h"
#include "qgemm.h"
#include "qgemm_internal.h"

namespace {

// fp64 -> binary16, round to nearest even, one rounding.
uint16_t f64_to_f16_rn(double x) {
  uint64_t u;
  std::memcpy(&u, &x, sizeof u);
  const uint16_t sign = static_cast<uint16_t>((u >> 48) & 0x8000u);
  const uint64_t mag = u & 0x7FFFFFFFFFFFFFFFull;
  const int exp_field = static_cast<int>(mag >> 52);
  if (exp_field == 0x7FF) {  // Inf or NaN
    const bool nan = (mag & ((1ull << 52) - 1)) != 0;
    return static_cast<uint16_t>(sign | 0x7C00u | (nan ? 0x200u : 0u));
  }
  if (exp_field == 0) return sign;  // zero or an fp64 subnormal: far below half the smallest fp16
  const int e = exp_field - 1023;                            // x = sig * 2^(e - 52)
  const uint64_t sig = (mag & ((1ull << 52) - 1)) | (1ull << 52);
  // ulp exponent of binary16 at this magnitude: 2^-24 in the subnormal range,
  // else 2^(e - 10)
  const int q = e < -14 ? -24 : e - 10;
  const int r = 52 + q - e;  // right shift that turns sig into units of 2^q
  uint64_t n;
  if (r >= 64) {
    n = 0;
  } else {
    n = sig >> r;
    const uint64_t rem = sig & ((1ull << r) - 1);
    const uint64_t half = 1ull << (r - 1);
    if (rem > half || (rem == half && (n & 1))) ++n;
  }
  uint32_t bits;
  if (q == -24) {
    bits = static_cast<uint32_t>(n);  // n == 1024 carries into the smallest normal
  } else {
    bits = (static_cast<uint32_t>(e + 15) << 10) + static_cast<uint32_t>(n - 1024);
  }
  if (bits >= 0x7C00u) bits = 0x7C00u;  // overflow to infinity
  return static_cast<uint16_t>(sign | bits);
}

double f16_to_f64(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 0x1F;
  const int m = h & 0x3FF;
  double v;
  if (e == 0) {
    v = std::ldexp(static_cast<double>(m), -24);
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = std::ldexp(static_cast<double>(m | 0x400), e - 25);
  }
  return sign ? -v : v;
}

bool is_f16_finite(uint16_t h) { return (h & 0x7C00u) != 0x7C00u; }

// Bit position of in-word offset j (see the layout in include/qgemm.h).
inline int code_shift(int bits, int j) {
  if (bits == 8) return 8 * j;
  return ((j & 1) ? 16 : 0) + bits * (j >> 1);
}

struct PackJob {
  const float* W;
  int N, K, bits, group;
  uint8_t* packed;
  uint16_t* scales;
  uint16_t* biases;
};

// Packs rows [r0, r1). Returns QGEMM_OK, or the first error found.
int pack_rows(const PackJob& jb, int r0, int r1) {
  const int K = jb.K, G = jb.group, bits = jb.bits;
  const int groups = K / G;
  const int per_word = 32 / bits;
  const size_t row_words = static_cast<size_t>(K) / per_word;
  std::vector<int> codes(G);
  for (int n = r0; n < r1; ++n) {
    const float* w = jb.W + static_cast<size_t>(n) * K;
    uint32_t* words = reinterpret_cast<uint32_t*>(jb.packed) + static_cast<size_t>(n) * row_words;
    for (size_t i = 0; i < row_words; ++i) words[i] = 0u;
    for (int g = 0; g < groups; ++g) {
      const float* wg = w + static_cast<size_t>(g) * G;
      for (int i = 0; i < G; ++i) {
        if (!std::isfinite(wg[i])) return QGEMM_ERR_NONFINITE;
      }
      const size_t sidx = static_cast<size_t>(g) * jb.N + n;  // group-major [K/group, N]
      if (bits == 1) {
        // Q1_0_g128: one sign bit per weight (1 = +1, for w >= 0 and -0),
        // s16 = fp16(mean |w|), the least-squares scale for fixed signs,
        // rounded once from the exact mean (G = 128 = 2^7)
        qg::ExactAbsSum sum;
        for (int i = 0; i < G; ++i) sum.add(wg[i]);
        const uint16_t s16 = sum.to_f16_rn(7);
        if (!is_f16_finite(s16)) return QGEMM_ERR_UNSUPPORTED;
        jb.scales[sidx] = s16;
        for (int i = 0; i < G; ++i) codes[i] = wg[i] >= 0.f ? 1 : 0;
      } else if (bits == 2) {
        double amax = 0.0;
        for (int i = 0; i < G; ++i) amax = std::max(amax, std::fabs(static_cast<double>(wg[i])));
        const uint16_t s16 = f64_to_f16_rn(amax);
        if (!is_f16_finite(s16)) return QGEMM_ERR_UNSUPPORTED;
        jb.scales[sidx] = s16;
        const double s = f16_to_f64(s16);
        for (int i = 0; i < G; ++i) {
          double t = 0.0;
          if (s != 0.0) t = std::min(1.0, std::max(-1.0, std::nearbyint(static_cast<double>(wg[i]) / s)));
          codes[i] = static_cast<int>(t);
        }
      } else {
        const double qmax = static_cast<double>((1 << bits) - 1);
        double lo = static_cast<double>(wg[0]), hi = lo;
        for (int i = 1; i < G; ++i) {
          lo = std::min(lo, static_cast<double>(wg[i]));
          hi = std::max(hi, static_cast<double>(wg[i]));
        }
        lo = lo + 0.0;  // a zero minimum is stored as +0
        hi = hi + 0.0;  // and a zero range gives a +0 scale, whichever zeros the group holds
        const uint16_t s16 = f64_to_f16_rn((hi - lo) / qmax);
        const uint16_t b16 = f64_to_f16_rn(lo);
        if (!is_f16_finite(s16) || !is_f16_finite(b16)) return QGEMM_ERR_UNSUPPORTED;
        jb.scales[sidx] = s16;
        jb.biases[sidx] = b16;
        const double s = f16_to_f64(s16), b = f16_to_f64(b16);
        for (int i = 0; i < G; ++i) {
          double q = 0.0;
          if (s != 0.0) q = std::min(qmax, std::max(0.0, std::nearbyint((static_cast<double>(wg[i]) - b) / s)));
          codes[i] = static_cast<int>(q);
        }
      }
      const int mask = (1 << bits) - 1;
      for (int i = 0; i < G; ++i) {
        const int k = g * G + i;
        const int word = k / per_word, j = k % per_word;
        words[word] |= static_cast<uint32_t>(codes[i] & mask) << code_shift(bits, j);
      }
    }
  }
  return QGEMM_OK;
}

int check_format(int32_t N, int32_t K, int32_t bits, int32_t group) {
  if (N <= 0 || K <= 0) return qg::fail(QGEMM_ERR_INVALID_ARG, "N and K must be positive (N=%d K=%d)", N, K);
  if (N > qg::kMaxDim || K > qg::kMaxDim)
    return qg::fail(QGEMM_ERR_UNSUPPORTED, "N=%d K=%d: at most %d each", N, K, qg::kMaxDim);
  const bool ok = (bits == 4 && group == 64) || (bits == 8 && group == 64) || (bits == 2 && group == 128) ||
                  (bits == 1 && group == 128);
  if (!ok) return qg::fail(QGEMM_ERR_UNSUPPORTED, "unsupported format bits=%d group=%d", bits, group);
  if (K % 128) return qg::fail(QGEMM_ERR_UNSUPPORTED, "K=%d is not a multiple of 128", K);
  return QGEMM_OK;
}

}  // namespace

extern "C" int qgemm_pack_sizes(int32_t N, int32_t K, int32_t bits, int32_t group, size_t* packed_bytes,
                                size_t* scales_bytes, size_t* biases_bytes) {
  if (!packed_bytes || !scales_bytes || !biases_bytes)
    return qg::fail(QGEMM_ERR_INVALID_ARG, "null size output");
  const int st = check_format(N, K, bits, group);
  if (st != QGEMM_OK) return st;
  *packed_bytes = static_cast<size_t>(N) * K * bits / 8;
  *scales_bytes = static_cast<size_t>(N) * (K / group) * 2;
  *biases_bytes = bits <= 2 ? 0 : *scales_bytes;
  return QGEMM_OK;
}

extern "C" int qgemm_pack(const float* W, int32_t N, int32_t K, int32_t bits, int32_t group, void* packed,
                          void* scales, void* biases) {
  const int st = check_format(N, K, bits, group);
  if (st != QGEMM_OK) return st;
  if (!W || !packed || !scales || (bits > 2 && !biases))
    return qg::fail(QGEMM_ERR_INVALID_ARG, "null buffer passed to qgemm_pack");
  if (reinterpret_cast<uintptr_t>(packed) % 4)
    return qg::fail(QGEMM_ERR_ALIGNMENT, "packed buffer must be 4-byte aligned");
  PackJob jb{W, N, K, bits, group, static_cast<uint8_t*>(packed), static_cast<uint16_t*>(scales),
             static_cast<uint16_t*>(biases)};
  const size_t work = static_cast<size_t>(N) * K;
  unsigned nthreads = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
  if (work < (1u << 20)) nthreads = 1;
  nthreads = std::min<unsigned>(nthreads, static_cast<unsigned>(N));
  std::vector<int> results(nthreads, QGEMM_OK);
  std::vector<std::thread> pool;
  const int chunk = (N + static_cast<int>(nthreads) - 1) / static_cast<int>(nthreads);
  for (unsigned t = 0; t < nthreads; ++t) {
    const int r0 = static_cast<int>(t) * chunk, r1 = std::min(N, r0 + chunk);
    if (r0 >= r1) continue;
    pool.emplace_back([&, t, r0, r1] { results[t] = pack_rows(jb, r0, r1); });
  }
  for (auto& th : pool) th.join();
  for (int r : results) {
    if (r == QGEMM_ERR_NONFINITE) return qg::fail(r, "W holds a NaN or infinite value");
    if (r == QGEMM_ERR_UNSUPPORTED) return qg::fail(r, "a group's scale or bias overflows fp16");
    if (r != QGEMM_OK) return qg::fail(r, "packing failed");
  }
  return QGEMM_OK;
}
