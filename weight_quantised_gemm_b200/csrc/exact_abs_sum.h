// The 1-bit format's scale, fp16(mean |w|) over a group of 128 fp32
// weights, rounded once from the exact mean (round to nearest, ties to
// even). An fp64 running sum is not exact when a group spans many binades,
// and its rounding order could then move the stored scale to a neighbouring
// fp16 value; this accumulator holds the sum exactly instead.
//
// Every finite fp32 magnitude is an integer multiple of 2^-149 below 2^128,
// so the sum of up to 128 of them is an integer below 2^284 in units of
// 2^-149: five 64-bit limbs hold it with no rounding. The packers on the
// host and on the device both use this header.
#pragma once

#include <cstdint>
#include <cstring>

#ifdef __CUDACC__
#define QG_HD __host__ __device__ __forceinline__
#else
#define QG_HD inline
#endif

namespace qg {

struct ExactAbsSum {
  static constexpr int kLimbs = 5;
  uint64_t limb[kLimbs] = {0, 0, 0, 0, 0};

  // Adds |f| (f finite).
  QG_HD void add(float f) {
#ifdef __CUDA_ARCH__
    uint32_t u = __float_as_uint(f);
#else
    uint32_t u;
    std::memcpy(&u, &f, sizeof u);
#endif
    u &= 0x7FFFFFFFu;
    const uint32_t be = u >> 23;
    uint64_t m = u & 0x7FFFFFu;
    int sh = 0;  // |f| = m * 2^(sh - 149)
    if (be) {
      m |= 0x800000u;
      sh = static_cast<int>(be) - 1;
    }
    const int L = sh >> 6, o = sh & 63;
    add_at(L, m << o);
    if (o) add_at(L + 1, m >> (64 - o));
  }

  QG_HD void add_at(int L, uint64_t v) {
    for (int i = L; i < kLimbs && v; ++i) {
      const uint64_t s = limb[i] + v;
      v = s < v ? 1u : 0u;  // carry out
      limb[i] = s;
    }
  }

  QG_HD int top_bit() const {  // index of the highest set bit, -1 for zero
    for (int i = kLimbs - 1; i >= 0; --i)
      if (limb[i])
        for (int b = 63; b >= 0; --b)
          if ((limb[i] >> b) & 1u) return 64 * i + b;
    return -1;
  }

  QG_HD uint32_t bit(int pos) const { return static_cast<uint32_t>((limb[pos >> 6] >> (pos & 63)) & 1u); }

  QG_HD bool any_below(int pos) const {  // any set bit at an index below pos
    for (int i = 0; i < kLimbs; ++i) {
      if (64 * (i + 1) <= pos) {
        if (limb[i]) return true;
      } else {
        const int r = pos - 64 * i;
        if (r > 0 && (limb[i] & ((1ull << r) - 1))) return true;
        break;
      }
    }
    return false;
  }

  // binary16 bits of sum * 2^-shift (shift = log2 of the group size),
  // rounded once to nearest, ties to even; overflow gives +infinity.
  QG_HD uint16_t to_f16_rn(int shift) const {
    const int h = top_bit();
    if (h < 0) return 0;
    const int base = 149 + shift;  // value = A * 2^-base
    const int E = h - base;        // value in [2^E, 2^(E+1))
    if (E > 15) return 0x7C00u;
    const int q = E - 10 > -24 ? E - 10 : -24;  // exponent of the fp16 ulp at this magnitude
    const int r = q + base;                      // A >> r is the value in ulps
    uint32_t n = 0;
    for (int b = 11; b >= 0; --b) n = (n << 1) | (r + b <= h ? bit(r + b) : 0u);
    const uint32_t half = bit(r - 1);
    if (half && (any_below(r - 1) || (n & 1u))) ++n;
    uint32_t bits = q == -24 ? n : (static_cast<uint32_t>(E + 15) << 10) + (n - 1024u);
    if (bits >= 0x7C00u) bits = 0x7C00u;
    return static_cast<uint16_t>(bits);
  }
};

}  // namespace qg

#undef QG_HD
