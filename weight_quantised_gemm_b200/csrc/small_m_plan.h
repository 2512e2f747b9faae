// Host-side choice of the small-M kernel's launch shape: rows per CTA and K
// slices per row block. Plain C++ (no CUDA), so the host tests can check it.
#pragma once

namespace qg {
namespace sm {

// Rows per CTA (16 NP, NP from the compiled set) and K slices per row block
// (a cluster of `ksplit` CTAs): the choice that puts the fewest row-stages of
// packed weights on the busiest CTA with the whole grid resident at once, the
// fewer slices on a tie. With 32 tokens a tie goes against CTAs of 32 rows
// first: a stage's activations are two (8-bit) to eight (ternary) times such
// a CTA's packed weights, and twice as many rows per CTA halve the
// activation bytes each SM reads (3072 x 12288 ternary at M = 32: 19.0 us
// against 25.4; 3072 x 3072 8-bit: 11.9 against 14.0). Narrow N with long K
// (MLP down, the out projection) needs the slices: 3072 rows make only 96
// CTAs of 32 rows, while 48 row blocks of 64 rows x 3 slices use 144 SMs
// with a third less per CTA.
struct Plan {
  int np, ksplit, grid;
};

constexpr int kMaxPlans = 28;  // 4 row choices x 7 slice counts

// All plans for `pairs` 16-row pairs and `nst` K stages whose grid fits `nsm`
// CTAs, cheapest first, into out[0 .. *count) (out holds kMaxPlans).
// np_mask: bit np set for each rows-per-CTA choice the caller compiled;
// demote_np2: 32-row plans lose ties on row-stages.
inline void plan_candidates(int pairs, int nst, int nsm, unsigned np_mask, bool demote_np2, Plan* out, int* count) {
  static constexpr int kNP[4] = {2, 4, 6, 8};
  static constexpr int kS[7] = {1, 2, 3, 4, 5, 6, 8};
  int n = 0;
  for (int np : kNP)
    for (int S : kS) {
      if (!(np_mask >> np & 1u)) continue;
      if (S > nst) continue;
      const int grid = (pairs + np - 1) / np * S;
      if (grid > nsm) continue;
      out[n++] = Plan{np, S, grid};
    }
  // cheapest first: row-stages on the busiest CTA, then (demote_np2) more
  // than 32 rows, then fewer slices
  auto cost = [&](const Plan& p) { return p.np * ((nst + p.ksplit - 1) / p.ksplit); };
  auto np2 = [&](const Plan& p) { return demote_np2 && p.np == 2 ? 1 : 0; };
  for (int i = 1; i < n; ++i)
    for (int j = i; j > 0; --j) {
      const Plan a = out[j - 1], b = out[j];
      if (cost(b) < cost(a) ||
          (cost(b) == cost(a) && (np2(b) < np2(a) || (np2(b) == np2(a) && b.ksplit < a.ksplit)))) {
        out[j - 1] = b;
        out[j] = a;
      }
    }
  *count = n;
}

}  // namespace sm
}  // namespace qg
