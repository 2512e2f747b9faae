// Host check of the small-M launch planner (small_m_plan.h) against its
// definition written out independently here: every (rows per CTA, K slices)
// pair from the compiled sets whose grid fits the SMs, ordered by row-stages
// on the busiest CTA, then (32 tokens) 32-row CTAs after the others, then
// fewer slices, then generation order. Also pins the choices for the FLUX
// linears on 148 SMs. Prints the number of cases checked and of mismatches;
// exit status 1 on any.
#include <algorithm>
#include <cstdio>
#include <tuple>
#include <vector>

#include "small_m_plan.h"

using qg::sm::Plan;

struct Want {
  int np, ks, grid;
};

static std::vector<Want> definition(int pairs, int nst, int nsm, unsigned mask, bool demote) {
  struct Row {
    int np, ks, grid, rowstages, late, order;
  };
  std::vector<Row> rows;
  const int nps[] = {2, 4, 6, 8}, kss[] = {1, 2, 3, 4, 5, 6, 8};
  int order = 0;
  for (int np : nps)
    for (int ks : kss) {
      if (!((mask >> np) & 1u) || ks > nst) continue;
      const int blocks = (pairs + np - 1) / np;
      if (blocks * ks > nsm) continue;
      const int stages = (nst + ks - 1) / ks;  // the longest slice
      rows.push_back({np, ks, blocks * ks, np * stages, demote && np == 2, order++});
    }
  std::sort(rows.begin(), rows.end(), [](const Row& a, const Row& b) {
    return std::tie(a.rowstages, a.late, a.ks, a.order) < std::tie(b.rowstages, b.late, b.ks, b.order);
  });
  std::vector<Want> w;
  for (const Row& r : rows) w.push_back({r.np, r.ks, r.grid});
  return w;
}

static long cases = 0, bad = 0;

static std::vector<Want> planned(int pairs, int nst, int nsm, unsigned mask, bool demote) {
  Plan out[qg::sm::kMaxPlans];
  int n = -1;
  qg::sm::plan_candidates(pairs, nst, nsm, mask, demote, out, &n);
  std::vector<Want> w;
  for (int i = 0; i < n; ++i) w.push_back({out[i].np, out[i].ksplit, out[i].grid});
  return w;
}

static void against_definition(int pairs, int nst, int nsm, unsigned mask, bool demote) {
  const auto a = planned(pairs, nst, nsm, mask, demote), b = definition(pairs, nst, nsm, mask, demote);
  ++cases;
  bool same = a.size() == b.size();
  for (size_t i = 0; same && i < a.size(); ++i)
    same = a[i].np == b[i].np && a[i].ks == b[i].ks && a[i].grid == b[i].grid;
  if (!same && bad++ < 8)
    std::printf("mismatch: pairs=%d nst=%d nsm=%d mask=%x demote=%d\n", pairs, nst, nsm, mask, demote);
}

// the first plan whose clusters fit: clusters of 3 and of 6 never do on 148 SMs at these sizes
static Want first_fitting(const std::vector<Want>& w) {
  for (const Want& p : w)
    if (p.ks != 3 && p.ks != 6) return p;
  return {0, 0, 0};
}

static void pin(const char* what, int N, int K, int bits, int M, Want want) {
  const int G = bits <= 2 ? 128 : 64, KS = 8 * G;
  const int MT = M <= 8 ? 8 : M <= 16 ? 16 : 32;
  const unsigned mask = MT == 32 ? (1u << 2 | 1u << 4 | 1u << 8) : (1u << 2 | 1u << 4 | 1u << 6 | 1u << 8);
  const Want got = first_fitting(planned(N / 16, (K + KS - 1) / KS, 148, mask, MT == 32));
  ++cases;
  if (got.np != want.np || got.ks != want.ks || got.grid != want.grid) {
    if (bad++ < 8)
      std::printf("pin %s: planned %d pairs x %d slices (%d CTAs), want %d x %d (%d)\n", what, got.np, got.ks,
                  got.grid, want.np, want.ks, want.grid);
  }
}

int main() {
  const unsigned masks[] = {1u << 2 | 1u << 4 | 1u << 6 | 1u << 8, 1u << 2 | 1u << 4 | 1u << 8, 1u << 8};
  for (int pairs = 1; pairs <= 1200; pairs += (pairs < 64 ? 1 : 7))
    for (int nst = 1; nst <= 26; ++nst)
      for (int nsm : {132, 148})
        for (unsigned mask : masks)
          for (bool demote : {false, true}) against_definition(pairs, nst, nsm, mask, demote);
  // measured launch shapes of the FLUX linears (decode and 32-token)
  pin("ternary 12288x3072 M=1", 12288, 3072, 2, 1, {6, 1, 128});
  pin("8-bit 12288x3072 M=1", 12288, 3072, 8, 1, {6, 1, 128});
  pin("8-bit 3072x12288 M=1", 3072, 12288, 8, 1, {6, 4, 128});
  pin("4-bit 9216x3072 M=16", 9216, 3072, 4, 16, {4, 1, 144});
  pin("8-bit 3072x12288 M=32", 3072, 12288, 8, 32, {8, 5, 120});
  pin("ternary 3072x12288 M=32", 3072, 12288, 2, 32, {4, 2, 96});
  pin("8-bit 3072x3072 M=32", 3072, 3072, 8, 32, {4, 2, 96});
  pin("ternary 3072x3072 M=32", 3072, 3072, 2, 32, {2, 1, 96});
  pin("4-bit 9216x3072 M=32", 9216, 3072, 4, 32, {4, 1, 144});
  std::printf("checked %ld mismatches %ld\n", cases, bad);
  return bad ? 1 : 0;
}
