// Host check of the small-M kernel's shared-memory addressing (the functions
// in small_m_layout.cuh, compiled here for the host) against two definitions
// written out independently below:
//  * the packed layout: the 32-bit word at logical row offset `off` holds
//    codes (off / 4) * (32 / BITS) .. + 32 / BITS - 1 of the stage row, in
//    order; a quad thread's chunk must hold its quarter of the group, codes
//    gs G + c G/4 .. + G/4 - 1, and for every MMA step s the word and the four
//    codes the kernel picks (step_word, step_quad) must be the thread's codes
//    gs G + c G/4 + 4 s .. + 3;
//  * the TMA box: a [piece][row][U bytes] box whose linear byte index L is
//    swizzled by XOR-ing its 16-byte chunk bits (4 and up) with its bits from
//    7 up, U / 16 - 1 of them: L ^ (((L >> 7) & (U / 16 - 1)) << 4); a chunk
//    never straddles a 16-byte unit, so it stays contiguous under the swizzle.
// Prints the number of cases checked and of mismatches; exit status 1 on any.
#include <cstdio>

#include "small_m_layout.cuh"

using namespace qg::sm;

static long box_offset(long piece, long row, long byte, long R, long U) {
  const long L = (piece * R + row) * U + byte;
  return L ^ (((L >> 7) & (U / 16 - 1)) << 4);
}

template <int BITS, int NP>
static void check(long& cases, long& bad) {
  using F = Fmt<BITS>;
  using CH = Chunk<BITS>;
  constexpr int R = 16 * NP;
  constexpr int CODES_PER_WORD = 32 / BITS;
  for (int ush = 5; ush <= 7; ++ush) {
    const int U = 1 << ush;
    if (F::ROWB % U) continue;  // the launcher only picks pieces that divide a stage row
    for (int gs = 0; gs < GS; ++gs)
      for (int c = 0; c < 4; ++c) {
        const int off = chunk_offset<BITS>(gs, c);
        const int k0 = gs * F::G + c * (F::G / 4);  // the thread's first code in the stage row
        bool holds = off >= 0 && off + CH::BYTES <= F::ROWB && off % (CH::BYTES < 4 ? 4 : CH::BYTES) == 0 &&
                     off % 16 + CH::BYTES <= 16 && (off / 4) * CODES_PER_WORD == k0 &&
                     CH::WORDS * CODES_PER_WORD == F::G / 4;
        for (int s = 0; s < F::STEPS; ++s) {
          const int w = step_word<BITS>(s), quad = step_quad<BITS>(s);
          holds = holds && w < CH::WORDS && (off / 4 + w) * CODES_PER_WORD + 4 * quad == k0 + 4 * s &&
                  4 * quad + 3 < CODES_PER_WORD;
        }
        for (int q = 0; q < NP; ++q)
          for (int g = 0; g < 8; ++g)
            for (int h = 0; h < 2; ++h) {
              const int r = 16 * q + g + 8 * h;
              const long kernel = piece_offset<R>(off, ush, swizzle_key16(g, ush)) + (static_cast<long>(r) << ush);
              const long want = box_offset(off / U, r, off % U, R, U);
              ++cases;
              if (!holds || kernel != want || kernel + CH::BYTES > static_cast<long>(R) * F::ROWB) {
                if (bad < 8)
                  std::printf("mismatch: bits=%d NP=%d U=%d gs=%d c=%d row=%d: kernel %ld, box %ld%s\n", BITS, NP, U,
                              gs, c, r, kernel, want, holds ? "" : " (the chunk does not hold the codes)");
                ++bad;
              }
            }
      }
  }
}

template <int BITS>
static void check_bits(long& cases, long& bad) {
  check<BITS, 2>(cases, bad);
  check<BITS, 4>(cases, bad);
  check<BITS, 6>(cases, bad);
  check<BITS, 8>(cases, bad);
}

int main() {
  long cases = 0, bad = 0;
  check_bits<1>(cases, bad);
  check_bits<2>(cases, bad);
  check_bits<4>(cases, bad);
  check_bits<8>(cases, bad);
  std::printf("checked %ld mismatches %ld\n", cases, bad);
  return bad ? 1 : 0;
}
