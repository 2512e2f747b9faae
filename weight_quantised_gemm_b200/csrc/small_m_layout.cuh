// Stage layout of the small-M kernel's packed weights and the kernel's
// addressing into it: the format constants, the logical offset of the word a
// quad thread reads, and the physical offset after the TMA swizzle. Host and
// device, so that a host test can check the addressing against the layout's
// definition.
#pragma once

namespace qg {
namespace sm {

constexpr int GS = 8;                   // scale groups per stage

template <int BITS>
struct Fmt {
  static constexpr int G = BITS <= 2 ? 128 : 64;  // group size
  static constexpr int GBYTES = G * BITS / 8;     // packed bytes per row and group
  static constexpr int KS = GS * G;               // k per stage
  static constexpr int ROWB = GS * GBYTES;        // packed bytes per row and stage
  static constexpr int STEPS = G / 16;            // mma k-steps per group
};

// Logical byte offset, inside a stage row of packed codes, of the 32-bit word
// that holds quad thread c's 4 codes (k = 4c .. 4c+3) of step k of group gs:
//   1-bit:   one word per two 16-k steps (quad threads share it);
//   ternary: one word per 16-k step (quad threads share it);
//   4-bit:   two words per step, thread c reads word c / 2;
//   8-bit:   four words per step, thread c reads word c.
template <int BITS>
__host__ __device__ __forceinline__ int word_offset(int gs, int k, int c) {
  constexpr int GB = Fmt<BITS>::GBYTES;
  if constexpr (BITS == 1) return gs * GB + 4 * (k >> 1);  // one word per two steps
  else if constexpr (BITS == 2) return gs * GB + 4 * k;
  else if constexpr (BITS == 4) return gs * GB + 8 * k + 4 * (c >> 1);
  else return gs * GB + 16 * k + 4 * c;
}

// The box lands as [off / U][row][U bytes] (U = 2^ush), each U-byte row piece
// swizzled by the TMA: the 16-byte unit index of byte x of a plane is XORed
// with x's bits from 7 up (3, 2 or 1 of them). For row r that key is
// (r >> (7 - ush)) & (U / 16 - 1), which for rows 16q + g and 16q + g + 8 is
// the same function of g alone; so the physical offset of logical byte `off`
// of row r splits into a per-step part and a per-row part:
//   piece_offset(off) + (r << ush).
__host__ __device__ __forceinline__ int swizzle_key16(int g, int ush) {
  return ((g >> (7 - ush)) & ((1 << (ush - 4)) - 1)) << 4;
}
template <int R>
__host__ __device__ __forceinline__ int piece_offset(int off, int ush, int key16) {
  return ((off >> ush) * R << ush) + ((off & ((1 << ush) - 1)) ^ key16);
}

}  // namespace sm
}  // namespace qg
