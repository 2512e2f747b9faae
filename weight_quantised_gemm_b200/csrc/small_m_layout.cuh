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

// Each quad thread c owns a contiguous quarter of every scale group: codes
// c G/4 .. (c + 1) G/4 - 1 of the group, CHUNK bytes of a packed row (1-bit
// 4, ternary and 4-bit 8, 8-bit 16), read with one shared-memory load per
// row and group. MMA step s of the group puts the thread's codes
// 4s .. 4s + 3 in the four k slots the fragment layout gives thread c: the
// tensor core sums all 16 slots of a step, so any assignment of the group's
// k to (step, thread, slot) works as long as the activations follow the same
// one (thread c's activation chunk is k = c G/4 .. + G/4 - 1 as well).
template <int BITS>
struct Chunk {
  static constexpr int BYTES = Fmt<BITS>::GBYTES / 4;  // packed bytes per thread, row and group
  static constexpr int WORDS = BYTES < 4 ? 1 : BYTES / 4;
  static constexpr int QUADS_PER_WORD = 8 / BITS;       // groups of four codes in a 32-bit word
};

// Logical byte offset, inside a stage row of packed codes, of quad thread
// c's chunk of scale group gs.
template <int BITS>
__host__ __device__ __forceinline__ int chunk_offset(int gs, int c) {
  return gs * Fmt<BITS>::GBYTES + c * Chunk<BITS>::BYTES;
}

// The word of a thread's chunk that holds its codes of step s, and which four
// codes of that word they are (codes 4 quad .. 4 quad + 3 of the word).
template <int BITS>
__host__ __device__ constexpr int step_word(int s) { return s / Chunk<BITS>::QUADS_PER_WORD; }
template <int BITS>
__host__ __device__ constexpr int step_quad(int s) { return s % Chunk<BITS>::QUADS_PER_WORD; }

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
