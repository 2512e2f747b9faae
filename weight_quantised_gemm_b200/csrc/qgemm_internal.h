// Internal interface between the host ABI layer and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "qgemm.h"

namespace qg {

// One validated GEMM problem, all pointers device pointers.
struct Problem {
  const void* X;         // bf16 [M, K]
  int M, N, K;
  int bits, group;
  const uint8_t* packed;
  const uint16_t* scales;  // fp16 bits [K/group, N] (group-major)
  const uint16_t* biases;  // fp16 bits [K/group, N] or nullptr (ternary)
  void* out;             // bf16 [M, N]
  const uint16_t* bias;  // bf16 bits [N] or nullptr
  cudaStream_t stream;
  bool overlap;          // launch with programmatic dependent launch (QGEMM_FLAG_OVERLAP_PREVIOUS)
  int epi;               // QGEMM_EPI_*
  const uint16_t* residual;  // bf16 bits [M, N] (QGEMM_EPI_RESIDUAL_GATE), may equal out
  const uint16_t* gate;      // bf16 bits [N] (QGEMM_EPI_RESIDUAL_GATE)
  bool floor_only = false;   // small-M: stream the weights through the ring, compute and write nothing
};

// Records a detail message for qgemm_last_error and returns `code`.
int fail(int code, const char* fmt, ...);
// Maps a CUDA error to QGEMM_ERR_CUDA (with its name recorded), or QGEMM_OK.
int cuda_check(cudaError_t e, const char* what);

uint64_t wait_limit_ns();
// The large-M kernel's CTA-pair form: -1 = the library's choice (the
// one-CTA form), 0 = never, 1 = always (QGEMM_LARGE_PAIR=0|1, read once).
int large_pair_mode();
// The small-M kernel family: -1 = the library's choice, 0 = the mma.sync
// kernel, 1 = the tcgen05 kernel (QGEMM_SMALL_TC=0|1, read once).
int small_tc_mode();
// Device address of the current device's status word (cached per device).
int status_word(unsigned int** ptr);
int sm_count(int* n);
// Raises the kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (device, kernel).
int smem_opt_in(const void* func, int bytes, const char* what);

// 2-D TMA descriptor: `inner` x `outer` elements, rows `row_stride_bytes`
// apart, box `box_inner` x `box_outer`. Reads outside the tensor return zeros
// and stores outside it are dropped.
int make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz,
                       const char* what);

// 3-D TMA descriptor: dims[0] x dims[1] x dims[2] elements with byte strides
// strides_bytes[0] (dimension 1) and strides_bytes[1] (dimension 2), in any
// order of size; box box[0] x box[1] x box[2].
int make_tensor_map_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, const uint64_t dims[3],
                       const uint64_t strides_bytes[2], const uint32_t box[3], CUtensorMapSwizzle swz,
                       const char* what);

// Kernel launchers (one per kernel family). Each enqueues on p.stream.
int launch_small_m(const Problem& p);
// The tcgen05 small-M kernel (M <= 16, no launch overlap).
int launch_small_m_tc(const Problem& p);
// Several small-M problems of one format in one launch (qgemm_grouped).
int launch_small_m_grouped(const Problem* probs, int count, bool overlap, cudaStream_t stream);
int launch_large_m(const Problem& p);
int launch_dequant_tile(const Problem& p, int n0, int k0, int rows, int cols);
int launch_debug_wait(uint64_t limit_ns, cudaStream_t stream);
int launch_pack_device(const float* W, int N, int K, int bits, void* packed, uint16_t* scales, uint16_t* biases,
                       cudaStream_t stream);

// Device status word values (0 = fine).
// Largest M, N or K the library accepts (2^30): keeps every launcher's int
// arithmetic (rounded-up tile and stage counts) inside int32.
constexpr int32_t kMaxDim = 1 << 30;

// Largest M of one small-M (register) kernel launch; its grouped form and its
// tcgen05 variant take at most 16. The small-M path as a whole takes up to
// kSmallPathMaxM: larger M runs as launches of kSmallMaxM tokens back to back.
constexpr int kSmallMaxM = 32;
constexpr int kSmallPathMaxM = 64;
constexpr int kSmallGroupedMaxM = 16;

// Grouped small-M launches: problems per launch, CTAs, and 32-row work items.
constexpr int kGroupedMaxProblems = 16;
constexpr int kGroupedMaxCtas = 256;
constexpr int kGroupedMaxItems = 4096;

constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusLayout = 2u;  // dynamic shared memory not aligned as the kernel requires
constexpr unsigned kStatusPackNonfinite = 4u;  // qgemm_pack_device met a NaN or an infinity
constexpr unsigned kStatusPackOverflow = 8u;   // qgemm_pack_device: a scale or bias overflows fp16

}  // namespace qg
