/*
 * qgemm — weight-only quantised GEMM for NVIDIA B200 (sm_100a).
 *
 * The operation (stable-diffusion.rs README, introduction): weights stay
 * packed in their quantised form in memory and are expanded to bf16 within the
 * GEMM kernel itself, tile by tile, so a layer whose dense weights would not
 * fit still runs.
 *
 *     out[M, N] = X[M, K] . dequant(W)[N, K]^T (+ bias[N])
 *
 * with X and out in bf16, W packed in one of four formats, and fp32
 * accumulation throughout (pictor README, numerics: accumulation stays in
 * fp32, without reduced-precision TF32 or fp16 multiply-accumulate).
 *
 * Formats (the pages give no bit layout, scale formula or rounding rule; this
 * library fixes the following):
 *   bits = 4 or 8, group = 64   group-wise affine, w ~ s * q + b, with an fp16
 *                               scale s and an fp16 bias b per 64 consecutive
 *                               k of a row, q in [0, 2^bits - 1]
 *                               (stable-diffusion.rs README, introduction: 8
 *                               bits for the linears whose output scales the
 *                               residual stream, 4 for the others);
 *   bits = 2, group = 128       ternary t in {-1, 0, +1} with one fp16 scale per
 *                               128 consecutive k (pictor README, "Extreme
 *                               quantization is first-class": TQ2_0_g128);
 *   bits = 1, group = 128       1-bit c in {-1, +1} with one fp16 scale per 128
 *                               consecutive k (the same README's Q1_0_g128,
 *                               named without a definition; this library's
 *                               reading: w ~ c * s, s = mean |w|).
 *
 * Bit layout (row-major over N, K contiguous, little-endian 32-bit words):
 *   8-bit   byte k holds q[k];
 *   4-bit   a word holds 8 consecutive k: in-word offset j = 2i in bits
 *           4i..4i+3, j = 2i+1 in bits 16+4i..19+4i;
 *   ternary a word holds 16 consecutive k: j = 2i in bits 2i..2i+1, j = 2i+1
 *           in bits 16+2i..17+2i; the code is t in 2-bit two's complement
 *           (00 = 0, 01 = +1, 11 = -1; 10 is invalid);
 *   1-bit   a word holds 32 consecutive k: j = 2i in bit i, j = 2i+1 in bit
 *           16+i; bit 1 is +1, bit 0 is -1;
 *   scales, biases: fp16 [K / group, N], group-major: the values of one
 *           group of k for all N rows are contiguous, so a tile's scales
 *           arrive in one TMA box with its codes.
 * Even and odd k sit in the two half-words so that one shift and one mask
 * move a neighbouring pair of codes into the two lanes of a bf16x2 register.
 *
 * Dequantised weight (what the kernels multiply; bit-exact contract):
 *   affine   wdeq = bf16_rn( fp32(s) * q + fp32(b) )  — one fp32 FMA, whose
 *            product is exact, then one round-to-nearest-even to bf16;
 *   ternary  wdeq = t * bf16_rn(fp32(s)), +0 for t = 0;
 *   1-bit    wdeq = c * bf16_rn(fp32(s)).
 *
 * Ownership: the caller allocates every buffer passed in; the library never
 * allocates, frees or keeps user memory. Device-side state is one static
 * status word per device (no allocation).
 * Errors: every call returns a qgemm_status; nothing throws across the ABI.
 * Asynchrony: device calls only enqueue work on the given stream (a
 * cudaStream_t passed as void*, NULL = the legacy default stream) and return
 * without synchronising, except qgemm_get_device_status.
 * Threads: calls are thread-safe; concurrent calls need distinct output
 * buffers.
 */
#ifndef QGEMM_H
#define QGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qgemm_status {
  QGEMM_OK = 0,
  QGEMM_ERR_INVALID_ARG = 1,     /* null pointer, negative or inconsistent size */
  QGEMM_ERR_UNSUPPORTED = 2,     /* format, shape or device this build does not handle */
  QGEMM_ERR_ALIGNMENT = 3,       /* a pointer is not 16-byte aligned */
  QGEMM_ERR_NONFINITE = 4,       /* a weight to pack is NaN or infinite */
  QGEMM_ERR_CUDA = 5,            /* a CUDA runtime or driver call failed */
  QGEMM_ERR_DEVICE_TIMEOUT = 6   /* a kernel's bounded wait ran out (see qgemm_get_device_status) */
} qgemm_status;

/* Kernel path selection for qgemm_ex (low byte of its `path` argument). */
enum {
  QGEMM_PATH_AUTO = 0,     /* pick per shape from the measured table */
  QGEMM_PATH_SMALL_M = 1,  /* memory-bound path: registers + mma.sync, M <= 64 (launches of
                              up to 32 token rows, back to back on the stream, past 32) */
  QGEMM_PATH_LARGE_M = 2   /* tensor-core path: TMA + dequant into TMEM + tcgen05 MMA */
};

/* Flags OR-ed into qgemm_ex's `path` argument.
 *
 * QGEMM_FLAG_OVERLAP_PREVIOUS: launch the kernel (either path) with
 * programmatic dependent launch. Its CTAs may start while the previous kernel
 * in the stream is still running (taking SMs as that kernel's CTAs leave) and
 * put the packed weights, scales and biases in flight at once (the large-M
 * path also dequantises them and runs its first stages' setup); they wait
 * for that kernel to complete (and its writes to be visible) before reading
 * X, bias, gate or residual and before writing out. Ask for it only when the
 * weight buffers are not written by the work that precedes the call in the
 * stream (static weights, as in inference). No counterpart in the method's
 * description: a launch-overlap option of this implementation. */
enum {
  QGEMM_FLAG_OVERLAP_PREVIOUS = 0x100,
  /* qgemm_grouped only: all problems in one persistent launch (below) */
  QGEMM_FLAG_GROUPED_ONE_LAUNCH = 0x200
};

/* A packed weight matrix resident in device memory. */
typedef struct qgemm_weights {
  int32_t N;             /* output features (rows of W) */
  int32_t K;             /* input features (columns of W) */
  int32_t bits;          /* 1 (1-bit), 2 (ternary), 4 or 8 */
  int32_t group;         /* 128 for 1-bit and ternary, 64 for 4- and 8-bit */
  const void* packed;    /* uint8 [N, K * bits / 8], 16-byte aligned */
  const void* scales;    /* fp16 [K / group, N], 16-byte aligned */
  const void* biases;    /* fp16 [K / group, N], 16-byte aligned; NULL for 1-bit and ternary */
} qgemm_weights;

/*
 * Byte sizes of the three packed arrays for an [N, K] weight.
 * Defined by the layout above. biases_bytes is 0 for 1-bit and ternary.
 * Returns INVALID_ARG for non-positive sizes or null outputs, UNSUPPORTED
 * for a (bits, group) pair other than (4,64), (8,64), (2,128), (1,128), for
 * K not a multiple of 128, or for N or K above 2^30.
 */
int qgemm_pack_sizes(int32_t N, int32_t K, int32_t bits, int32_t group,
                     size_t* packed_bytes, size_t* scales_bytes, size_t* biases_bytes);

/*
 * Round-to-nearest group quantisation of a host fp32 matrix W [N, K]
 * (row-major) into caller-allocated host buffers sized by qgemm_pack_sizes.
 * Arithmetic is fp64, ties to even:
 *   affine:  s = fp16(fl64((max - min) / (2^bits - 1))), b = fp16(min),
 *            q = clamp(rint((w - b) / s), 0, 2^bits - 1), q = 0 where s == 0;
 *   ternary: s = fp16(max |w|), t = clamp(rint(w / s), -1, 1), t = 0 where s == 0;
 *   1-bit:   s = fp16(mean |w|), rounded once from the exact mean of the
 *            group's magnitudes; c = +1 where w >= 0 (and for -0), else -1.
 * The weights stay packed at rest (stable-diffusion.rs README, introduction).
 * Returns NONFINITE if W holds NaN/Inf, UNSUPPORTED if a scale or bias
 * overflows fp16, plus the errors of qgemm_pack_sizes. biases may be NULL for
 * 1-bit and ternary. Host-only; no device is touched.
 */
int qgemm_pack(const float* W, int32_t N, int32_t K, int32_t bits, int32_t group,
               void* packed, void* scales, void* biases);

/*
 * qgemm_pack on the GPU: the same packing of a device fp32 matrix W [N, K]
 * (row-major) into caller-allocated device buffers, bit-identical to
 * qgemm_pack's output (the same steps in the same order). Enqueued on
 * `stream`; a non-finite weight or an fp16 overflow is reported later by
 * qgemm_get_device_status as QGEMM_ERR_NONFINITE or QGEMM_ERR_UNSUPPORTED.
 * All pointers 16-byte aligned; biases may be NULL for 1-bit and ternary.
 * Argument errors are those of qgemm_pack_sizes, plus INVALID_ARG / ALIGNMENT.
 */
int qgemm_pack_device(const void* W, int32_t N, int32_t K, int32_t bits, int32_t group,
                      void* packed, void* scales, void* biases, void* stream);

/*
 * The at-rest file of a packed weight (host buffers): magic "QGEMMW01", then
 * int32 N, K, bits, group and uint64 packed_bytes, scales_bytes,
 * biases_bytes (little-endian), then the three arrays in that order.
 * qgemm_save writes one; qgemm_load_header reads its shape and format (check
 * them, size buffers with qgemm_pack_sizes); qgemm_load fills caller-
 * allocated host buffers (biases may be NULL for 1-bit and ternary). Both
 * readers check the whole file before returning OK or copying anything: a
 * bad magic, array sizes that do not match the format, a file length other
 * than the header plus the three arrays, or an I/O failure return
 * QGEMM_ERR_INVALID_ARG (format errors: those of qgemm_pack_sizes). No
 * counterpart as an interface in the pages.
 */
int qgemm_save(const char* path, int32_t N, int32_t K, int32_t bits, int32_t group,
               const void* packed, const void* scales, const void* biases);
int qgemm_load_header(const char* path, int32_t* N, int32_t* K, int32_t* bits, int32_t* group);
int qgemm_load(const char* path, void* packed, void* scales, void* biases);

/*
 * out = X . dequant(W)^T (+ bias), enqueued on `stream`.
 *   X     device bf16 [M, K] row-major, 16-byte aligned
 *   M     tokens (rows of X); M = 0 is a no-op returning OK
 *   W     device-resident packed weights (struct itself is host memory)
 *   out   device bf16 [M, N] row-major, 16-byte aligned
 *   bias  device bf16 [N] or NULL
 * Requires K % 128 == 0, N % 16 == 0 and M, N, K <= 2^30, the same limit as
 * qgemm_pack_sizes (larger: UNSUPPORTED) (1-bit weights with K % 256 != 0
 * always take the large-M path). The path (small-M register path or
 * large-M tensor-core path) is chosen per (bits, M, N, K) from a measured
 * table; the environment variable QGEMM_PATH=small|large overrides it for
 * every shape the named path can take (QGEMM_PATH=small leaves M > 16, and
 * 1-bit weights with K % 256 != 0, to the table). qgemm_select_path reports
 * the same choice. QGEMM_SMALL_TC=1 runs the small-M path's launches without
 * QGEMM_FLAG_OVERLAP_PREVIOUS on its tcgen05 kernel (weights decoded into
 * tensor memory, N = 16 tokens per MMA) instead of the warp-level mma.sync
 * kernel; it is slower on B200 at every measured shape and off by default.
 * Returns after enqueueing; a device-side failure (a bounded wait that ran
 * out) is reported later by qgemm_get_device_status.
 */
int qgemm(const void* X, int32_t M, const qgemm_weights* W, void* out,
          const void* bias, void* stream);

/* As qgemm, with an explicit QGEMM_PATH_* choice (AUTO defers to the table and
 * the QGEMM_PATH variable), optionally OR-ed with QGEMM_FLAG_* bits. Unknown
 * path values or flag bits return QGEMM_ERR_INVALID_ARG. */
int qgemm_ex(const void* X, int32_t M, const qgemm_weights* W, void* out,
             const void* bias, int32_t path, void* stream);

/* Fused epilogues for qgemm_fused: the elementwise steps on either side of a
 * FLUX block's linears. The pages (stable-diffusion.rs README, introduction)
 * single out the linears whose output scales the residual stream but give no
 * formulas; these are FLUX's: the MLP up projection's tanh GELU, and a residual-writing
 * layer's gated update of the residual stream. v = acc + bias in fp32; the
 * result is rounded to bf16 once. */
enum {
  QGEMM_EPI_NONE = 0,          /* out = bf16(v) */
  QGEMM_EPI_GELU_TANH = 1,     /* out = bf16(0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))) */
  QGEMM_EPI_RESIDUAL_GATE = 2  /* out = bf16(residual + gate[n] * v) */
};

typedef struct qgemm_epilogue {
  int32_t op;            /* QGEMM_EPI_* */
  const void* residual;  /* QGEMM_EPI_RESIDUAL_GATE: device bf16 [M, N], 16-byte aligned; may equal out
                            (in-place update of the residual stream) */
  const void* gate;      /* QGEMM_EPI_RESIDUAL_GATE: device bf16 [N], one gate per output feature */
} qgemm_epilogue;

/* As qgemm_ex, with a fused epilogue (NULL or QGEMM_EPI_NONE: plain qgemm_ex).
 * Errors: unknown op, or a missing or misaligned residual or gate, return
 * QGEMM_ERR_INVALID_ARG / QGEMM_ERR_ALIGNMENT before anything is enqueued.
 * No counterpart as an interface in the pages. */
int qgemm_fused(const void* X, int32_t M, const qgemm_weights* W, void* out,
                const void* bias, const qgemm_epilogue* epi, int32_t path, void* stream);

/* One GEMV of a grouped call: out = X . dequant(W)^T (+ bias), as qgemm. */
typedef struct qgemm_problem {
  const void* X;         /* device bf16 [M, K], 16-byte aligned */
  int32_t M;             /* tokens, 0 to 16 (0: the problem is skipped) */
  qgemm_weights W;       /* device-resident packed weights */
  void* out;             /* device bf16 [M, N], 16-byte aligned */
  const void* bias;      /* device bf16 [N] or NULL */
} qgemm_problem;

/*
 * Several independent small-M GEMVs (M <= 16 each), each computing what qgemm
 * computes for it, on `stream`. At decode-sized M a GEMV is a read of its
 * packed weights, and a single read of 10-40 MB is bound by the launch and
 * first-byte latency rather than by bandwidth (pictor README, "Extreme
 * quantization is first-class": GEMV paths built for sub-byte weights). By
 * default the problems run as consecutive launches of the small-M kernel,
 * each after the first launched with programmatic dependent launch, so that
 * its weight stream starts while the one before finishes (the problems are
 * independent, so none waits for another's data); with
 * QGEMM_FLAG_GROUPED_ONE_LAUNCH one persistent launch streams all the
 * problems' weights back to back instead. The consecutive launches measured
 * faster on every block of the FLUX decode linears (4-bit QKV + MLP up at
 * M = 1: 17.5 us against 24.4). Requires 1 to 16 problems whose weights share
 * one format (bits), each a shape the small-M path takes (1-bit: K % 256 ==
 * 0) and, for the one-launch form, at most 4096 x 32 rows per problem and
 * 4096 blocks of 32 rows in all (else UNSUPPORTED). No output may overlap
 * another problem's X, out or bias.
 * flags: QGEMM_FLAG_OVERLAP_PREVIOUS (for the first launch, as for qgemm_ex)
 * and QGEMM_FLAG_GROUPED_ONE_LAUNCH, or 0. Argument errors
 * are those of qgemm_ex, checked for every problem before anything is
 * enqueued. No counterpart as an interface in the pages.
 */
int qgemm_grouped(const qgemm_problem* problems, int32_t count, int32_t flags, void* stream);

/* The path qgemm would take for this shape: QGEMM_PATH_SMALL_M or
 * QGEMM_PATH_LARGE_M, or a negative qgemm_status for an invalid shape. */
int qgemm_select_path(int32_t M, int32_t N, int32_t K, int32_t bits);

/*
 * Debug entry point for the bit-exact gate: writes the dequantised weights
 * W[n0 : n0+rows, k0 : k0+cols] as bf16 [rows, cols] (row-major, `out` a
 * 16-byte aligned device buffer), using the same device dequantisation
 * routine the large-M kernel applies to each shared-memory tile.
 * Requires n0, k0 >= 0, n0 + rows <= N, k0 + cols <= K, k0 % 8 == 0 and
 * cols % 8 == 0. Enqueued on `stream`.
 */
int qgemm_dequant_tile(const qgemm_weights* W, int32_t n0, int32_t k0, int32_t rows,
                       int32_t cols, void* out, void* stream);

/*
 * Debug entry point for measurement: the small-M kernel exactly as qgemm would
 * launch it for (M, W) (same grid, same thread-block clusters, same stage ring
 * and TMA boxes, QGEMM_FLAG_OVERLAP_PREVIOUS honoured), streaming the packed
 * weights, scales and biases (and, where the kernel stages them, the
 * activation rows of X) through its ring while computing and writing nothing.
 * Its time is the floor of the weight stream itself for this shape: launch,
 * first-byte latency and bandwidth, without the arithmetic. X: device bf16
 * [M, K], 16-byte aligned. Requires a shape the small-M path takes (M <= 64;
 * 1-bit weights with K % 256 == 0), else UNSUPPORTED. No counterpart in the
 * pages: an instrument of this implementation.
 */
int qgemm_debug_stream(const void* X, int32_t M, const qgemm_weights* W, int32_t flags, void* stream);

/*
 * Reads and clears the current device's status word (all conditions
 * recorded since the last read) in one atomic step enqueued on `stream`,
 * after the work already there, then synchronises `stream`. A condition a
 * kernel on another stream records meanwhile is never lost: this call or the
 * next one reports it. Returns, first match:
 *   QGEMM_ERR_CUDA          the stream reports a CUDA error;
 *   QGEMM_ERR_NONFINITE     qgemm_pack_device met a NaN or infinite weight;
 *   QGEMM_ERR_UNSUPPORTED   qgemm_pack_device: a scale or bias overflows fp16;
 *   QGEMM_ERR_CUDA          a kernel found its shared memory misaligned and
 *                           returned without computing;
 *   QGEMM_ERR_DEVICE_TIMEOUT a kernel gave up a bounded wait;
 *   QGEMM_OK                none of these.
 * qgemm_last_error() then names the condition and the raw status word.
 */
int qgemm_get_device_status(void* stream);

/* Upper bound, in nanoseconds, on any single wait inside a kernel (default
 * 2e9, also settable with QGEMM_WAIT_LIMIT_NS). 0 restores the default. */
int qgemm_set_wait_limit_ns(uint64_t limit_ns);

/* Test hook for the timeout path: launches one block that waits on a
 * barrier nothing will complete, giving up after `limit_ns`; the device
 * status word then reads QGEMM_ERR_DEVICE_TIMEOUT. Faults and traps nothing. */
int qgemm_debug_wait_timeout(uint64_t limit_ns, void* stream);

/* Static description of a status code. */
const char* qgemm_status_str(int status);

/* Detail of the calling thread's last failed call ("" if none). */
const char* qgemm_last_error(void);

/* Library version string. */
const char* qgemm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H */
