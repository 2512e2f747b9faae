// The C ABI: argument validation, path choice and dispatch to the kernels.

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "qgemm.h"
#include "qgemm_internal.h"

namespace qg {

namespace {
thread_local std::string t_last_error;
std::atomic<uint64_t> g_wait_limit_ns{0};  // 0 = not yet resolved; read by every launch, set by any thread
std::once_flag g_env_once;
int g_env_path = QGEMM_PATH_AUTO;
int g_env_pair = -1;
int g_env_small_tc = -1;

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

void read_env() {
  if (const char* p = std::getenv("QGEMM_PATH")) {
    if (!std::strcmp(p, "small")) g_env_path = QGEMM_PATH_SMALL_M;
    else if (!std::strcmp(p, "large")) g_env_path = QGEMM_PATH_LARGE_M;
  }
  if (const char* pr = std::getenv("QGEMM_LARGE_PAIR")) {
    if (!std::strcmp(pr, "0")) g_env_pair = 0;
    else if (!std::strcmp(pr, "1")) g_env_pair = 1;
  }
  if (const char* tc = std::getenv("QGEMM_SMALL_TC")) {
    if (!std::strcmp(tc, "0")) g_env_small_tc = 0;
    else if (!std::strcmp(tc, "1")) g_env_small_tc = 1;
  }
  if (const char* w = std::getenv("QGEMM_WAIT_LIMIT_NS")) {
    const unsigned long long v = std::strtoull(w, nullptr, 10);
    uint64_t unset = 0;
    if (v > 0) g_wait_limit_ns.compare_exchange_strong(unset, v);
  }
}

// Largest M served by the small-M path, per format and shape class, from
// timing both paths at M = 1..64 on B200 (the bench's path crossover sweep):
// below the crossover the weights' bytes set the time and the register path
// streams them faster than the tile pipeline fills.
#include "path_table.inc"

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_weights(const qgemm_weights* W) {
  if (!W) return fail(QGEMM_ERR_INVALID_ARG, "null weights descriptor");
  if (W->N <= 0 || W->K <= 0) return fail(QGEMM_ERR_INVALID_ARG, "N=%d K=%d must be positive", W->N, W->K);
  if (W->N > kMaxDim || W->K > kMaxDim)
    return fail(QGEMM_ERR_UNSUPPORTED, "N=%d K=%d: at most %d each", W->N, W->K, kMaxDim);
  const bool fmt_ok = (W->bits == 4 && W->group == 64) || (W->bits == 8 && W->group == 64) ||
                      (W->bits == 2 && W->group == 128) || (W->bits == 1 && W->group == 128);
  if (!fmt_ok) return fail(QGEMM_ERR_UNSUPPORTED, "unsupported format bits=%d group=%d", W->bits, W->group);
  if (W->K % 128) return fail(QGEMM_ERR_UNSUPPORTED, "K=%d is not a multiple of 128", W->K);
  if (W->N % 16) return fail(QGEMM_ERR_UNSUPPORTED, "N=%d is not a multiple of 16", W->N);
  if (!W->packed || !W->scales || (W->bits > 2 && !W->biases))
    return fail(QGEMM_ERR_INVALID_ARG, "null packed/scales/biases pointer");
  if (!aligned16(W->packed) || !aligned16(W->scales) || (W->biases && !aligned16(W->biases)))
    return fail(QGEMM_ERR_ALIGNMENT, "packed weights, scales and biases must be 16-byte aligned");
  return QGEMM_OK;
}

}  // namespace

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return QGEMM_OK;
  return fail(QGEMM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

uint64_t wait_limit_ns() {
  std::call_once(g_env_once, read_env);
  const uint64_t v = g_wait_limit_ns.load();
  return v ? v : kDefaultWaitLimitNs;
}

// Whether the small-M path can take this shape at all: M <= 64 (launches of
// up to 32 token rows), and 1-bit
// rows streamed in pieces of at least 32 bytes (K % 256 == 0).
bool small_path_takes(int M, int K, int bits) { return M <= kSmallPathMaxM && !(bits == 1 && K % 256); }

// The small-M path for any M it takes: one launch up to kSmallMaxM tokens,
// else launches of kSmallMaxM token rows back to back on the caller's stream
// (each streams all the weights; they write disjoint output rows). Launches
// after the first overlap their weight stream with the previous one's last
// stages (programmatic dependent launch): each reads its activations and
// writes its rows only once the launch before it has finished, which in turn
// ran after whatever preceded the call.
int launch_small_rows(const Problem& p) {
  if (p.M <= kSmallMaxM)
    return small_tc_mode() == 1 && !p.overlap && !p.floor_only && p.M <= kSmallGroupedMaxM ? launch_small_m_tc(p)
                                                                                          : launch_small_m(p);
  for (int m0 = 0; m0 < p.M; m0 += kSmallMaxM) {
    Problem q = p;
    q.M = p.M - m0 < kSmallMaxM ? p.M - m0 : kSmallMaxM;
    q.X = static_cast<const uint16_t*>(p.X) + static_cast<size_t>(m0) * p.K;
    if (p.out) q.out = static_cast<uint16_t*>(p.out) + static_cast<size_t>(m0) * p.N;
    if (p.residual) q.residual = p.residual + static_cast<size_t>(m0) * p.N;
    if (m0 > 0) q.overlap = true;
    const int st = launch_small_m(q);
    if (st != QGEMM_OK) return st;
  }
  return QGEMM_OK;
}

int large_pair_mode() {
  std::call_once(g_env_once, read_env);
  return g_env_pair;
}

int small_tc_mode() {
  std::call_once(g_env_once, read_env);
  return g_env_small_tc;
}

int select_path(int M, int N, int K, int bits) {
  if (!small_path_takes(M, K, bits)) return QGEMM_PATH_LARGE_M;
  for (const PathEntry& e : kPathTable)
    if (e.bits == bits && N <= e.n_max && K >= e.k_min && K <= e.k_max)
      return M <= e.small_max ? QGEMM_PATH_SMALL_M : QGEMM_PATH_LARGE_M;
  return QGEMM_PATH_LARGE_M;
}

// The path of a QGEMM_PATH_AUTO call: the QGEMM_PATH variable's choice where
// that path can take the shape, else the measured table.
int auto_path(int M, int N, int K, int bits) {
  std::call_once(g_env_once, read_env);
  if (g_env_path == QGEMM_PATH_LARGE_M) return QGEMM_PATH_LARGE_M;
  if (g_env_path == QGEMM_PATH_SMALL_M && small_path_takes(M, K, bits)) return QGEMM_PATH_SMALL_M;
  return select_path(M, N, K, bits);
}

}  // namespace qg

using namespace qg;

extern "C" int qgemm_fused(const void* X, int32_t M, const qgemm_weights* W, void* out, const void* bias,
                           const qgemm_epilogue* epi, int32_t path, void* stream) {
  int st = validate_weights(W);
  if (st != QGEMM_OK) return st;
  if (M < 0) return fail(QGEMM_ERR_INVALID_ARG, "M=%d is negative", M);
  if (M > kMaxDim) return fail(QGEMM_ERR_UNSUPPORTED, "M=%d: at most %d", M, kMaxDim);
  const int32_t flags = path & ~0xFF;
  path &= 0xFF;
  if (path < QGEMM_PATH_AUTO || path > QGEMM_PATH_LARGE_M) return fail(QGEMM_ERR_INVALID_ARG, "bad path %d", path);
  if (flags & ~QGEMM_FLAG_OVERLAP_PREVIOUS) return fail(QGEMM_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  const int op = epi ? epi->op : QGEMM_EPI_NONE;
  if (op < QGEMM_EPI_NONE || op > QGEMM_EPI_RESIDUAL_GATE) return fail(QGEMM_ERR_INVALID_ARG, "bad epilogue %d", op);
  if (op == QGEMM_EPI_RESIDUAL_GATE) {
    if (!epi->residual || !epi->gate) return fail(QGEMM_ERR_INVALID_ARG, "the residual update needs residual and gate");
    if (!aligned16(epi->residual)) return fail(QGEMM_ERR_ALIGNMENT, "residual must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(epi->gate) & 1u) return fail(QGEMM_ERR_ALIGNMENT, "gate must be 2-byte aligned");
  }
  if (M == 0) return QGEMM_OK;
  if (!X || !out) return fail(QGEMM_ERR_INVALID_ARG, "null X or out");
  if (!aligned16(X) || !aligned16(out)) return fail(QGEMM_ERR_ALIGNMENT, "X and out must be 16-byte aligned");
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) return fail(QGEMM_ERR_ALIGNMENT, "bias must be 2-byte aligned");
  if (path == QGEMM_PATH_AUTO) path = auto_path(M, W->N, W->K, W->bits);
  if (path == QGEMM_PATH_SMALL_M && M > kSmallPathMaxM)
    return fail(QGEMM_ERR_UNSUPPORTED, "the small-M path takes M <= %d (M=%d)", kSmallPathMaxM, M);
  if (path == QGEMM_PATH_SMALL_M && W->bits == 1 && W->K % 256)
    return fail(QGEMM_ERR_UNSUPPORTED, "the small-M path takes 1-bit weights with K %% 256 == 0 (K=%d)", W->K);
  Problem p{X, M, W->N, W->K, W->bits, W->group, static_cast<const uint8_t*>(W->packed),
            static_cast<const uint16_t*>(W->scales), static_cast<const uint16_t*>(W->biases), out,
            static_cast<const uint16_t*>(bias), static_cast<cudaStream_t>(stream),
            (flags & QGEMM_FLAG_OVERLAP_PREVIOUS) != 0, op,
            op == QGEMM_EPI_RESIDUAL_GATE ? static_cast<const uint16_t*>(epi->residual) : nullptr,
            op == QGEMM_EPI_RESIDUAL_GATE ? static_cast<const uint16_t*>(epi->gate) : nullptr};
  if (path == QGEMM_PATH_SMALL_M) return launch_small_rows(p);
  return launch_large_m(p);
}

extern "C" int qgemm_ex(const void* X, int32_t M, const qgemm_weights* W, void* out, const void* bias,
                        int32_t path, void* stream) {
  return qgemm_fused(X, M, W, out, bias, nullptr, path, stream);
}

extern "C" int qgemm_pack_device(const void* W, int32_t N, int32_t K, int32_t bits, int32_t group, void* packed,
                                 void* scales, void* biases, void* stream) {
  size_t pb, sb, bb;
  int st = qgemm_pack_sizes(N, K, bits, group, &pb, &sb, &bb);
  if (st != QGEMM_OK) return st;
  if (!W || !packed || !scales || (bits > 2 && !biases))
    return fail(QGEMM_ERR_INVALID_ARG, "null buffer passed to qgemm_pack_device");
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scales) || (bits > 2 && !aligned16(biases)))
    return fail(QGEMM_ERR_ALIGNMENT, "W, packed, scales and biases must be 16-byte aligned");
  return launch_pack_device(static_cast<const float*>(W), N, K, bits, packed, static_cast<uint16_t*>(scales),
                            static_cast<uint16_t*>(biases), static_cast<cudaStream_t>(stream));
}

extern "C" int qgemm(const void* X, int32_t M, const qgemm_weights* W, void* out, const void* bias, void* stream) {
  return qgemm_ex(X, M, W, out, bias, QGEMM_PATH_AUTO, stream);
}

extern "C" int qgemm_select_path(int32_t M, int32_t N, int32_t K, int32_t bits) {
  if (M < 0 || N <= 0 || K <= 0) return -QGEMM_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return -QGEMM_ERR_UNSUPPORTED;
  if (bits != 1 && bits != 2 && bits != 4 && bits != 8) return -QGEMM_ERR_UNSUPPORTED;
  return auto_path(M, N, K, bits);
}

extern "C" int qgemm_dequant_tile(const qgemm_weights* W, int32_t n0, int32_t k0, int32_t rows, int32_t cols,
                                  void* out, void* stream) {
  int st = validate_weights(W);
  if (st != QGEMM_OK) return st;
  if (!out) return fail(QGEMM_ERR_INVALID_ARG, "null out");
  if (n0 < 0 || k0 < 0 || rows < 0 || cols < 0 || n0 + static_cast<int64_t>(rows) > W->N ||
      k0 + static_cast<int64_t>(cols) > W->K)
    return fail(QGEMM_ERR_INVALID_ARG, "tile [%d+%d, %d+%d] is outside W [%d, %d]", n0, rows, k0, cols, W->N, W->K);
  if (k0 % 8 || cols % 8) return fail(QGEMM_ERR_INVALID_ARG, "k0 and cols must be multiples of 8");
  if (!aligned16(out)) return fail(QGEMM_ERR_ALIGNMENT, "out must be 16-byte aligned");
  if (rows == 0 || cols == 0) return QGEMM_OK;
  Problem p{nullptr, 0, W->N, W->K, W->bits, W->group, static_cast<const uint8_t*>(W->packed),
            static_cast<const uint16_t*>(W->scales), static_cast<const uint16_t*>(W->biases), out, nullptr,
            static_cast<cudaStream_t>(stream)};
  return launch_dequant_tile(p, n0, k0, rows, cols);
}

extern "C" int qgemm_grouped(const qgemm_problem* problems, int32_t count, int32_t flags, void* stream) {
  if (!problems) return fail(QGEMM_ERR_INVALID_ARG, "null problem list");
  if (count < 1 || count > kGroupedMaxProblems)
    return fail(QGEMM_ERR_INVALID_ARG, "count=%d: 1 to %d problems per grouped call", count, kGroupedMaxProblems);
  if (flags & ~(QGEMM_FLAG_OVERLAP_PREVIOUS | QGEMM_FLAG_GROUPED_ONE_LAUNCH))
    return fail(QGEMM_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  Problem probs[kGroupedMaxProblems];
  bool any = false;
  for (int i = 0; i < count; ++i) {
    const qgemm_problem& q = problems[i];
    int st = validate_weights(&q.W);
    if (st != QGEMM_OK) return st;
    if (q.W.bits != problems[0].W.bits)
      return fail(QGEMM_ERR_UNSUPPORTED, "grouped: problem %d has %d-bit weights, problem 0 %d-bit", i, q.W.bits,
                  problems[0].W.bits);
    if (q.M < 0 || q.M > kSmallGroupedMaxM)
      return fail(QGEMM_ERR_UNSUPPORTED, "grouped: problem %d has M=%d (0 to %d)", i, q.M, kSmallGroupedMaxM);
    if (!small_path_takes(q.M, q.W.K, q.W.bits))
      return fail(QGEMM_ERR_UNSUPPORTED, "grouped: problem %d (1-bit weights need K %% 256 == 0)", i);
    if (q.M > 0) {
      if (!q.X || !q.out) return fail(QGEMM_ERR_INVALID_ARG, "grouped: problem %d has a null X or out", i);
      if (!aligned16(q.X) || !aligned16(q.out))
        return fail(QGEMM_ERR_ALIGNMENT, "grouped: problem %d: X and out must be 16-byte aligned", i);
      if (q.bias && (reinterpret_cast<uintptr_t>(q.bias) & 1u))
        return fail(QGEMM_ERR_ALIGNMENT, "grouped: problem %d: bias must be 2-byte aligned", i);
      any = true;
    }
    probs[i] = Problem{q.X, q.M, q.W.N, q.W.K, q.W.bits, q.W.group, static_cast<const uint8_t*>(q.W.packed),
                       static_cast<const uint16_t*>(q.W.scales), static_cast<const uint16_t*>(q.W.biases), q.out,
                       static_cast<const uint16_t*>(q.bias), static_cast<cudaStream_t>(stream),
                       (flags & QGEMM_FLAG_OVERLAP_PREVIOUS) != 0, QGEMM_EPI_NONE, nullptr, nullptr};
  }
  if (!any) return QGEMM_OK;
  if (flags & QGEMM_FLAG_GROUPED_ONE_LAUNCH)
    return launch_small_m_grouped(probs, count, (flags & QGEMM_FLAG_OVERLAP_PREVIOUS) != 0,
                                  static_cast<cudaStream_t>(stream));
  // consecutive launches, the later ones overlapping the one before: the
  // problems are independent (no output overlaps another problem's operands)
  bool first = true;
  for (int i = 0; i < count; ++i) {
    if (probs[i].M == 0) continue;
    Problem p = probs[i];
    if (!first) p.overlap = true;
    first = false;
    const int st = launch_small_rows(p);
    if (st != QGEMM_OK) return st;
  }
  return QGEMM_OK;
}

extern "C" int qgemm_debug_stream(const void* X, int32_t M, const qgemm_weights* W, int32_t flags, void* stream) {
  int st = validate_weights(W);
  if (st != QGEMM_OK) return st;
  if (M < 0) return fail(QGEMM_ERR_INVALID_ARG, "M=%d is negative", M);
  if (flags & ~QGEMM_FLAG_OVERLAP_PREVIOUS) return fail(QGEMM_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (!small_path_takes(M, W->K, W->bits))
    return fail(QGEMM_ERR_UNSUPPORTED, "the small-M path does not take M=%d, K=%d, bits=%d", M, W->K, W->bits);
  if (M == 0) return QGEMM_OK;
  if (!X) return fail(QGEMM_ERR_INVALID_ARG, "null X");
  if (!aligned16(X)) return fail(QGEMM_ERR_ALIGNMENT, "X must be 16-byte aligned");
  Problem p{X, M, W->N, W->K, W->bits, W->group, static_cast<const uint8_t*>(W->packed),
            static_cast<const uint16_t*>(W->scales), static_cast<const uint16_t*>(W->biases), nullptr, nullptr,
            static_cast<cudaStream_t>(stream), (flags & QGEMM_FLAG_OVERLAP_PREVIOUS) != 0, QGEMM_EPI_NONE,
            nullptr, nullptr, true};
  return launch_small_rows(p);
}

extern "C" int qgemm_set_wait_limit_ns(uint64_t limit_ns) {
  std::call_once(g_env_once, read_env);
  g_wait_limit_ns.store(limit_ns ? limit_ns : kDefaultWaitLimitNs);
  return QGEMM_OK;
}

extern "C" int qgemm_debug_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0) return fail(QGEMM_ERR_INVALID_ARG, "limit_ns must be positive");
  return launch_debug_wait(limit_ns, static_cast<cudaStream_t>(stream));
}

extern "C" const char* qgemm_status_str(int status) {
  switch (status) {
    case QGEMM_OK: return "ok";
    case QGEMM_ERR_INVALID_ARG: return "invalid argument";
    case QGEMM_ERR_UNSUPPORTED: return "unsupported format, shape or device";
    case QGEMM_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case QGEMM_ERR_NONFINITE: return "non-finite weight";
    case QGEMM_ERR_CUDA: return "CUDA error";
    case QGEMM_ERR_DEVICE_TIMEOUT: return "a device-side wait timed out";
    default: return "unknown status";
  }
}

extern "C" const char* qgemm_last_error(void) { return t_last_error.c_str(); }

extern "C" const char* qgemm_version(void) { return "qgemm 0.1 (sm_100a)"; }
