// Device status word, device queries and the bounded-wait test hook.

#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

#include "ptx.cuh"
#include "qgemm_internal.h"

namespace qg {

// One status word per device that loads this library. Kernels OR a code into
// it when a bounded wait gives up; qgemm_get_device_status reads and clears
// it. A file-scope device variable: nothing is allocated.
__device__ unsigned int g_status_word;
// The value the status word held when qgemm_get_device_status last took it.
__device__ unsigned int g_status_taken;

namespace {
constexpr int kMaxDevices = 64;
unsigned int* g_status_ptr[kMaxDevices];
int g_sm_count[kMaxDevices];
std::mutex g_mu;

std::mutex g_take_mu;  // one qgemm_get_device_status at a time: they share g_status_taken

// Reads and clears the status word in one atomic step, so that a code a
// kernel on another stream sets in between is never lost: it is either
// taken now or left for the next read.
__global__ void take_status_kernel(unsigned int* word, unsigned int* taken) { *taken = atomicExch(word, 0u); }

int current_device(int* dev) {
  int st = cuda_check(cudaGetDevice(dev), "cudaGetDevice");
  if (st != QGEMM_OK) return st;
  if (*dev < 0 || *dev >= kMaxDevices) return fail(QGEMM_ERR_UNSUPPORTED, "device ordinal %d out of range", *dev);
  return QGEMM_OK;
}

__global__ void debug_wait_kernel(uint64_t limit_ns, unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ptx::smem_u32(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbarrier_init();
  // Nothing ever arrives on this barrier: the wait must run out and report.
  if (!ptx::mbar_wait(b, 0, limit_ns, nullptr)) ptx::set_status(status, kStatusTimeout);
}
}  // namespace

int status_word(unsigned int** ptr) {
  int dev;
  int st = current_device(&dev);
  if (st != QGEMM_OK) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    st = cuda_check(cudaGetSymbolAddress(&p, g_status_word), "cudaGetSymbolAddress(status word)");
    if (st != QGEMM_OK) return st;
    g_status_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *ptr = g_status_ptr[dev];
  return QGEMM_OK;
}

int smem_opt_in(const void* func, int bytes, const char* what) {
  int dev;
  int st = current_device(&dev);
  if (st != QGEMM_OK) return st;
  static std::set<std::pair<int, const void*>> done;  // (device, kernel) pairs already configured
  std::lock_guard<std::mutex> lk(g_mu);
  if (done.count({dev, func})) return QGEMM_OK;
  st = cuda_check(cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes), what);
  if (st == QGEMM_OK) done.insert({dev, func});
  return st;
}

int sm_count(int* n) {
  int dev;
  int st = current_device(&dev);
  if (st != QGEMM_OK) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[dev]) {
    int v = 0;
    st = cuda_check(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute");
    if (st != QGEMM_OK) return st;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(QGEMM_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device is sm_%d%d", major, minor);
    g_sm_count[dev] = v;
  }
  *n = g_sm_count[dev];
  return QGEMM_OK;
}

int launch_debug_wait(uint64_t limit_ns, cudaStream_t stream) {
  int n;
  int st = sm_count(&n);
  if (st != QGEMM_OK) return st;
  unsigned int* status;
  st = status_word(&status);
  if (st != QGEMM_OK) return st;
  debug_wait_kernel<<<1, 1, 0, stream>>>(limit_ns, status);
  return cuda_check(cudaGetLastError(), "debug_wait_kernel launch");
}

}  // namespace qg

extern "C" int qgemm_get_device_status(void* stream) {
  using namespace qg;
  unsigned int* status;
  int st = status_word(&status);
  if (st != QGEMM_OK) return st;
  std::lock_guard<std::mutex> lk(g_take_mu);
  void* taken = nullptr;
  st = cuda_check(cudaGetSymbolAddress(&taken, g_status_taken), "cudaGetSymbolAddress(status copy)");
  if (st != QGEMM_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  take_status_kernel<<<1, 1, 0, s>>>(status, static_cast<unsigned int*>(taken));
  st = cuda_check(cudaGetLastError(), "take_status_kernel launch");
  if (st != QGEMM_OK) return st;
  unsigned int v = 0;
  st = cuda_check(cudaMemcpyAsync(&v, taken, sizeof v, cudaMemcpyDeviceToHost, s), "read status word");
  if (st != QGEMM_OK) return st;
  st = cuda_check(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (st != QGEMM_OK) return st;
  if (v) {
    if (v & kStatusPackNonfinite)
      return fail(QGEMM_ERR_NONFINITE, "qgemm_pack_device met a non-finite weight (status word 0x%x)", v);
    if (v & kStatusPackOverflow)
      return fail(QGEMM_ERR_UNSUPPORTED, "qgemm_pack_device: a group's scale or bias overflows fp16 (status word 0x%x)",
                  v);
    if (v & kStatusLayout)
      return fail(QGEMM_ERR_CUDA, "a kernel found its shared-memory base off its alignment (status word 0x%x)", v);
    return fail(QGEMM_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (status word 0x%x)", v);
  }
  return QGEMM_OK;
}
