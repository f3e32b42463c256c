// status.cu -- the per-device status word the kernels set instead of faulting
// (out-of-range block ids, context lengths, slots, copy pairs, and pipeline
// waits that gave up), plus the host-side error message and launch counter.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {
__device__ unsigned int g_status_word;

thread_local char g_last_error[512] = "";

// One CTA waits on an mbarrier that expects an arrival nothing makes, with a
// short limit: the wait must give up, record PA_DEVERR_TIMEOUT and return.
__global__ void wait_timeout_selftest_kernel(unsigned int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, status, limit_ns);
}
std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;
unsigned int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;
}  // namespace

pa_status fail(pa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

unsigned int* device_status_word() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    return nullptr;
  }
  {
    std::lock_guard<std::mutex> lk(g_status_mu);
    if (g_status_ptr[dev]) return g_status_ptr[dev];
  }
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_status_word);
  if (e != cudaSuccess || !ptr) {
    fail(PA_ERR_CUDA, "cudaGetSymbolAddress(status word): %s", cudaGetErrorString(e));
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_status_mu);
  g_status_ptr[dev] = static_cast<unsigned int*>(ptr);
  return g_status_ptr[dev];
}

}  // namespace pa

extern "C" const char* pa_last_error(void) { return pa::g_last_error; }

extern "C" uint64_t pa_launch_count(void) {
  return pa::g_launches.load(std::memory_order_relaxed);
}

extern "C" pa_status pa_device_status(unsigned int* flags_out, int clear) {
  if (!flags_out) return pa::fail(PA_ERR_INVALID, "pa_device_status: flags_out is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "pa_device_status: %s", cudaGetErrorString(e));
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, pa::g_status_word, sizeof(v));
  if (e != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "pa_device_status: %s", cudaGetErrorString(e));
  *flags_out = v;
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(pa::g_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess)
      return pa::fail(PA_ERR_CUDA, "pa_device_status: %s", cudaGetErrorString(e));
  }
  return PA_OK;
}

extern "C" pa_status pa_selftest_wait_timeout(unsigned int* flags_out) {
  if (!flags_out) return pa::fail(PA_ERR_INVALID, "pa_selftest_wait_timeout: flags_out is NULL");
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  unsigned int before = 0;
  pa_status st = pa_device_status(&before, 1);
  if (st != PA_OK) return st;
  pa::wait_timeout_selftest_kernel<<<1, 32>>>(status, 20000000ull);  // 20 ms
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "pa_selftest_wait_timeout: %s", cudaGetErrorString(e));
  pa::count_launch();
  st = pa_device_status(flags_out, 1);
  if (st != PA_OK) return st;
  if (before) {  // keep what the caller had not read yet
    const unsigned int merged = before;
    cudaMemcpyToSymbol(pa::g_status_word, &merged, sizeof(merged));
  }
  return PA_OK;
}
