// The library's device error word: kernels OR PA_DEVERR_* bits into it when they
// skip an out-of-range index or give up a bounded wait; pa_device_error_read
// returns and clears it.
#include <atomic>
#include <cstdio>

#include "common.cuh"

namespace pa {

__device__ uint32_t g_error_word;

namespace {
constexpr int kMaxDevices = 64;
std::atomic<uint32_t*> g_error_addr[kMaxDevices];
}  // namespace

// Device address of the error word for the current device, looked up once per
// device (cudaGetSymbolAddress) and cached.
uint32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  uint32_t* p = g_error_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return nullptr;
  g_error_addr[dev].store(static_cast<uint32_t*>(addr), std::memory_order_release);
  return static_cast<uint32_t*>(addr);
}

namespace {
thread_local char g_last_cuda_error[256] = "";
}  // namespace

void note_cuda_error(cudaError_t e) {
  if (e == cudaSuccess) return;
  const char* name = cudaGetErrorName(e);
  const char* text = cudaGetErrorString(e);
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", name ? name : "?",
           text ? text : "?");
}

// One thread waits, with the decode kernels' bounded wait, on an mbarrier that nothing
// ever completes: the bound (about one second) must end the wait and report it.
__global__ void bounded_wait_selftest_kernel(uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  mbar_init(b, 1);
  mbar_init_fence();
  if (!mbar_wait_bounded(b, 0)) set_error(err, PA_DEVERR_TIMEOUT);
}

}  // namespace pa

extern "C" int pa_selftest_bounded_wait(pa_stream_t stream) {
  uint32_t* err = pa::device_error_word();
  if (!err) {
    pa::note_cuda_error(cudaGetLastError());
    return PA_ERR_CUDA;
  }
  pa::bounded_wait_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(err);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    pa::note_cuda_error(e);
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

extern "C" const char* pa_last_cuda_error(void) { return pa::g_last_cuda_error; }

extern "C" int pa_device_error_read(uint32_t* bits) {
  if (!bits) return PA_ERR_INVALID_ARG;
  *bits = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(bits, pa::g_error_word, sizeof(uint32_t));
  const uint32_t zero = 0;
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(uint32_t));
  if (e != cudaSuccess) {
    pa::note_cuda_error(e);
    return PA_ERR_CUDA;
  }
  return PA_OK;
}
