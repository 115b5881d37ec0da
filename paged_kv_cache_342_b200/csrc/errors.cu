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

}  // namespace pa

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
