// The library's device error word: kernels OR PA_DEVERR_* bits into it when they
// skip an out-of-range index or give up a bounded wait; pa_device_error_read
// returns and clears it.
#include <atomic>

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

}  // namespace pa

extern "C" int pa_device_error_read(uint32_t* bits) {
  if (!bits) return PA_ERR_INVALID_ARG;
  *bits = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(bits, pa::g_error_word, sizeof(uint32_t)) != cudaSuccess)
    return PA_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(uint32_t)) != cudaSuccess)
    return PA_ERR_CUDA;
  return PA_OK;
}
