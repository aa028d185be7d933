// Per-device runtime state of libtq: the device error word and cached device
// attributes. No device memory is allocated: the error word is a file-scope
// __device__ variable, one per device that loads the library.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "tq_internal.h"

namespace {
__device__ uint32_t g_tq_error_word;

constexpr int kMaxDevices = 64;
std::atomic<uintptr_t> g_err_ptr[kMaxDevices];
std::atomic<int> g_sm_count[kMaxDevices];
}  // namespace

int tq_sm_count(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = g_sm_count[dev].load();
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
  g_sm_count[dev].store(v);
  return v;
}

uint32_t* tq_error_word(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  uintptr_t p = g_err_ptr[dev].load();
  if (p) return reinterpret_cast<uint32_t*>(p);
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_tq_error_word) != cudaSuccess) return nullptr;
  g_err_ptr[dev].store(reinterpret_cast<uintptr_t>(addr));
  return static_cast<uint32_t*>(addr);
}

tq_status tq_read_error_word(void* stream, uint32_t* bits) {
  uint32_t* dptr = tq_error_word();
  if (!dptr) return TQ_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, dptr, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaMemsetAsync(dptr, 0, sizeof(uint32_t), st) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ERR_CUDA;
  if (bits) *bits = host;
  if (host & TQ_DEVERR_TIMEOUT) return TQ_ERR_TIMEOUT;
  if (host) return TQ_ERR_DEVICE;
  return TQ_OK;
}

void* tq_tensor_map_encode_fn(void) {
  static void* fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  });
  return fn;
}
