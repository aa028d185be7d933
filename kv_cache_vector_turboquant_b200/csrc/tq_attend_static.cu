// tq_attend_decode_static: the fused decode-step attention for callers that
// cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc at all: a plugin running
// inside a serving framework that owns every byte of device memory through its
// own pool, or a latency-bound decode loop where an allocation would
// synchronise the device or could fail part-way through a generation. This
// entry point takes the split-S scratch of tq_attend_decode from a fixed
// array in device memory that is part of the library itself (one per device
// that loads the library, held until the process exits), so the caller only
// passes inputs and outputs.
#include <cuda_runtime.h>

#include <atomic>

#include "tq_internal.h"

namespace {

// The scratch array. In host code its name is only a stand-in for the symbol
// (not a device address); the device address is looked up per device below.
__device__ __align__(256) unsigned char g_tq_attend_scratch[TQ_ATTEND_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<uintptr_t> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device; looked up once
// per device (with that device current) and cached. nullptr on failure.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const uintptr_t cached = g_scratch_addr[dev].load();
  if (cached) return reinterpret_cast<void*>(cached);
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_tq_attend_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
  g_scratch_addr[dev].store(reinterpret_cast<uintptr_t>(ptr));
  return ptr;
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" tq_status tq_attend_decode_static(const tq_ctx* k, const tq_ctx* v, const void* q_f16, int B, int hq,
                                             int hkv, const void* k_packed, const float* k_norms,
                                             const void* v_packed, const float* v_norms, int64_t s_max,
                                             const int32_t* positions, void* out_f16, tq_stream stream) {
  if (!k || !v) return TQ_ERR_INVALID_ARG;
  if (k->d != v->d) return TQ_ERR_INVALID_ARG;
  if (B < 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || s_max <= 0) return TQ_ERR_INVALID_ARG;
  if (B == 0) return TQ_OK;
  if (!q_f16 || !k_packed || !k_norms || !v_packed || !v_norms || !positions || !out_f16)
    return TQ_ERR_INVALID_ARG;
  if (!aligned_to(q_f16, 16) || !aligned_to(k_packed, 16) || !aligned_to(v_packed, 16) ||
      !aligned_to(out_f16, 16) || !aligned_to(k_norms, 4) || !aligned_to(v_norms, 4) || !aligned_to(positions, 4))
    return TQ_ERR_ALIGNMENT;
  const size_t need = tq_attend_workspace_bytes_impl(B, hq, k->d, s_max);
  if (need == 0) return TQ_ERR_INVALID_ARG;
  if (need > TQ_ATTEND_STATIC_SCRATCH_BYTES) return TQ_ERR_WORKSPACE;  // too large for the fixed scratch
  void* ws = scratch_address();
  if (!ws) return TQ_ERR_CUDA;
  return tq_launch_attend(k, v, q_f16, B, hq, hkv, k_packed, k_norms, v_packed, v_norms, s_max, positions,
                          out_f16, ws, TQ_ATTEND_STATIC_SCRATCH_BYTES, stream);
}
