// Test hook: one tcgen05 MMA of kind::f16 (M = 128, N = K = 16, f32
// accumulator, no accumulate input) on caller operands, with the descriptors,
// swizzle and tensor-memory lane layout of the tensor-core encode kernel. It
// lets the tests pin the arithmetic that the encode kernel's error bound
// assumes (exact products; addend magnitudes cut at 2^(E-25); the sum rounded
// toward zero) on the hardware the library runs on.
#include <cuda_runtime.h>

#include <atomic>

#include "tq_common.cuh"
#include "tq_umma.cuh"

namespace tq {

// One CTA of 128 threads. Shared memory (1024-aligned): A atom [128 rows x
// 128 B] (16 KB), B atom [16 rows x 128 B] (2 KB), the mbarrier and the
// tensor-memory address slot.
__global__ void __launch_bounds__(128, 1)
    umma_block_probe_kernel(const __half* __restrict__ A, const __half* __restrict__ B, float* __restrict__ D,
                            uint32_t* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  constexpr uint32_t A_OFF = 0, B_OFF = 16384, BAR_OFF = 16384 + 2048, SLOT_OFF = BAR_OFF + 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // operands in the K-major 128-byte-swizzled layout (only K = 16 columns used)
  for (int i = tid; i < 128 * 16; i += 128) {
    const int r = i >> 4, k = i & 15;
    const uint32_t off = A_OFF + r * 128 + ((((k * 2) >> 4) ^ (r & 7)) << 4) + ((k * 2) & 15);
    *reinterpret_cast<__half*>(sm + off) = A[i];
  }
  for (int i = tid; i < 16 * 16; i += 128) {
    const int r = i >> 4, k = i & 15;
    const uint32_t off = B_OFF + r * 128 + ((((k * 2) >> 4) ^ (r & 7)) << 4) + ((k * 2) & 15);
    *reinterpret_cast<__half*>(sm + off) = B[i];
  }
  fence_proxy_async_smem();
  const uint32_t bar = base + BAR_OFF;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(base + SLOT_OFF, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + SLOT_OFF);
  if (tid == 0) {
    umma_f16(tmem, umma_desc_sw128(base + A_OFF), umma_desc_sw128(base + B_OFF), umma_idesc_f16(128, 16), false);
    umma_commit(bar);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, 0, TQ_WAIT_LIMIT_CYCLES));
  if (!ok) {
    if (lane == 0) record_error(err, TQ_DEVERR_TIMEOUT);
  } else {
    tc_fence_after();
    uint32_t r[16];
    tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16), r);
    tmem_wait_ld();
    tmem_regs_after_wait(r);
#pragma unroll
    for (int c = 0; c < 16; ++c) D[(32 * warp + lane) * 16 + c] = __uint_as_float(r[c]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

}  // namespace tq

using namespace tq;

extern "C" tq_status tq_test_umma_block(const void* a_f16, const void* b_f16, float* d, tq_stream stream) {
  if (!a_f16 || !b_f16 || !d) return TQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a_f16) & 1) || (reinterpret_cast<uintptr_t>(b_f16) & 1) ||
      (reinterpret_cast<uintptr_t>(d) & 3))
    return TQ_ERR_ALIGNMENT;
  uint32_t* err = tq_error_word();
  if (!err) return TQ_ERR_CUDA;
  constexpr int smem = 1024 + 16384 + 2048 + 64;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  static std::atomic<uint64_t> configured{0};  // one bit per device
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    if (cudaFuncSetAttribute(umma_block_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return TQ_ERR_CUDA;
    configured.fetch_or(bit);
  }
  umma_block_probe_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half*>(a_f16), static_cast<const __half*>(b_f16), d, err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
