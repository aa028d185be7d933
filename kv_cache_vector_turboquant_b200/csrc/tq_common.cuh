// Device helpers shared by the libtq kernels (sm_100a): mbarrier waits with
// a bound, 1-D bulk (TMA) copies, packed f32x2 arithmetic and the device
// error word. Hand-written PTX, no library kernels.
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_internal.h"

#define TQ_DEV __device__ __forceinline__

// Bound on every mbarrier wait: about one second at B200 clocks. A wait that
// runs out records TQ_DEVERR_TIMEOUT and the kernel returns.
#define TQ_WAIT_LIMIT_CYCLES (2000000000LL)

namespace tq {

TQ_DEV int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

TQ_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

TQ_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

TQ_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

TQ_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

TQ_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

TQ_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of the barrier to complete, for at most `limit`
// SM clock cycles. Returns false if the bound ran out.
// Programmatic dependent launch (sm_90 and later). A kernel launched with
// programmatic stream serialisation (tq_launch_pdl) may start while the
// previous kernel of the stream is still finishing: grid_dep_wait() blocks the
// calling thread until that kernel has completed and its memory operations
// are visible, so every thread that touches global memory calls it first;
// grid_dep_launch() lets the next such kernel start once every CTA of this
// grid has issued it or exited. A CTA that has not started has issued
// nothing, so dependents are scheduled only when every CTA of this grid is
// running or done: a dependent CTA waiting for this grid never holds an SM
// that one of its CTAs still needs, whatever the grid size.
TQ_DEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
TQ_DEV void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

TQ_DEV bool mbar_wait_bounded(uint32_t bar, uint32_t parity, long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}

// ---------------------------------------------------------------- bulk copies

// 1-D bulk copy global -> shared (TMA engine), completion counted in bytes on
// the mbarrier. Both addresses 16-byte aligned, bytes a multiple of 16.
// No multicast.
TQ_DEV void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 1-D bulk copy shared -> global, tracked by this thread's bulk group.
TQ_DEV void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
TQ_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
TQ_DEV void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
TQ_DEV void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (bulk copies) that reads them next.
TQ_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- f32x2

// Packed two-wide f32 arithmetic of sm_100 (one instruction for both
// lanes of the pair), each component rounded exactly like its scalar op.
using f2 = float2;

TQ_DEV f2 add2(f2 a, f2 b) { return __fadd2_rn(a, b); }
TQ_DEV f2 sub2(f2 a, f2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
TQ_DEV f2 mul2(f2 a, f2 b) { return __fmul2_rn(a, b); }
TQ_DEV f2 fma2(f2 a, f2 b, f2 c) { return __ffma2_rn(a, b, c); }
// Round toward -inf (used to take floor(q) through the 2^23 magic constant).
TQ_DEV f2 add2_rm(f2 a, f2 b) { return __fadd2_rd(a, b); }

// In-register Walsh-Hadamard butterflies over N pairs v[j] = (e_{2j}, e_{2j+1})
// for the element strides 2, 4, ..., N (pair strides 1 .. N/2). The stride-1
// butterfly inside each pair is done by the caller. Natural order, no scaling.
template <int NP>
TQ_DEV void wht_pairs(f2 (&v)[NP]) {
#pragma unroll
  for (int hp = 1; hp < NP; hp <<= 1) {
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      if ((j & hp) == 0) {
        const f2 a = v[j], b = v[j + hp];
        v[j] = add2(a, b);
        v[j + hp] = sub2(a, b);
      }
    }
  }
}

// ---------------------------------------------------------------- error word

TQ_DEV void record_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

TQ_DEV uint32_t lane_id() {
  uint32_t l;
  asm("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

// Launch with programmatic stream serialisation (see grid_dep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t tq_launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace tq
