// Test hooks of libtq (include/tq_test.h), built into libtq_test.so, which is
// linked against libtq.so and never loaded by the product path. The hooks
// call libtq.so's own internal launchers, so the kernels they start record
// into the same device error word and read the same run-time check state as
// the public entry points.
#include <stdint.h>

#include "tq_internal.h"
#include "tq_test.h"

namespace {
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
}  // namespace

extern "C" {

// tq_encode with the row copies withheld, so every wait of the kernel runs
// out after a short bound.
tq_status tq_test_encode_stalled(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, float* norms,
                                 tq_stream stream) {
  if (!ctx || n <= 0 || !x_f16 || !packed || !norms) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(norms, 4)) return TQ_ERR_ALIGNMENT;
  return tq_launch_encode(ctx, x_f16, n, packed, norms, nullptr, 1, 1, stream, 1);
}

// tq_decode (paths 1, 2) or tq_decode_os (paths 3, 4: `norms` holds the side
// words) through a chosen kernel.
tq_status tq_test_decode_path(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x_f16,
                              int path, tq_stream stream) {
  if (!ctx || n <= 0 || !x_f16 || !packed || !norms) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(norms, 4)) return TQ_ERR_ALIGNMENT;
  const uint32_t* side = reinterpret_cast<const uint32_t*>(norms);
  switch (path) {
    case 1: return tq_launch_decode(ctx, packed, norms, n, x_f16, stream);
    case 2: return tq_launch_decode_tc(ctx, packed, norms, n, x_f16, stream);
    case 3: return tq_launch_decode_os(ctx, packed, side, n, x_f16, stream);
    case 4: return tq_launch_decode_tc_os(ctx, packed, side, n, x_f16, stream);
    default: return TQ_ERR_INVALID_ARG;
  }
}

// tq_encode through a chosen kernel.
tq_status tq_test_encode_path(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, float* norms, int path,
                              tq_stream stream) {
  if (!ctx || n <= 0 || !x_f16 || !packed || !norms) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(norms, 4)) return TQ_ERR_ALIGNMENT;
  switch (path) {
    case 1: return tq_launch_encode(ctx, x_f16, n, packed, norms, nullptr, 1, 1, stream, 0);
    case 2: return tq_launch_encode_tc(ctx, x_f16, n, packed, norms, stream, 0);
    case 3: return tq_launch_encode_tc(ctx, x_f16, n, packed, norms, stream, 1);
    default: return TQ_ERR_INVALID_ARG;
  }
}

// Forget the current device's tensor-core check result (optionally forcing
// the next check to report a mismatch).
tq_status tq_test_reset_tensor_core_check(int force_fail) { return tq_tensor_core_check_reset(force_fail); }

tq_status tq_test_attend_plan(int d, int hw, int nt, int paged, int reserved, int max_dyn, int32_t* out) {
  if (!out) return TQ_ERR_INVALID_ARG;
  return tq_attend_fast_plan(d, hw, nt, paged, reserved, max_dyn, out) ? TQ_OK : TQ_ERR_UNSUPPORTED;
}

}  // extern "C"
