/*
 * tq_test.h -- test hooks of libtq. Not for production use.
 *
 * These calls are exported by libtq_test.so, a separate library linked
 * against libtq.so (found beside it through $ORIGIN). They run libtq.so's own
 * kernels and launchers, so they record into the same device error word
 * (tq_device_error) as the public calls. The product library libtq.so
 * exports none of them.
 */
#ifndef TQ_TEST_H_
#define TQ_TEST_H_

#include "tq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * tq_encode with the kernel's row copies withheld: the kernel's first
 * bounded mbarrier wait runs out (after about 10 ms instead of the usual
 * second), the kernel records TQ_DEVERR_TIMEOUT in the device error word and
 * returns without writing `packed` or `norms`. Lets a test check that a wait
 * that never completes ends with an error status the host can read
 * (tq_device_error -> TQ_ERR_TIMEOUT) and a context that stays usable.
 * Same arguments, alignment rules and asynchrony as tq_encode; n must be > 0.
 */
tq_status tq_test_encode_stalled(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, float* norms,
                                 tq_stream stream);

/*
 * tq_encode through a chosen kernel, whatever n is:
 *   path 1  the CUDA-core kernel (tq_encode's choice below
 *           128 x SM-count vectors),
 *   path 2  the tensor-core kernel (tq_encode's choice from there on),
 *   path 3  the tensor-core kernel with its row copies withheld, like
 *           tq_test_encode_stalled: TQ_DEVERR_TIMEOUT after about 10 ms per
 *           wait, nothing written.
 * Same arguments, alignment rules and asynchrony as tq_encode; n must be > 0;
 * any other path is TQ_ERR_INVALID_ARG.
 */
tq_status tq_test_encode_path(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, float* norms, int path,
                              tq_stream stream);

/*
 * tq_decode through a chosen kernel, whatever n is: path 1 the CUDA-core
 * kernel (tq_decode's choice below 128 x SM-count vectors, and at
 * head_dim 256), path 2 the tensor-core kernel (head_dim 64 and 128 only:
 * TQ_ERR_UNSUPPORTED at 256). Paths 3 and 4 are the same two kernels for
 * tq_decode_os: `norms` then points at its uint32 side words. Same
 * arguments, alignment rules and asynchrony as tq_decode; n must be > 0; any
 * other path is TQ_ERR_INVALID_ARG.
 */
tq_status tq_test_decode_path(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x_f16,
                              int path, tq_stream stream);

/*
 * One fifth-generation tensor-core MMA (tcgen05.mma kind::f16, M = 128,
 * N = K = 16, f32 accumulator starting from zero), with the shared-memory
 * layout and tensor-memory readback of the tensor-core encode kernel:
 *   d[m][n] = sum_k a[m][k] * b[n][k]
 *   a_f16  device, [128][16] fp16 (row-major), 2-byte aligned;
 *   b_f16  device, [16][16] fp16 (row-major: b[n][k]), 2-byte aligned;
 *   d      device, [128][16] float32 out, 4-byte aligned.
 * Lets the tests check, on the GPU the library runs on, the rounding that the
 * encode kernel's exactness argument assumes. One CTA, asynchronous on
 * `stream`; TQ_ERR_INVALID_ARG for a null pointer, TQ_ERR_ALIGNMENT for a
 * misaligned one; a wait that runs out is reported through tq_device_error.
 */
tq_status tq_test_umma_block(const void* a_f16, const void* b_f16, float* d, tq_stream stream);

/*
 * Forget the current device's result of the tensor-core check
 * (tq_tensor_core_check), so that the next bulk tq_encode / tq_decode or
 * tq_tensor_core_check runs it again. With force_fail != 0 that next check
 * reports a mismatch whatever the MMA returned, so a test can see bulk
 * launches fall back to the CUDA-core kernels. Host only.
 */
tq_status tq_test_reset_tensor_core_check(int force_fail);

/*
 * The fast attention kernel's shared-memory plan (host arithmetic only, no
 * CUDA call): for head_dim d (128 or 256), hw kv heads (4, 8 or 16) and nt
 * column tiles (1 or 2) per CTA, a paged (1) or contiguous (0) cache, a
 * device that reserves `reserved` bytes before the dynamic region and grants
 * `max_dyn` bytes of it.
 *   out  host, [8 + 4 * 8] int32 out: stages, warp groups, table offset,
 *        table bytes, header bytes, K / V / norm bytes per stage, then the
 *        offsets of the K, V, K-norm and V-norm buffers of stages 0..7 (-1
 *        past the last stage).
 * TQ_ERR_INVALID_ARG for out == NULL, TQ_ERR_UNSUPPORTED if the shape is not
 * the fast kernel's or no plan of at least two stages per group fits.
 */
tq_status tq_test_attend_plan(int d, int hw, int nt, int paged, int reserved, int max_dyn, int32_t* out);

#ifdef __cplusplus
}
#endif

#endif /* TQ_TEST_H_ */
