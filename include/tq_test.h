/*
 * tq_test.h -- test hooks of libtq. Not for production use.
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

#ifdef __cplusplus
}
#endif

#endif /* TQ_TEST_H_ */
