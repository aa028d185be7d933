// Internal definitions shared by the host code and the CUDA kernels of libtq.
// Not part of the public ABI (include/tq.h is).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "tq.h"

#define TQ_MAX_D 256
#define TQ_MAX_L 16
#define TQ_MAX_CELLS 272

// Codec tables, passed by value in every kernel launch (constant bank), so
// warp-uniform lookups (sign masks, levels) cost no registers or loads.
struct tq_codec_tables {
  // XOR mask for the fp16 pair (2k, 2k+1): bit 15 set <=> coordinate 2k is
  // negated, bit 31 set <=> coordinate 2k+1 is negated.
  uint32_t sign_h2[TQ_MAX_D / 2];
  // sign_h2[k] ^ sign_h2[k + 32], k < 32: the change of mask between the two
  // 64-coordinate halves of a head_dim-128 vector (a lane holding the upper
  // half applies it on top of the lower half's mask).
  uint32_t sign_h2_dx[32];
  // float32 sign masks per coordinate (bit 31 set <=> negated), and the
  // change between the two 64-coordinate halves of a head_dim-128 vector
  // (used by the offset + fp16-scale variant, which flips signs after
  // subtracting the offset in f32)
  uint32_t sign_f32[TQ_MAX_D];
  uint32_t sign_f32_dx[64];
  float levels[TQ_MAX_L];      // format levels c_k (2^-14 grid), ascending
  float bounds[TQ_MAX_L - 1];  // decision boundaries t_j in z units (2^-15 grid)
  // Encode quantizer lookup table, in "q units" q = z * inv_delta + q_offset:
  // cells are the unit intervals [n, n+1); each holds at most one boundary,
  // at least `margin` away from the cell edges.
  float tau[TQ_MAX_L - 1];  // boundaries in q units (exact in f32)
  float q_offset;           // q of z = 0 (an integer + a fraction)
  float inv_delta;          // 1/delta, a power of two
  float guard_q;            // half-width of the f64 recheck band, q units
  int lut_cells;            // number of cells (q in [0, lut_cells))
  // per cell: {bits of the boundary inside it (3e38 if none), count of
  // boundaries below the cell}; kernels replicate it into shared memory
  uint32_t cell[TQ_MAX_CELLS][2];
  int d;
  int bits;
};

struct tq_ctx {
  int d;
  int bits;
  uint64_t seed;
  double lloyd_max[TQ_MAX_L];  // unrounded fp64 Lloyd-Max levels
  tq_codec_tables t;
};

// Guard band of the encode quantizer in z units (N(0,1) scale). The f32 path
// decides every coordinate whose scaled rotated value is farther than this
// from a boundary; the f32 rounding error bound, u((log2 d + 1) sqrt(d) + 38)
// with u = 2^-24, is 5.6e-6 at head_dim 64, 7.7e-6 at 128 and 1.1e-5 at 256,
// below the band, so those decisions equal the exact ones. Closer
// coordinates are redone in fp64.
inline double tq_guard_z(int head_dim) { return head_dim <= 128 ? 1.0e-5 : 2.0e-5; }

// Kernel launchers (defined in the .cu files). Arguments are validated by the
// ABI layer before these are called.
tq_status tq_launch_encode(const tq_ctx* ctx, const void* x, int64_t n, void* packed, float* norms,
                           const int32_t* slot, int h, int64_t s_max, void* stream, int fault_inject,
                           int slot_abs = 0);
// Append of the K and V tensors of one step in one launch (tq_encode.cu):
// the same rows and caches as two tq_launch_encode append calls with the
// same context. TQ_ERR_UNSUPPORTED (nothing launched) when n is too large for
// one launch; the caller then makes the two calls.
tq_status tq_launch_encode_append2(const tq_ctx* ctx, const void* xk, const void* xv, int64_t n, void* k_packed,
                                  float* k_norms, void* v_packed, float* v_norms, const int32_t* slot, int h,
                                  int64_t s_max, void* stream);
// Bulk encode on the tensor cores (tq_encode_tc.cu): the same outputs as
// tq_launch_encode without append slots. tq_encode uses it from
// tq_encode_tc_min_rows() vectors on (one 128-vector tile per SM).
// TQ_ERR_UNSUPPORTED (nothing launched) when the kernel cannot be launched
// as planned; the caller then takes the CUDA-core kernel.
tq_status tq_launch_encode_tc(const tq_ctx* ctx, const void* x, int64_t n, void* packed, float* norms, void* stream,
                              int fault_inject);
int64_t tq_encode_tc_min_rows(void);
// Bulk decode on the tensor cores (tq_decode_tc.cu), head_dim <= 128: the same
// outputs as tq_launch_decode. TQ_ERR_UNSUPPORTED otherwise (then the CUDA-core
// kernel is used). tq_decode uses it from tq_encode_tc_min_rows() vectors on.
tq_status tq_launch_decode_tc(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x,
                              void* stream);
// The offset + fp16-scale variant of it: the same outputs as tq_launch_decode_os.
tq_status tq_launch_decode_tc_os(const tq_ctx* ctx, const void* packed, const uint32_t* side, int64_t n, void* x,
                                 void* stream);
tq_status tq_launch_encode_os(const tq_ctx* ctx, const void* x, int64_t n, void* packed, uint32_t* side,
                              void* stream);
tq_status tq_launch_decode_os(const tq_ctx* ctx, const void* packed, const uint32_t* side, int64_t n, void* x,
                              void* stream);
tq_status tq_launch_decode(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n,
                           void* x, void* stream);
tq_status tq_launch_attend(const tq_ctx* k, const tq_ctx* v, const void* q, int B, int hq, int hkv,
                           const void* k_packed, const float* k_norms, const void* v_packed,
                           const float* v_norms, int64_t s_max, const int32_t* positions, void* out,
                           void* workspace, size_t ws_bytes, void* stream);
tq_status tq_launch_attend_paged(const tq_ctx* k, const tq_ctx* v, const void* q, int B, int hq, int hkv,
                                 const void* k_cache, const float* k_norms, const void* v_cache,
                                 const float* v_norms, int64_t num_blocks, const int32_t* block_tables,
                                 int max_blocks, const int32_t* context_lens, void* out, void* workspace,
                                 size_t ws_bytes, void* stream);
size_t tq_attend_workspace_bytes_impl(int B, int hq, int head_dim, int64_t s_max);
// The fast attention kernel's shared-memory plan for head_dim d, hw kv heads
// and nt column tiles per CTA, a paged or contiguous cache, `reserved` bytes
// before the dynamic region and `max_dyn` bytes of it (host arithmetic only).
// out[0..7] = stages, warp groups, table offset, table bytes, header bytes,
// K / V / norm bytes per stage; out[8 + 8 k + s] = offset of buffer k (K, V,
// K norms, V norms) of stage s, -1 past the stages. False if no plan fits.
bool tq_attend_fast_plan(int d, int hw, int nt, int paged, int reserved, int max_dyn, int32_t* out);

// 1 if the tensor-core encode and decode kernels may run on the current
// device: the run-time check of the tensor core's rounding (tq_mma_check.cu)
// has passed there, running it first if it has not run yet (unless `stream`
// is being captured: then 0 without running it, so the call takes the
// CUDA-core kernel).
int tq_tensor_cores_usable(void* stream);
// Forget the current device's check result; force_fail != 0 makes the next
// check report a mismatch (used by the test hooks of libtq_test.so).
tq_status tq_tensor_core_check_reset(int force_fail);

// cuTensorMapEncodeTiled from the driver (cached; null if unavailable).
void* tq_tensor_map_encode_fn(void);

// Number of SMs of device `dev` (cached).
int tq_sm_count(int dev);

// Device error word of the current device (device pointer), and its reader.
uint32_t* tq_error_word(void);
tq_status tq_read_error_word(void* stream, uint32_t* bits);
