/*
 * tq.h -- TurboQuant KV-cache codec for NVIDIA B200 (sm_100a): C ABI.
 *
 * The codec follows the "aither-kvcache" project page (pypi.org), section
 * "Algorithm": each key or value vector of length head_dim is reduced to a
 * float32 L2 norm and a unit direction; the direction is rotated by a fixed,
 * data-oblivious random orthogonal map (here: a seeded +-1 sign flip followed
 * by the orthonormal Walsh-Hadamard transform, as in the "TurboQuant efficient
 * inference" post, section "What TurboQuant is"), each rotated coordinate is
 * scaled by sqrt(head_dim) and rounded to the nearest level of the Lloyd-Max
 * codebook for N(0,1) with 2^bits levels, and the indices are packed into a
 * little-endian bitstream. Decoding reverses every step. The fused decode-step
 * attention follows the same page, section "Zero-buffer fused attention":
 * rotate the query once, score and accumulate in the rotated domain, rotate
 * the output back once.
 *
 * Conventions for every call below:
 *  - Ownership: the caller allocates and frees all device memory. The library
 *    never allocates device memory and never frees caller memory. A context
 *    (tq_ctx) is a small host object; it is immutable after tq_create and may
 *    be shared by threads.
 *  - Execution: device work is enqueued asynchronously on `stream` (a
 *    cudaStream_t; NULL = the legacy default stream) of the current device.
 *    Argument validation happens on the host before anything is enqueued; on
 *    any error nothing is enqueued. The encode and decode kernels are
 *    launched with programmatic stream serialisation: a kernel may start its
 *    set-up (shared and tensor memory only) while the previous kernel of the
 *    stream is finishing, and touches global memory only after that kernel
 *    has completed, so stream order holds for every buffer.
 *  - Layout: fp16 data is IEEE binary16 stored as uint16; every tensor is
 *    dense row-major; leading dimensions are flattened, so any [..., d] tensor
 *    is `n` rows.
 *  - Alignment: device pointers to fp16 rows and packed rows must be 16-byte
 *    aligned; float pointers 4-byte aligned; int32 pointers 4-byte aligned.
 *  - NaN or Inf input gives unspecified codes (never an out-of-bounds access).
 *  - Device-side faults found by a kernel (a wait that ran out, an index out
 *    of range) are recorded in a device error word; read it with
 *    tq_device_error().
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_ctx tq_ctx;
typedef void* tq_stream; /* cudaStream_t */

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1, /* bad size, null pointer, hq % hkv != 0 ... */
  TQ_ERR_UNSUPPORTED = 2, /* head_dim not in {64,128,256} or bits not in {2,3,4} */
  TQ_ERR_ALIGNMENT = 3,   /* a pointer violates the alignment rule above */
  TQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
  TQ_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  TQ_ERR_TIMEOUT = 6,     /* a device-side bounded wait ran out */
  TQ_ERR_NOMEM = 7,       /* host allocation failed */
  TQ_ERR_DEVICE = 8       /* a kernel recorded an out-of-range index */
} tq_status;

/* Bits of the device error word (tq_device_error). */
#define TQ_DEVERR_TIMEOUT 0x1u     /* an mbarrier wait ran out; the kernel returned early */
#define TQ_DEVERR_SLOT_RANGE 0x2u  /* tq_encode_append: a slot outside [0, s_max) was skipped */
#define TQ_DEVERR_POS_RANGE 0x4u   /* tq_attend_decode: a position > s_max was clamped */
#define TQ_DEVERR_SMEM_LAYOUT 0x8u /* tq_attend_decode: shared memory not where the launch planned it; no output */
#define TQ_DEVERR_BLOCK_RANGE 0x10u /* tq_attend_decode_paged: a block number outside [0, num_blocks) was clamped */

/* Human-readable name of a status. Never NULL. */
const char* tq_status_string(tq_status s);

/*
 * Create a codec context ("aither-kvcache", section "API Reference":
 * TurboQuant(head_dim, bits, seed=42)).
 *   head_dim: 64, 128 or 256.   bits: 2, 3 or 4.
 *   seed: seed of the splitmix64 stream whose i-th output (bit 63) gives the
 *         sign of coordinate i.
 * Builds, on the host only, the Lloyd-Max codebook for N(0,1) (fp64 Lloyd
 * iteration, then levels rounded to the 2^-14 grid; boundaries are midpoints
 * of the rounded levels) and the sign table. Touches no GPU.
 * Returns TQ_ERR_UNSUPPORTED, TQ_ERR_INVALID_ARG (out == NULL) or
 * TQ_ERR_NOMEM; *out is set only on TQ_OK.
 */
tq_status tq_create(int head_dim, int bits, uint64_t seed, tq_ctx** out);

/* Free a context. NULL is ignored. The caller must not use it afterwards. */
void tq_destroy(tq_ctx* ctx);

/* Parameters of a context (for serialisation: a packed cache is decodable by
 * any context created with the same three values). 0 for NULL. */
int tq_head_dim(const tq_ctx* ctx);
int tq_bits(const tq_ctx* ctx);
uint64_t tq_seed(const tq_ctx* ctx);

/* Packed bytes per vector, head_dim * bits / 8 ("aither-kvcache", "Quick
 * Start -- TurboQuant": 128 fp16 -> 64 uint8 at 4 bits). 0 for NULL. */
size_t tq_packed_bytes(const tq_ctx* ctx);

/*
 * Copy the context's tables to host memory (any of the pointers may be NULL):
 *   levels[2^bits]      ascending float32 codebook levels (N(0,1) units),
 *   boundaries[2^bits-1] float32 decision boundaries,
 *   sign_bits[head_dim/8] bit i set <=> sign of coordinate i is -1
 *                        (bit i%8 of byte i/8).
 * Host only. TQ_ERR_INVALID_ARG for a NULL context.
 */
tq_status tq_get_tables(const tq_ctx* ctx, float* levels, float* boundaries, uint8_t* sign_bits);

/*
 * Encode n vectors ("aither-kvcache", section "Algorithm", steps 1-5).
 *   x_f16   device, [n, head_dim] fp16, 16-byte aligned.
 *   packed  device, [n, tq_packed_bytes] uint8 out, 16-byte aligned;
 *           code i of a row occupies stream bits [i*bits, i*bits+bits),
 *           stream bit k = bit (k mod 8) of byte k/8.
 *   norms   device, [n] float32 out: the L2 norm of each input row.
 * Codes are those of exact arithmetic (coordinates within a proven f32 error
 * band of a decision boundary are redone in fp64); norms are within 1e-6 of
 * the exact norm of the fp16 row (relative; both kernels sum the squares in
 * f32 on the CUDA cores). Launches of at least 128 x SM-count vectors run
 * on the tensor cores (the 16-point Hadamard blocks as tcgen05 MMAs), smaller
 * ones on the CUDA cores; both give the same codes, norms may differ in the
 * last bits.
 * n == 0 is a no-op (pointers may then be NULL). Inputs and outputs must not
 * overlap. The call is asynchronous on `stream`.
 */
tq_status tq_encode(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, float* norms,
                    tq_stream stream);

/*
 * Decode n vectors ("aither-kvcache", section "Algorithm": decoding reverses
 * steps 4-1): x_hat = norm * D H (c[idx] / sqrt(head_dim)), rounded to fp16.
 *   packed  device, [n, tq_packed_bytes] uint8, 16-byte aligned.
 *   norms   device, [n] float32.
 *   x_f16   device, [n, head_dim] fp16 out, 16-byte aligned.
 * H c is summed exactly; the only roundings are the product by
 * norm / head_dim and the fp16 conversion. A decoded coordinate whose
 * magnitude rounds above 65504 (possible for rows whose norm is near the
 * fp16 range, e.g. entries near +-65504) becomes +-Inf, as an fp16
 * conversion of that value does. Launches of at least
 * 128 x SM-count vectors at head_dim 64 and 128 run on the tensor cores (the
 * 32-point Hadamard blocks as tcgen05 MMAs with A in tensor memory, the
 * remaining stages as f32 butterflies), other launches on the CUDA cores;
 * the outputs are bit-identical.
 * n == 0 is a no-op. Asynchronous on `stream`.
 */
tq_status tq_decode(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x_f16,
                    tq_stream stream);

/*
 * Streaming append ("aither-kvcache", section "Custom inference loop": encode
 * where the cache is written): encode one new token per sequence into a
 * preallocated packed cache.
 *   x_f16        device, [n_seq, h, head_dim] fp16, 16-byte aligned.
 *   cache_packed device, [n_seq, s_max, h, tq_packed_bytes] uint8, 16-byte aligned.
 *   cache_norms  device, [n_seq, s_max, h] float32.
 *   slot         device, [n_seq] int32: the cache position written for each
 *                sequence. A slot outside [0, s_max) is skipped and flagged
 *                with TQ_DEVERR_SLOT_RANGE.
 * The codes written are bit-identical to tq_encode of the same rows.
 */
tq_status tq_encode_append(const tq_ctx* ctx, const void* x_f16, int n_seq, int h, void* cache_packed,
                           float* cache_norms, int64_t s_max, const int32_t* slot, tq_stream stream);

/*
 * tq_encode_append for the key and the value of the new token of every
 * sequence in one launch (an addition of this library: the "aither-kvcache"
 * page's custom inference loop writes K and V at each step; a decode step of
 * a few thousand rows is bound by launch latency, so one launch instead of
 * two shortens the step). The result is that of
 *   tq_encode_append(ctx, k_f16, n_seq, h, k_cache, k_norms, s_max, slot, stream);
 *   tq_encode_append(ctx, v_f16, n_seq, h, v_cache, v_norms, s_max, slot, stream);
 * with one context for both tensors (same head_dim, bits and seed); for two
 * different codecs make the two calls. Arguments, layouts, alignment rules
 * and errors as tq_encode_append, for each tensor; the two caches must not
 * overlap. Asynchronous on `stream`.
 */
tq_status tq_encode_append_kv(const tq_ctx* ctx, const void* k_f16, const void* v_f16, int n_seq, int h,
                              void* k_cache, float* k_norms, void* v_cache, float* v_norms, int64_t s_max,
                              const int32_t* slot, tq_stream stream);

/*
 * The offset + half-precision-scale variant ("TurboQuant efficient
 * inference", section "1. The quantizer": remove a small per-vector offset,
 * rotate, round each coordinate to a level, keep one scale alongside; codes
 * packed two per byte at 4 bits, scales in half precision). Per vector:
 * offset mu16 = fp16(mean(x)) (the mean accumulated in f32), y = x - mu16,
 * scale n16 = fp16(||y||); the codes are those of tq_encode applied to y
 * with n16 in place of the norm (decided exactly, as tq_encode's).
 *   packed  device, [n, tq_packed_bytes] uint8 out (same layout as tq_encode).
 *   side    device, [n] uint32 out: fp16 bits of mu16 | fp16 bits of n16 << 16.
 * A constant vector gets scale 0 and decodes to itself; a vector with
 * ||x - mean|| above the fp16 range gets an infinite scale and an
 * unspecified decode. Asynchronous on `stream`.
 */
tq_status tq_encode_os(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, uint32_t* side,
                       tq_stream stream);

/*
 * Decode of the offset variant: x_hat = mu16 + (n16 / head_dim) D H_pm c[idx]
 * (H_pm the +-1 Walsh-Hadamard matrix), computed in f32 (a product and a sum
 * of the offset, each rounded once) and rounded to fp16.
 *   packed, side as written by tq_encode_os; x_f16 device [n, head_dim] out.
 * Launches of at least 128 x SM-count vectors at head_dim 64 and 128 run on
 * the tensor cores (as tq_decode), other launches on the CUDA cores; the
 * outputs are bit-identical. Asynchronous on `stream`.
 */
tq_status tq_decode_os(const tq_ctx* ctx, const void* packed, const uint32_t* side, int64_t n, void* x_f16,
                       tq_stream stream);

/*
 * Encode-on-write into a paged cache ("aither-kvcache", section "Custom
 * inference loop": encode where the K/V of new tokens are written; the
 * slot-mapping form of serving engines): token t of x is encoded and written
 * to slot slot_mapping[t] of a pool of num_slots slots.
 *   x_f16        device, [n_tok, h, d] fp16, 16-byte aligned.
 *   cache_packed device, [num_slots, h, P] uint8, 16-byte aligned; the pool
 *                of tq_attend_decode_paged is [num_blocks, TQ_PAGE_BLOCK, h,
 *                P], i.e. num_slots = num_blocks * TQ_PAGE_BLOCK with slot =
 *                block * TQ_PAGE_BLOCK + offset.
 *   cache_norms  device, [num_slots, h] float32.
 *   slot_mapping device, [n_tok] int32. A negative slot (a padding token)
 *                is skipped; a slot >= num_slots is skipped and flagged with
 *                TQ_DEVERR_SLOT_RANGE.
 * Rows of other slots are not touched. The codes written are bit-identical
 * to tq_encode of the same rows.
 */
tq_status tq_encode_slots(const tq_ctx* ctx, const void* x_f16, int64_t n_tok, int h, void* cache_packed,
                          float* cache_norms, int64_t num_slots, const int32_t* slot_mapping, tq_stream stream);

/*
 * Workspace (device bytes) that tq_attend_decode needs for a batch of B
 * sequences, hq query heads, head_dim and caches of s_max positions: the
 * split-S partial results (running max, sum and rotated accumulator per
 * split). 0 for invalid sizes.
 */
size_t tq_attend_workspace_bytes(int B, int hq, int head_dim, int64_t s_max);

/*
 * One decode step of attention over packed K/V caches, without decoding them
 * ("aither-kvcache", section "Zero-buffer fused attention"; "TurboQuant
 * efficient inference", section "2. A fused decode path"):
 *   o[b,h] = sum_t softmax_t(q[b,h] . k_hat[b,t,g(h)] / sqrt(d)) v_hat[b,t,g(h)]
 * over t < positions[b], where g(h) = h / (hq / hkv) and k_hat, v_hat are the
 * decoded cache rows. Computed as q~ = H D_K q once per head, scores
 * (n_t / d) (1/sqrt(d)) q~ . c_K[idx_t], an accumulator of n_t c_V[idx_t] in
 * the rotated domain, and o = D_V H acc / d at the end.
 *   k, v        contexts of the key and value caches (same head_dim).
 *   q_f16       device, [B, hq, d] fp16, 16-byte aligned.
 *   k_packed    device, [B, s_max, hkv, Pk] uint8, 16-byte aligned.
 *   k_norms     device, [B, s_max, hkv] float32.  (v likewise, Pv bytes)
 *   positions   device, [B] int32: number of valid cache positions per
 *               sequence. <= 0 gives a zero output row; > s_max is clamped
 *               and flagged with TQ_DEVERR_POS_RANGE.
 *   out_f16     device, [B, hq, d] fp16 out, 16-byte aligned.
 *   workspace   device scratch of at least
 *               tq_attend_workspace_bytes(B, hq, d, s_max) bytes, 16-byte
 *               aligned; its contents on entry do not matter.
 * Asynchronous on `stream`; calls that share a workspace must not overlap.
 */
tq_status tq_attend_decode(const tq_ctx* k, const tq_ctx* v, const void* q_f16, int B, int hq, int hkv,
                           const void* k_packed, const float* k_norms, const void* v_packed,
                           const float* v_norms, int64_t s_max, const int32_t* positions, void* out_f16,
                           void* workspace, size_t ws_bytes, tq_stream stream);

/*
 * tq_attend_decode over a paged cache ("aither-kvcache", sections "Paged KV
 * cache" and "API Reference": TQPagedAttention's block_tables and
 * context_lens): the cache is a pool of blocks of TQ_PAGE_BLOCK positions,
 * and each sequence lists the blocks that hold its positions in order.
 *   k_cache     device, [num_blocks, TQ_PAGE_BLOCK, hkv, Pk] uint8, 16-byte
 *               aligned.
 *   k_norms     device, [num_blocks, TQ_PAGE_BLOCK, hkv] float32. (v likewise)
 *   block_tables device, [B, max_blocks] int32: entry j of row b is the
 *               block holding positions [16 j, 16 j + 16) of sequence b.
 *               Entries past the sequence's context are not read; an entry
 *               outside [0, num_blocks) that is read is clamped and flagged
 *               with TQ_DEVERR_BLOCK_RANGE.
 *   context_lens device, [B] int32: valid positions per sequence, as
 *               `positions` of tq_attend_decode with s_max = max_blocks * 16.
 *   workspace   at least tq_attend_workspace_bytes(B, hq, d, max_blocks * 16).
 * Other arguments, results and errors as tq_attend_decode; with an identity
 * block table over a [B, S, hkv, P] cache (S a multiple of 16) the output is
 * bit-identical to tq_attend_decode's.
 */
#define TQ_PAGE_BLOCK 16
tq_status tq_attend_decode_paged(const tq_ctx* k, const tq_ctx* v, const void* q_f16, int B, int hq, int hkv,
                                 const void* k_cache, const float* k_norms, const void* v_cache,
                                 const float* v_norms, int64_t num_blocks, const int32_t* block_tables,
                                 int max_blocks, const int32_t* context_lens, void* out_f16, void* workspace,
                                 size_t ws_bytes, tq_stream stream);

/*
 * No counterpart in the paper: an addition of this library.
 *
 * tq_attend_decode for callers that cannot allocate device memory -- for
 * example a plugin inside a serving framework that owns every byte of device
 * memory through its own pool, or a decode loop that must not risk a
 * device-synchronising or failing cudaMalloc in the middle of a generation.
 * Same arguments, layouts, alignment rules and results as tq_attend_decode,
 * without the workspace: the split-S scratch is a fixed array of
 * TQ_ATTEND_STATIC_SCRATCH_BYTES in device memory that belongs to the
 * library (one per device that loads it, kept until the process exits). The
 * call allocates nothing.
 *  - Returns TQ_ERR_WORKSPACE, without enqueuing anything, when the scratch
 *    this call needs, tq_attend_workspace_bytes(B, hq, head_dim, s_max), is
 *    larger than TQ_ATTEND_STATIC_SCRATCH_BYTES.
 *  - The first call on a device looks up the array's device address for that
 *    device (with the device current); make that first call before any
 *    stream capture.
 *  - Every call on a device shares the one array, and the array keeps what
 *    the last call left there (each call overwrites every entry it reads).
 *    Calls that overlap on the GPU -- on different streams, or from host
 *    threads that do not order their streams -- race on it.
 */
#define TQ_ATTEND_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
tq_status tq_attend_decode_static(const tq_ctx* k, const tq_ctx* v, const void* q_f16, int B, int hq, int hkv,
                                  const void* k_packed, const float* k_norms, const void* v_packed,
                                  const float* v_norms, int64_t s_max, const int32_t* positions, void* out_f16,
                                  tq_stream stream);

/*
 * Check, on the current device, the tensor-core arithmetic that the bulk
 * encode and decode kernels rely on, and report the result (an addition of
 * this library; the pages have no tensor-core path). The exactness of the
 * tensor-core encode's codes outside its guard band, and of the tensor-core
 * decode, rests on a rounding model of tcgen05.mma kind::f16 with f32
 * accumulation that NVIDIA does not document (products exact, addends cut at
 * 2^(E-25) below the largest addend's exponent E, the sum rounded toward
 * zero). The check runs one MMA on a table that tells that model from its
 * neighbours and compares every output on the device.
 *   passed  host out: 1 if the device follows the model (bulk launches of
 *           tq_encode and tq_decode run on the tensor cores), 0 if not (they
 *           run on the CUDA cores, with the same codes and decoded values).
 * The check runs once per device and process, on a stream of its own, and
 * this call waits for it. tq_encode and tq_decode run it themselves before
 * their first bulk launch on a device (that call then waits too), except
 * while their stream is being captured into a CUDA graph: such a call takes
 * the CUDA-core kernel. Call this once per device before capturing bulk
 * encodes or decodes. TQ_ERR_CUDA if a CUDA call of the check failed.
 */
tq_status tq_tensor_core_check(int* passed);

/*
 * Read and clear the device error word of the current device (a bitwise OR
 * of TQ_DEVERR_* set by kernels since the last call). Synchronises `stream`.
 * Returns TQ_ERR_TIMEOUT if TQ_DEVERR_TIMEOUT was set, TQ_ERR_DEVICE if
 * another bit was set, else TQ_OK; *bits (optional) receives the word.
 * There is one word per device, shared by every context, stream and host
 * thread of the process that uses the library on that device: a call
 * reports what any kernel of the library on that device recorded, and
 * clears it for every other user too. Kernels still running on other
 * streams may set bits after the read.
 */
tq_status tq_device_error(tq_stream stream, uint32_t* bits);

/*
 * The same query in the form a caller holding a context uses after it has
 * synchronised its stream(s): reads and clears the error word of the current
 * device (the word is per device, not per context: the context is only
 * validated). Returns TQ_ERR_INVALID_ARG for a NULL context, TQ_ERR_TIMEOUT
 * if TQ_DEVERR_TIMEOUT was set, TQ_ERR_DEVICE if another bit was set, else
 * TQ_OK. It synchronises the legacy default stream before the read.
 */
tq_status tq_check_device_error(const tq_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
