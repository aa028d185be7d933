// Host side of libtq: context creation (codebook, sign table, quantizer
// lookup parameters), argument validation and the exported C ABI.
//
// The codebook is the Lloyd-Max quantizer for N(0,1) ("aither-kvcache" PyPI
// page, section "Algorithm", step 3; "TurboQuant efficient inference", section
// "What TurboQuant is": levels computed from the bell-curve density, no
// calibration data). It is built here in fp64 on the positive half-line (the
// density is symmetric, so the middle boundary is 0 and the negative levels
// mirror the positive ones), then rounded to the 2^-14 grid.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>

#include "tq_internal.h"

namespace {

const double kInvSqrt2 = 0.70710678118654752440;
const double kInvSqrt2Pi = 0.39894228040143267794;

// Upper tail P(X >= x) of N(0,1); 0 at +inf.
double upper_tail(double x) { return std::isinf(x) ? 0.0 : 0.5 * std::erfc(x * kInvSqrt2); }
// Standard normal density; 0 at +inf.
double density(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }

// Positive half of the Lloyd-Max codebook with 2*m levels: on [0, inf) the
// cells are [b_0 = 0, b_1), ..., [b_{m-1}, inf) with b_k the midpoints of the
// neighbouring levels; each level is the mean of X over its cell. Iterated to
// a fixed point (the optimum is unique for a log-concave density).
void lloyd_max_positive(int m, double* level) {
  for (int k = 0; k < m; ++k) level[k] = 3.0 * (k + 0.5) / m;  // start: uniform on [0, 3]
  double b[TQ_MAX_L / 2 + 1];
  for (int it = 0; it < 1000000; ++it) {
    b[0] = 0.0;
    for (int k = 1; k < m; ++k) b[k] = 0.5 * (level[k - 1] + level[k]);
    b[m] = INFINITY;
    double moved = 0.0;
    for (int k = 0; k < m; ++k) {
      const double mass = upper_tail(b[k]) - upper_tail(b[k + 1]);
      const double mean = (density(b[k]) - density(b[k + 1])) / mass;
      moved = std::fmax(moved, std::fabs(mean - level[k]));
      level[k] = mean;
    }
    if (moved < 1e-15) break;
  }
}

uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Choose the quantizer lookup grid: cells of width delta = 2^-e (z units),
// each holding at most one boundary, at least `margin` (in cell units) from
// both cell edges, with a fractional offset f of the cell grid.
bool choose_grid(const float* bounds, int nb, double* delta_out, double* frac_out) {
  double min_gap = INFINITY;
  for (int j = 1; j < nb; ++j) min_gap = std::fmin(min_gap, (double)bounds[j] - bounds[j - 1]);
  for (int e = 0; e <= 6; ++e) {
    const double delta = std::ldexp(1.0, -e);
    if (!(min_gap > delta)) continue;
    double best = -1.0, best_f = 0.0;
    for (int k = 0; k < 16; ++k) {
      const double f = k / 16.0;
      double margin = 1.0;
      for (int j = 0; j < nb; ++j) {
        const double q = bounds[j] / delta + f;
        const double fr = q - std::floor(q);
        margin = std::fmin(margin, std::fmin(fr, 1.0 - fr));
      }
      if (margin > best) {
        best = margin;
        best_f = f;
      }
    }
    if (best >= 1.0 / 64.0) {
      *delta_out = delta;
      *frac_out = best_f;
      return true;
    }
  }
  return false;
}

bool valid_dims(int d, int bits) { return (d == 64 || d == 128 || d == 256) && bits >= 2 && bits <= 4; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" {

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_ALIGNMENT: return "TQ_ERR_ALIGNMENT";
    case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
    case TQ_ERR_NOMEM: return "TQ_ERR_NOMEM";
    case TQ_ERR_DEVICE: return "TQ_ERR_DEVICE";
  }
  return "TQ_ERR_UNKNOWN";
}

tq_status tq_create(int head_dim, int bits, uint64_t seed, tq_ctx** out) {
  if (!out) return TQ_ERR_INVALID_ARG;
  if (!valid_dims(head_dim, bits)) return TQ_ERR_UNSUPPORTED;
  tq_ctx* c = new (std::nothrow) tq_ctx;
  if (!c) return TQ_ERR_NOMEM;
  std::memset(c, 0, sizeof(*c));
  c->d = head_dim;
  c->bits = bits;
  c->seed = seed;
  const int L = 1 << bits, m = L / 2;

  double pos[TQ_MAX_L / 2];
  lloyd_max_positive(m, pos);
  for (int k = 0; k < m; ++k) {
    c->lloyd_max[m + k] = pos[k];
    c->lloyd_max[m - 1 - k] = -pos[k];
  }
  tq_codec_tables& t = c->t;
  t.d = head_dim;
  t.bits = bits;
  // levels on the 2^-14 grid (exact in f32), boundaries their midpoints (2^-15 grid)
  for (int k = 0; k < L; ++k) t.levels[k] = (float)(std::nearbyint(std::ldexp(c->lloyd_max[k], 14)) / 16384.0);
  for (int j = 0; j < L - 1; ++j) t.bounds[j] = 0.5f * (t.levels[j] + t.levels[j + 1]);

  uint64_t state = seed;
  for (int i = 0; i < head_dim; i += 2) {
    const uint64_t a = splitmix64_next(state), b = splitmix64_next(state);
    t.sign_h2[i / 2] = ((a >> 63) ? 0x8000u : 0u) | ((b >> 63) ? 0x80000000u : 0u);
  }
  for (int k = 0; k < 32 && k + 32 < head_dim / 2; ++k) t.sign_h2_dx[k] = t.sign_h2[k] ^ t.sign_h2[k + 32];
  for (int i = 0; i < head_dim; ++i) t.sign_f32[i] = ((t.sign_h2[i / 2] >> (15 + 16 * (i & 1))) & 1u) << 31;
  for (int i = 0; i < 64 && i + 64 < head_dim; ++i) t.sign_f32_dx[i] = t.sign_f32[i] ^ t.sign_f32[i + 64];

  double delta = 0.0, frac = 0.0;
  if (!choose_grid(t.bounds, L - 1, &delta, &frac)) {
    delete c;
    return TQ_ERR_UNSUPPORTED;
  }
  const int K = (int)std::ceil(std::sqrt((double)head_dim) / delta) + 2;
  t.inv_delta = (float)(1.0 / delta);
  t.q_offset = (float)(K + frac);
  t.lut_cells = 2 * K + 2;
  t.guard_q = (float)(tq_guard_z(head_dim) / delta);
  for (int j = 0; j < L - 1; ++j) t.tau[j] = (float)(t.bounds[j] / delta + (K + frac));
  if (t.lut_cells > TQ_MAX_CELLS) {
    delete c;
    return TQ_ERR_UNSUPPORTED;
  }
  for (int cell = 0; cell < t.lut_cells; ++cell) {
    uint32_t below = 0;
    float thr = 3.0e38f;  // no boundary in this cell
    for (int j = 0; j < L - 1; ++j) {
      if (t.tau[j] < (float)cell)
        ++below;
      else if (t.tau[j] < (float)(cell + 1))
        thr = t.tau[j];
    }
    uint32_t tb;
    std::memcpy(&tb, &thr, 4);
    t.cell[cell][0] = tb;
    t.cell[cell][1] = below;
  }
  *out = c;
  return TQ_OK;
}

void tq_destroy(tq_ctx* ctx) { delete ctx; }

int tq_head_dim(const tq_ctx* ctx) { return ctx ? ctx->d : 0; }
int tq_bits(const tq_ctx* ctx) { return ctx ? ctx->bits : 0; }
uint64_t tq_seed(const tq_ctx* ctx) { return ctx ? ctx->seed : 0; }
size_t tq_packed_bytes(const tq_ctx* ctx) { return ctx ? (size_t)ctx->d * ctx->bits / 8 : 0; }

tq_status tq_get_tables(const tq_ctx* ctx, float* levels, float* boundaries, uint8_t* sign_bits) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  const int L = 1 << ctx->bits;
  if (levels)
    for (int k = 0; k < L; ++k) levels[k] = ctx->t.levels[k];
  if (boundaries)
    for (int j = 0; j < L - 1; ++j) boundaries[j] = ctx->t.bounds[j];
  if (sign_bits) {
    std::memset(sign_bits, 0, (size_t)ctx->d / 8);
    for (int i = 0; i < ctx->d; ++i) {
      const uint32_t w = ctx->t.sign_h2[i / 2];
      const uint32_t neg = (i & 1) ? (w >> 31) & 1u : (w >> 15) & 1u;
      sign_bits[i / 8] |= (uint8_t)(neg << (i % 8));
    }
  }
  return TQ_OK;
}

tq_status tq_encode(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, float* norms,
                    tq_stream stream) {
  if (!ctx || n < 0) return TQ_ERR_INVALID_ARG;
  if (n == 0) return TQ_OK;
  if (!x_f16 || !packed || !norms) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(norms, 4)) return TQ_ERR_ALIGNMENT;
  if (n >= tq_encode_tc_min_rows() && tq_tensor_cores_usable(stream)) {
    const tq_status st = tq_launch_encode_tc(ctx, x_f16, n, packed, norms, stream, 0);
    if (st != TQ_ERR_UNSUPPORTED) return st;
  }
  return tq_launch_encode(ctx, x_f16, n, packed, norms, nullptr, 1, 1, stream, 0);
}

tq_status tq_decode(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x_f16,
                    tq_stream stream) {
  if (!ctx || n < 0) return TQ_ERR_INVALID_ARG;
  if (n == 0) return TQ_OK;
  if (!x_f16 || !packed || !norms) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(norms, 4)) return TQ_ERR_ALIGNMENT;
  if (n >= tq_encode_tc_min_rows() && tq_tensor_cores_usable(stream)) {
    // the tensor-core kernel at head_dim <= 128
    const tq_status st = tq_launch_decode_tc(ctx, packed, norms, n, x_f16, stream);
    if (st != TQ_ERR_UNSUPPORTED) return st;
  }
  return tq_launch_decode(ctx, packed, norms, n, x_f16, stream);
}

tq_status tq_encode_append(const tq_ctx* ctx, const void* x_f16, int n_seq, int h, void* cache_packed,
                           float* cache_norms, int64_t s_max, const int32_t* slot, tq_stream stream) {
  if (!ctx || n_seq < 0 || h <= 0 || s_max <= 0) return TQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TQ_OK;
  if (!x_f16 || !cache_packed || !cache_norms || !slot) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(cache_packed, 16) || !aligned(cache_norms, 4) || !aligned(slot, 4))
    return TQ_ERR_ALIGNMENT;
  return tq_launch_encode(ctx, x_f16, (int64_t)n_seq * h, cache_packed, cache_norms, slot, h, s_max, stream, 0);
}

tq_status tq_encode_append_kv(const tq_ctx* ctx, const void* k_f16, const void* v_f16, int n_seq, int h,
                              void* k_cache, float* k_norms, void* v_cache, float* v_norms, int64_t s_max,
                              const int32_t* slot, tq_stream stream) {
  if (!ctx || n_seq < 0 || h <= 0 || s_max <= 0) return TQ_ERR_INVALID_ARG;
  if (n_seq == 0) return TQ_OK;
  if (!k_f16 || !v_f16 || !k_cache || !k_norms || !v_cache || !v_norms || !slot) return TQ_ERR_INVALID_ARG;
  if (!aligned(k_f16, 16) || !aligned(v_f16, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(k_norms, 4) || !aligned(v_norms, 4) || !aligned(slot, 4))
    return TQ_ERR_ALIGNMENT;
  const int64_t n = (int64_t)n_seq * h;
  const tq_status st =
      tq_launch_encode_append2(ctx, k_f16, v_f16, n, k_cache, k_norms, v_cache, v_norms, slot, h, s_max, stream);
  if (st != TQ_ERR_UNSUPPORTED) return st;
  const tq_status sk = tq_launch_encode(ctx, k_f16, n, k_cache, k_norms, slot, h, s_max, stream, 0);
  if (sk != TQ_OK) return sk;
  return tq_launch_encode(ctx, v_f16, n, v_cache, v_norms, slot, h, s_max, stream, 0);
}

tq_status tq_encode_os(const tq_ctx* ctx, const void* x_f16, int64_t n, void* packed, uint32_t* side,
                       tq_stream stream) {
  if (!ctx || n < 0) return TQ_ERR_INVALID_ARG;
  if (n == 0) return TQ_OK;
  if (!x_f16 || !packed || !side) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(side, 4)) return TQ_ERR_ALIGNMENT;
  return tq_launch_encode_os(ctx, x_f16, n, packed, side, stream);
}

tq_status tq_decode_os(const tq_ctx* ctx, const void* packed, const uint32_t* side, int64_t n, void* x_f16,
                       tq_stream stream) {
  if (!ctx || n < 0) return TQ_ERR_INVALID_ARG;
  if (n == 0) return TQ_OK;
  if (!x_f16 || !packed || !side) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(packed, 16) || !aligned(side, 4)) return TQ_ERR_ALIGNMENT;
  if (n >= tq_encode_tc_min_rows() && tq_tensor_cores_usable(stream)) {
    // the tensor-core kernel at head_dim <= 128, as tq_decode
    const tq_status st = tq_launch_decode_tc_os(ctx, packed, side, n, x_f16, stream);
    if (st != TQ_ERR_UNSUPPORTED) return st;
  }
  return tq_launch_decode_os(ctx, packed, side, n, x_f16, stream);
}

tq_status tq_encode_slots(const tq_ctx* ctx, const void* x_f16, int64_t n_tok, int h, void* cache_packed,
                          float* cache_norms, int64_t num_slots, const int32_t* slot_mapping, tq_stream stream) {
  if (!ctx || n_tok < 0 || h <= 0 || num_slots <= 0) return TQ_ERR_INVALID_ARG;
  if (n_tok == 0) return TQ_OK;
  if (!x_f16 || !cache_packed || !cache_norms || !slot_mapping) return TQ_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(cache_packed, 16) || !aligned(cache_norms, 4) || !aligned(slot_mapping, 4))
    return TQ_ERR_ALIGNMENT;
  return tq_launch_encode(ctx, x_f16, n_tok * h, cache_packed, cache_norms, slot_mapping, h, num_slots, stream, 0, 1);
}

size_t tq_attend_workspace_bytes(int B, int hq, int head_dim, int64_t s_max) {
  if (B <= 0 || hq <= 0 || s_max <= 0 || !(head_dim == 64 || head_dim == 128 || head_dim == 256)) return 0;
  return tq_attend_workspace_bytes_impl(B, hq, head_dim, s_max);
}

tq_status tq_attend_decode(const tq_ctx* k, const tq_ctx* v, const void* q_f16, int B, int hq, int hkv,
                           const void* k_packed, const float* k_norms, const void* v_packed,
                           const float* v_norms, int64_t s_max, const int32_t* positions, void* out_f16,
                           void* workspace, size_t ws_bytes, tq_stream stream) {
  if (!k || !v) return TQ_ERR_INVALID_ARG;
  if (k->d != v->d) return TQ_ERR_INVALID_ARG;
  if (B < 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || s_max <= 0) return TQ_ERR_INVALID_ARG;
  if (B == 0) return TQ_OK;
  if (!q_f16 || !k_packed || !k_norms || !v_packed || !v_norms || !positions || !out_f16)
    return TQ_ERR_INVALID_ARG;
  if (!aligned(q_f16, 16) || !aligned(k_packed, 16) || !aligned(v_packed, 16) || !aligned(out_f16, 16) ||
      !aligned(k_norms, 4) || !aligned(v_norms, 4) || !aligned(positions, 4))
    return TQ_ERR_ALIGNMENT;
  const size_t need = tq_attend_workspace_bytes(B, hq, k->d, s_max);
  if (need == 0) return TQ_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < need) return TQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return TQ_ERR_ALIGNMENT;
  return tq_launch_attend(k, v, q_f16, B, hq, hkv, k_packed, k_norms, v_packed, v_norms, s_max, positions,
                          out_f16, workspace, ws_bytes, stream);
}

tq_status tq_attend_decode_paged(const tq_ctx* k, const tq_ctx* v, const void* q_f16, int B, int hq, int hkv,
                                 const void* k_cache, const float* k_norms, const void* v_cache,
                                 const float* v_norms, int64_t num_blocks, const int32_t* block_tables,
                                 int max_blocks, const int32_t* context_lens, void* out_f16, void* workspace,
                                 size_t ws_bytes, tq_stream stream) {
  if (!k || !v) return TQ_ERR_INVALID_ARG;
  if (k->d != v->d) return TQ_ERR_INVALID_ARG;
  if (B < 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || num_blocks <= 0 || max_blocks <= 0)
    return TQ_ERR_INVALID_ARG;
  if (num_blocks > ((int64_t)1 << 26)) return TQ_ERR_UNSUPPORTED;  // cache rows stay below 2^30
  if (B == 0) return TQ_OK;
  if (!q_f16 || !k_cache || !k_norms || !v_cache || !v_norms || !block_tables || !context_lens || !out_f16)
    return TQ_ERR_INVALID_ARG;
  if (!aligned(q_f16, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out_f16, 16) ||
      !aligned(k_norms, 4) || !aligned(v_norms, 4) || !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return TQ_ERR_ALIGNMENT;
  const int64_t s_max = (int64_t)max_blocks * TQ_PAGE_BLOCK;
  const size_t need = tq_attend_workspace_bytes(B, hq, k->d, s_max);
  if (need == 0) return TQ_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < need) return TQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return TQ_ERR_ALIGNMENT;
  return tq_launch_attend_paged(k, v, q_f16, B, hq, hkv, k_cache, k_norms, v_cache, v_norms, num_blocks,
                                block_tables, max_blocks, context_lens, out_f16, workspace, ws_bytes, stream);
}

tq_status tq_device_error(tq_stream stream, uint32_t* bits) { return tq_read_error_word(stream, bits); }

tq_status tq_check_device_error(const tq_ctx* ctx) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  return tq_read_error_word(nullptr, nullptr);
}

}  // extern "C"
