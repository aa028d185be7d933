// Encode kernel: fp16 vectors -> (packed Lloyd-Max codes, f32 norms).
//
// Method ("aither-kvcache" PyPI page, section "Algorithm", steps 1-5;
// "TurboQuant efficient inference", section "What TurboQuant is"): per vector
// x of length d, N = ||x||_2 stored as float32; z = sqrt(d) * H D x / N with D
// the seeded +-1 sign flip and H the orthonormal Walsh-Hadamard matrix;
// index_i = #{j : z_i >= t_j} over the Lloyd-Max decision boundaries t_j;
// indices packed little-endian, b bits each.
//
// B200 mapping:
//  * every lane owns 64 coordinates of one vector (1, 2 or 4 lanes per vector
//    for d = 64, 128, 256), so a CTA of 16 warps fits one SM; a warp owns a
//    tile of 32 lane-rows (4 KB, contiguous in memory) and runs its own
//    2-stage pipeline of one 1-D bulk copy (TMA) per tile;
//  * a lane reads its 16-byte chunk c ^ s into register slot c (s = a few bits
//    of its vector index), which spreads a quarter-warp's 128-bit shared loads
//    over distinct bank groups. Permuting the input of a Walsh-Hadamard
//    transform by XOR with s only multiplies output i by (-1)^popcount(i & s),
//    so the transform runs unchanged and the affected codes are mirrored
//    (code -> 2^b - 1 - code, the codebook is symmetric) by one XOR per word;
//  * the sign flip is an XOR of fp16 sign bits (masks from shared memory, in
//    the lane's chunk order), fused with the first butterfly stage at the
//    fp16 -> f32 conversion;
//  * the other Walsh-Hadamard stages run in registers with packed f32x2
//    add/sub, then one or two shuffle stages across the lanes of a vector;
//  * nearest level: q = w * (1 / (delta N)) + offset is floored through the
//    2^23 round-down trick into a cell of a lane-replicated shared table that
//    holds the one boundary inside the cell; one compare gives the index;
//  * coordinates within TQ_GUARD_Z of a boundary are redone exactly in fp64
//    by the whole warp (the f32 error bound is below that band), so the codes
//    are those of exact arithmetic;
//  * packed words are staged in the warp's shared output tile (rows
//    contiguous, as in memory) and leave through one 1-D bulk store (TMA).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

#include "tq_common.cuh"

namespace tq {

constexpr int ENC_WARPS = 16;
constexpr int ENC_STAGES = 2;
constexpr int ENC_C = 64;  // coordinates per lane
constexpr float MAGIC_2P23 = 8388608.0f;

template <int D, int BITS>
struct EncCfg {
  static constexpr int C = ENC_C;
  static constexpr int LPV = D / C;         // lanes per vector
  static constexpr int NP = C / 2;          // f32x2 pairs per lane
  static constexpr int VPW = 32 / LPV;      // vectors per warp tile
  static constexpr int P = D * BITS / 8;    // packed bytes per vector
  static constexpr int WL = C * BITS / 32;  // packed 32-bit words per lane
  static constexpr int IN_ROW = 2 * C;       // input lane-row (contiguous tile)
  static constexpr int OUT_ROW = WL;         // packed lane-row (contiguous tile, as in memory)
  static constexpr int L = 1 << BITS;
  static constexpr int GROUPS = C / 32;  // guard groups of 32 coordinates
  static constexpr int IN_STAGE = 32 * IN_ROW;
  static constexpr int OUT_WORDS = 32 * OUT_ROW;
};

struct EncArgs {
  const __half* x;
  int64_t n;  // vectors
  uint8_t* packed;
  float* norms;
  const int32_t* slot;  // append mode when non-null
  int h;                // heads per sequence (append mode)
  int64_t s_max;        // cache positions per sequence (append mode)
  uint32_t* err;
  int fault_inject;      // test hook: 1 = never issue the row copies
  long long wait_limit;  // bound on each mbarrier wait, SM cycles
};

// Shared memory layout (bytes), per CTA.
template <int D, int BITS>
struct EncSmem {
  using Cfg = EncCfg<D, BITS>;
  static constexpr int BAR = 0;                                            // warps x stages u64
  static constexpr int MASK = 256;                                         // sign masks, LPV x 32 u32
  static constexpr int SCR = MASK + 4 * 32 * 4;                            // per warp 32-float scratch
  static constexpr int IN = SCR + ENC_WARPS * 32 * 4;                      // input stages
  static constexpr int OUT = IN + ENC_WARPS * ENC_STAGES * Cfg::IN_STAGE;  // output rows
  static constexpr int LUT = OUT + ENC_WARPS * Cfg::OUT_WORDS * 4;          // cell table
  static size_t bytes(int cells) { return (size_t)LUT + (size_t)cells * 32 * 8; }
};

TQ_DEV uint2 lds_u2(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

// Pack code m (< 2^BITS) of coordinate i into the lane's word array.
template <int BITS, int WL>
TQ_DEV void put_code(uint32_t (&words)[WL], int i, uint32_t m) {
  const int off = i * BITS;
  // the code's bits are still zero in words[]: add == or (one shift-add)
  words[off >> 5] += m << (off & 31);
  if ((off & 31) + BITS > 32) words[(off >> 5) + 1] += m >> (32 - (off & 31));
}


template <int D, int BITS>
__global__ void __launch_bounds__(ENC_WARPS * 32, 1)
    encode_kernel(const __grid_constant__ tq_codec_tables T, const __grid_constant__ EncArgs a) {
  using Cfg = EncCfg<D, BITS>;
  using Sm = EncSmem<D, BITS>;
  constexpr int C = Cfg::C, NP = Cfg::NP, LPV = Cfg::LPV, VPW = Cfg::VPW, WL = Cfg::WL, L = Cfg::L;
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- lane-replicated cell table: entry (cell, lane) = {boundary bits, count below}
  {
    uint2* lut = reinterpret_cast<uint2*>(smem + Sm::LUT);
    const int cells = T.lut_cells;
    for (int e = threadIdx.x; e < cells * 32; e += blockDim.x) {
      const int cell = e >> 5;
      uint32_t below = 0;
      float thr = 3.0e38f;  // no boundary in this cell
#pragma unroll
      for (int j = 0; j < L - 1; ++j) {
        const float t = T.tau[j];
        if (t < (float)cell)
          ++below;
        else if (t < (float)(cell + 1))
          thr = t;
      }
      lut[e] = make_uint2(__float_as_uint(thr), below);
    }
  }
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem + Sm::MASK);
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) smask[i] = T.sign_h2[i];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sm::BAR) + warp * ENC_STAGES;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < ENC_STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();

  uint8_t* in_stage0 = smem + Sm::IN + warp * ENC_STAGES * Cfg::IN_STAGE;
  uint32_t* out_rows = reinterpret_cast<uint32_t*>(smem + Sm::OUT) + warp * Cfg::OUT_WORDS;
  float* scratch = reinterpret_cast<float*>(smem + Sm::SCR) + warp * 32;
  const uint32_t lut_lane = smem_u32(smem + Sm::LUT) + lane * 8u;
  const int part = lane & (LPV - 1);  // which 64-coordinate part of its vector this lane holds
  const uint4* my_masks = reinterpret_cast<const uint4*>(smask + part * NP);
  // chunk swizzle of this lane (shared by the lanes of a vector) and the
  // code-word mask that mirrors the codes of chunks whose output sign it flips
  const uint32_t swz = (uint32_t)(lane / LPV) & 7u;
  uint32_t flipw[WL];
#pragma unroll
  for (int w = 0; w < WL; ++w) flipw[w] = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (__popc((uint32_t)j & swz) & 1) {
#pragma unroll
      for (int i = 8 * j; i < 8 * j + 8; ++i) put_code<BITS>(flipw, i, (uint32_t)(L - 1));
    }
  }

  const int64_t n_tiles = (a.n + VPW - 1) / VPW;
  const int64_t gw = (int64_t)blockIdx.x * ENC_WARPS + warp;
  const int64_t n_warps = (int64_t)gridDim.x * ENC_WARPS;

  auto issue = [&](int64_t tile, int stage) {  // called by the whole warp
    const int64_t v0 = tile * VPW;
    const int valid_lanes = (int)min64(VPW, a.n - v0) * LPV;
    if (lane == 0) {
      const uint32_t bar = smem_u32(&bars[stage]);
      const uint32_t bytes = (uint32_t)(valid_lanes * 2 * C);
      mbar_arrive_expect_tx(bar, bytes);
      if (!a.fault_inject) bulk_g2s(smem_u32(in_stage0 + stage * Cfg::IN_STAGE), a.x + v0 * D, bytes, bar);
    }
    __syncwarp();
  };

#pragma unroll
  for (int s = 0; s < ENC_STAGES; ++s) {
    const int64_t t = gw + s * n_warps;
    if (t < n_tiles) issue(t, s);
  }

  const float Rscale = T.inv_delta;
  const float qoff = T.q_offset;
  const float gq = T.guard_q;

  int stage = 0;
  uint32_t parity = 0;  // bit s: parity of the next completion of stage s
  bool stored_once = false;
  for (int64_t tile = gw; tile < n_tiles; tile += n_warps) {
    const int64_t v0 = tile * VPW;
    const int valid_lanes = (int)min64(VPW, a.n - v0) * LPV;
    // every lane polls; the warp acts on one agreed outcome
    const bool ok = __all_sync(FULL, mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u, a.wait_limit));
    if (!ok) {
      if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
      // give the copies already issued into the other stage a bounded time to land
#pragma unroll
      for (int s = 1; s < ENC_STAGES; ++s) {
        const int os = (stage + s) % ENC_STAGES;
        if (tile + s * n_warps < n_tiles)
          (void)mbar_wait_bounded(smem_u32(&bars[os]), (parity >> os) & 1u, a.wait_limit);
      }
      if (lane == 0) bulk_wait_all<0>();
      return;
    }
    parity ^= 1u << stage;
    const bool active = lane < valid_lanes;
    const uint8_t* my_row = in_stage0 + stage * Cfg::IN_STAGE + lane * Cfg::IN_ROW;

    // ---- load (slot c <- chunk c ^ swz), sign flip (XOR of fp16 sign bits), first butterfly stage
    f2 v[NP];
#pragma unroll
    for (int c = 0; c < C / 8; ++c) {
      const uint32_t ch = (uint32_t)c ^ swz;
      uint4 r = make_uint4(0, 0, 0, 0);
      if (active) r = *reinterpret_cast<const uint4*>(my_row + 16 * ch);
      const uint4 mk = my_masks[ch];
      const uint32_t w4[4] = {r.x ^ mk.x, r.y ^ mk.y, r.z ^ mk.z, r.w ^ mk.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[q]));
        v[4 * c + q] = make_float2(f.x + f.y, f.x - f.y);
      }
    }
    // ---- sum of squares: (x0+x1)^2 + (x0-x1)^2 = 2 (x0^2 + x1^2); 8 chains
    f2 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = mul2(v[j], v[j]);
#pragma unroll
    for (int k = 4; k < NP; ++k) acc[k & 3] = fma2(v[k], v[k], acc[k & 3]);
    const f2 s4 = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
    float sum2 = s4.x + s4.y;
#pragma unroll
    for (int m = 1; m < LPV; m <<= 1) sum2 += __shfl_xor_sync(FULL, sum2, m);
    const float nrm = sqrtf(0.5f * sum2);

    // ---- remaining Walsh-Hadamard stages: in registers, then across the lanes of the vector
    wht_pairs<NP>(v);
#pragma unroll
    for (int m = 1; m < LPV; m <<= 1) {
      const f2 sg = (part & m) ? make_float2(-1.f, -1.f) : make_float2(1.f, 1.f);
#pragma unroll
      for (int k = 0; k < NP; ++k) {
        f2 o;
        o.x = __shfl_xor_sync(FULL, v[k].x, m);
        o.y = __shfl_xor_sync(FULL, v[k].y, m);
        v[k] = fma2(v[k], sg, o);
      }
    }

    // ---- quantize + pack
    const bool special = !(nrm > 0.f) || !(nrm <= 3.0e38f);  // zero or non-finite vector
    const float R = special ? 0.f : __fdiv_rn(Rscale, nrm);
    uint32_t words[WL];
#pragma unroll
    for (int w = 0; w < WL; ++w) words[w] = 0;
    uint32_t gmask = 0;
    if (!special) {
      const f2 R2 = make_float2(R, R), Q2 = make_float2(qoff, qoff), M2 = make_float2(MAGIC_2P23, MAGIC_2P23);
#pragma unroll
      for (int g = 0; g < Cfg::GROUPS; ++g) {
        float gmin = 3.0e38f;  // closest approach to a boundary in this group (q units)
#pragma unroll
        for (int k = g * 16; k < g * 16 + 16; ++k) {
          const f2 q2 = fma2(v[k], R2, Q2);
          const f2 qm = add2_rm(q2, M2);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float q = e ? q2.y : q2.x;
            const uint32_t qb = __float_as_uint(e ? qm.y : qm.x);
            const uint2 ent = lds_u2(qb * 256u + lut_lane);
            const float dl = __uint_as_float(ent.x) - q;
            gmin = fminf(gmin, fabsf(dl));
            put_code<BITS>(words, 2 * k + e, ent.y + (__float_as_uint(dl) >> 31));
          }
        }
        gmask |= (gmin < gq) ? (1u << g) : 0u;
      }
    } else {
#pragma unroll
      for (int i = 0; i < C; ++i) put_code<BITS>(words, i, (uint32_t)(L / 2));
    }
    if (!active) gmask = 0;
    // the previous tile's bulk store must have finished reading the staging tile
    if (lane == 0 && stored_once) bulk_wait_read<0>();
    __syncwarp();
#pragma unroll
    for (int w = 0; w < WL; ++w) words[w] ^= special ? 0u : flipw[w];
    if (WL % 4 == 0) {
#pragma unroll
      for (int w = 0; w < WL; w += 4)
        *reinterpret_cast<uint4*>(out_rows + lane * WL + w) = make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
    } else {
#pragma unroll
      for (int w = 0; w < WL; w += 2)
        *reinterpret_cast<uint2*>(out_rows + lane * WL + w) = make_uint2(words[w], words[w + 1]);
    }

    // ---- exact recheck of the coordinates inside the guard band (rare)
    uint32_t any = __ballot_sync(FULL, gmask != 0);
    while (any) {
      const int src = __ffs(any) - 1;
      any &= any - 1;
      uint32_t sg = __shfl_sync(FULL, gmask, src);
      const float srcR = __shfl_sync(FULL, R, src);
      const int src_part = src & (LPV - 1);
      const int vec_lane0 = src - src_part;
      while (sg) {
        const int g = __ffs(sg) - 1;
        sg &= sg - 1;
        // the source lane publishes the 32 rotated values of group g (their
        // signs may be flipped by its chunk swizzle: the flags are symmetric)
#pragma unroll
        for (int gg = 0; gg < Cfg::GROUPS; ++gg) {
          if (gg == g && lane == src) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              scratch[2 * k] = v[gg * 16 + k].x;
              scratch[2 * k + 1] = v[gg * 16 + k].y;
            }
          }
        }
        __syncwarp();
        const float wj = scratch[lane];
        __syncwarp();
        // the same f32 arithmetic as the main pass gives the same flags
        const float q = fmaf(wj, srcR, qoff);
        const uint32_t qb = __float_as_uint(__fadd_rd(q, MAGIC_2P23));
        const uint2 ent = lds_u2(qb * 256u + lut_lane);
        const float dl = __uint_as_float(ent.x) - q;
        uint32_t cm = __ballot_sync(FULL, fabsf(dl) < gq);
        while (cm) {
          const int j = __ffs(cm) - 1;
          cm &= cm - 1;
          const int i_local = g * 32 + j;
          const int gi = src_part * C + i_local;  // coordinate index in the vector
          // w_gi = sum_k s_k (-1)^popcount(gi & k) x_k: exact in fp64 for fp16 x
          double part_sum = 0.0, sq = 0.0;
#pragma unroll
          for (int t = 0; t < D / 32; ++t) {
            const int kk = lane + 32 * t;
            const __half hx = reinterpret_cast<const __half*>(
                in_stage0 + stage * Cfg::IN_STAGE + vec_lane0 * Cfg::IN_ROW)[kk];
            const double xk = (double)__half2float(hx);
            const uint32_t sbit = (smask[kk >> 1] >> (15 + 16 * (kk & 1))) & 1u;
            const uint32_t neg = sbit ^ (uint32_t)(__popc(gi & kk) & 1);
            part_sum += neg ? -xk : xk;
            sq = fma(xk, xk, sq);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            part_sum += __shfl_xor_sync(FULL, part_sum, o);
            sq += __shfl_xor_sync(FULL, sq, o);
          }
          const double n64 = sqrt(sq);
          uint32_t m = 0;
#pragma unroll
          for (int jj = 0; jj < L - 1; ++jj) m += (part_sum >= (double)T.bounds[jj] * n64) ? 1u : 0u;
          if (lane == 0) {
            const int off = i_local * BITS;
            uint32_t* row = out_rows + src * Cfg::OUT_ROW;
            const uint32_t msk = (uint32_t)(L - 1);
            row[off >> 5] = (row[off >> 5] & ~(msk << (off & 31))) | (m << (off & 31));
            if ((off & 31) + BITS > 32) {
              const int sh = 32 - (off & 31);
              row[(off >> 5) + 1] = (row[(off >> 5) + 1] & ~(msk >> sh)) | (m >> sh);
            }
          }
        }
      }
    }
    __syncwarp();

    // ---- write the tile
    if (a.slot == nullptr) {
      const uint32_t bytes = (uint32_t)(valid_lanes * WL * 4);
      if (bytes % 16 == 0) {  // always for full tiles; 1-D bulk copies move multiples of 16 bytes
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          bulk_s2g(a.packed + v0 * Cfg::P, smem_u32(out_rows), bytes);
          bulk_commit();
        }
        stored_once = true;
      } else {  // a partial tile of 24-byte rows: plain coalesced stores
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.packed + v0 * Cfg::P);
        for (int w = lane; w < valid_lanes * WL; w += 32) dst[w] = out_rows[w];
      }
      if (active && part == 0) a.norms[v0 + lane / LPV] = nrm;
    } else if (active) {
      const int64_t r = v0 + lane / LPV;
      const int64_t seq = r / a.h;
      const int head = (int)(r - seq * a.h);
      const int32_t s = a.slot[seq];
      if (s >= 0 && s < a.s_max) {
        const int64_t drow = (seq * a.s_max + s) * a.h + head;
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.packed + drow * Cfg::P) + part * WL;
#pragma unroll
        for (int w = 0; w < WL; ++w) dst[w] = out_rows[lane * Cfg::OUT_ROW + w];
        if (part == 0) a.norms[drow] = nrm;
      } else if (part == 0) {
        record_error(a.err, TQ_DEVERR_SLOT_RANGE);
      }
    }
    __syncwarp();

    // ---- refill this stage
    const int64_t next = tile + ENC_STAGES * n_warps;
    if (next < n_tiles) issue(next, stage);
    if (++stage == ENC_STAGES) stage = 0;
  }
  if (lane == 0) bulk_wait_all<0>();
}

template <int D, int BITS>
static cudaError_t launch_encode_t(const tq_codec_tables& T, const EncArgs& a, cudaStream_t st) {
  using Cfg = EncCfg<D, BITS>;
  const size_t smem = EncSmem<D, BITS>::bytes(T.lut_cells);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> configured{0};  // one bit per device
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(encode_kernel<D, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const int64_t tiles = (a.n + Cfg::VPW - 1) / Cfg::VPW;
  const int64_t ctas_needed = (tiles + ENC_WARPS - 1) / ENC_WARPS;
  const int grid = (int)std::min<int64_t>(ctas_needed, (int64_t)tq_sm_count(dev));
  encode_kernel<D, BITS><<<grid, ENC_WARPS * 32, smem, st>>>(T, a);
  return cudaGetLastError();
}

}  // namespace tq

using namespace tq;

tq_status tq_launch_encode(const tq_ctx* ctx, const void* x, int64_t n, void* packed, float* norms,
                           const int32_t* slot, int h, int64_t s_max, void* stream, int fault_inject) {
  if (n == 0) return TQ_OK;
  EncArgs a;
  a.x = static_cast<const __half*>(x);
  a.n = n;
  a.packed = static_cast<uint8_t*>(packed);
  a.norms = norms;
  a.slot = slot;
  a.h = h;
  a.s_max = s_max;
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.fault_inject = fault_inject;
  a.wait_limit = fault_inject ? 20000000LL : TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
  const tq_codec_tables& T = ctx->t;
#define TQ_ENC_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_encode_t<D_, B_>(T, a, st);
  TQ_ENC_CASE(64, 2) TQ_ENC_CASE(64, 3) TQ_ENC_CASE(64, 4)
  TQ_ENC_CASE(128, 2) TQ_ENC_CASE(128, 3) TQ_ENC_CASE(128, 4)
  TQ_ENC_CASE(256, 2) TQ_ENC_CASE(256, 3) TQ_ENC_CASE(256, 4)
#undef TQ_ENC_CASE
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
