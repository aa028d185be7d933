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
//  * a lane owns 64 coordinates (one, two or four lanes per vector for
//    d = 64, 128, 256; 128 registers, 16 warps per SM). A warp's tile is 32
//    such lane-rows; each warp runs its own 2-stage pipeline of 2-D tensor
//    copies (TMA, 128-byte swizzle, no multicast) of 64-coordinate boxes, so
//    the 128-bit shared loads that follow are conflict-free while every
//    register holds the coordinate of its natural position;
//  * the sign flip is an XOR of fp16 sign bits; the first butterfly stage is
//    fused with the fp16 -> f32 conversion (mixed-precision adds);
//  * the Walsh-Hadamard stages run in registers with packed f32x2 add/sub,
//    then one or two shuffle stages across the lanes of a vector;
//  * nearest level: q = w * (1 / (delta N)) + offset is floored through the
//    2^23 round-down trick into a cell of a shared table (16 lane copies)
//    that holds the one boundary inside the cell; one compare gives the index;
//  * coordinates within the guard band of a boundary are redone exactly in
//    fp64 by the whole warp (the f32 error bound is below the band), so the
//    codes are those of exact arithmetic;
//  * each lane stores its packed row with 128-bit stores (the 32 rows of a
//    tile are contiguous in memory).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "tq_common.cuh"

namespace tq {

constexpr int ENC_STAGES = 2;
constexpr int ENC_BOX_ROWS = 32;                                // lane-rows per tile
constexpr int ENC_BOX_COLS = 64;                                // fp16 per box row: 128 bytes
constexpr int ENC_BOX_BYTES = ENC_BOX_ROWS * ENC_BOX_COLS * 2;  // 4096
constexpr int ENC_LUT_COPIES = 16;
constexpr float MAGIC_2P23 = 8388608.0f;

constexpr int ENC_CMAX = 64;  // coordinates per lane at most

template <int D, int BITS>
struct EncCfg {
  static constexpr int C = D < ENC_CMAX ? D : ENC_CMAX;  // coordinates per lane
  static constexpr int LPV = D / C;            // lanes per vector
  static constexpr int NP = C / 2;             // f32x2 pairs per lane
  static constexpr int VPW = 32 / LPV;         // vectors per warp tile
  static constexpr int P = D * BITS / 8;       // packed bytes per vector
  static constexpr int PL = C * BITS / 8;      // packed bytes per lane-row
  static constexpr int WL = C * BITS / 32;     // packed 32-bit words per lane
  static constexpr int L = 1 << BITS;
  static constexpr int GROUPS = C / 32;        // guard groups of 32 coordinates
  static constexpr int BOXES = C / ENC_BOX_COLS;
  static constexpr int STAGE = BOXES * ENC_BOX_BYTES;
};

struct EncArgs {
  CUtensorMap tm_x;  // input as [n * lanes-per-vector rows, C] fp16, box 64 x 32, 128-byte swizzle
  // two = 1: a second tensor of n vectors in the same launch (append mode,
  // K and V of one step): the tiles after the first tensor's read tm_x2 and
  // write packed2 / norms2
  CUtensorMap tm_x2;
  uint8_t* packed2;
  float* norms2;
  int two;
  int64_t n;         // vectors
  int64_t vec_base;  // index of vector 0 of this launch in the caller's tensor (append mode)
  uint8_t* packed;
  float* norms;
  const int32_t* slot;  // append mode when non-null: a slot per sequence (slot_abs = 0) or per token (1)
  int h;                // heads per sequence (append mode)
  int64_t s_max;        // cache positions per sequence (append mode) or slots of the pool (slot_abs)
  int slot_abs;         // 1: row slot[token] of a pool of s_max rows; a negative slot is skipped silently
  uint32_t* err;
  uint32_t* side;        // offset variant: per vector fp16 offset | fp16 scale << 16 (instead of norms)
  int fault_inject;      // test hook: 1 = never issue the tile copies
  long long wait_limit;  // bound on each mbarrier wait, SM cycles
};

// Shared memory, per CTA: fixed header, then (1024-byte aligned, for the
// swizzle pattern) the warps' stage buffers, then the cell table.
template <int D, int BITS, int W>
struct EncSmem {
  using Cfg = EncCfg<D, BITS>;
  static constexpr int BAR = 0;                    // warps x stages u64
  static constexpr int BND = 256;                  // boundaries in z units, f32
  static constexpr int MASK = 320;                 // sign masks, D/2 u32
  static constexpr int SCR = 1024;                 // per warp 32-float scratch
  static constexpr int HEADER = SCR + 16 * 32 * 4;  // 3072
  static constexpr int IN_BYTES = W * ENC_STAGES * Cfg::STAGE;
  static size_t bytes(int cells) {
    return (size_t)HEADER + 1024 + IN_BYTES + (size_t)cells * ENC_LUT_COPIES * 8;
  }
};

TQ_DEV uint2 lds_u2(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

TQ_DEV uint4 lds_u4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}

TQ_DEV uint16_t lds_u16(uint32_t addr) {
  uint16_t r;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(addr));
  return r;
}

TQ_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// (x0 + x1, x0 - x1) in f32 for the fp16 pair (x0, x1) in the low and high
// halves of h2: one conversion and two mixed-precision (f16 op f32) adds of
// sm_100, each rounded once, as the plain f32 sum and difference are.
TQ_DEV f2 first_butterfly(uint32_t h2) {
  const uint16_t x0 = (uint16_t)(h2 & 0xffffu), x1 = (uint16_t)(h2 >> 16);
  float a1, s, d;
  asm("cvt.f32.f16 %0, %1;" : "=f"(a1) : "h"(x1));
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(s) : "h"(x0), "f"(a1));
  asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(x0), "f"(a1));
  return make_float2(s, d);
}

// acc + x0 + x1 for the fp16 pair in h2 (two mixed-precision adds).
TQ_DEV float add_f16_pair(uint32_t h2, float acc) {
  const uint16_t x0 = (uint16_t)(h2 & 0xffffu), x1 = (uint16_t)(h2 >> 16);
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(acc) : "h"(x0), "f"(acc));
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(acc) : "h"(x1), "f"(acc));
  return acc;
}

// (x0 - mu, x1 - mu) in f32 for the fp16 pair in h2, each rounded once.
TQ_DEV f2 sub_offset_pair(uint32_t h2, float mu) {
  const uint16_t x0 = (uint16_t)(h2 & 0xffffu), x1 = (uint16_t)(h2 >> 16);
  float y0, y1;
  asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(y0) : "h"(x0), "f"(mu));
  asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(y1) : "h"(x1), "f"(mu));
  return make_float2(y0, y1);
}

// Pack code m (< 2^BITS) of coordinate i into the lane's word array.
template <int BITS, int WL>
TQ_DEV void put_code(uint32_t (&words)[WL], int i, uint32_t m) {
  const int off = i * BITS;
  // the code's bits are still zero in words[]: add == or (one shift-add)
  words[off >> 5] += m << (off & 31);
  if ((off & 31) + BITS > 32) words[(off >> 5) + 1] += m >> (32 - (off & 31));
}

// Replace code i (runtime index) by m in the lane's word array. Every word
// goes through the same masked update, so the array is never indexed at run
// time (which would move it to local memory).
template <int BITS, int WL>
TQ_DEV void set_code(uint32_t (&words)[WL], int i, uint32_t m) {
  const int off = i * BITS, w0 = off >> 5, sh = off & 31;
  const uint32_t msk = (1u << BITS) - 1u;
  const bool straddles = sh + BITS > 32;
  const uint32_t lo_mask = msk << sh, lo_val = m << sh;
  const uint32_t hi_mask = straddles ? msk >> (32 - sh) : 0u, hi_val = straddles ? m >> (32 - sh) : 0u;
#pragma unroll
  for (int w = 0; w < WL; ++w) {
    const uint32_t mk = (w == w0 ? lo_mask : 0u) | (w == w0 + 1 ? hi_mask : 0u);
    const uint32_t v = (w == w0 ? lo_val : 0u) | (w == w0 + 1 ? hi_val : 0u);
    words[w] = (words[w] & ~mk) | v;
  }
}

// Shared address of coordinate k (0 <= k < C) of lane-row r in a stage
// written by the swizzled tensor copies: box k/64, 16-byte chunk
// ((k/8) % 8) ^ (r % 8) of the row's 128 bytes.
TQ_DEV uint32_t swz_addr(uint32_t stage_addr, int r, int k) {
  return stage_addr + (uint32_t)(k >> 6) * ENC_BOX_BYTES + (uint32_t)r * 128u +
         ((uint32_t)(((k >> 3) & 7) ^ (r & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

// Exact codes of the coordinates of one guard group of the source lane that
// lie inside the guard band. On entry scratch[0..31] holds the group's 32
// rotated f32 values (published by the source lane); on return scratch[j]
// holds, as a uint32, the exact code of coordinate j for every bit j of the
// returned mask. Called by the whole warp; rare, so kept out of line.
template <int D, int BITS, bool OS>
__device__ __noinline__ uint32_t recheck_group(float* scratch, float srcR, float qoff, float gq, uint32_t lut_lane,
                                               uint32_t st_addr, int row0, int gi0, const uint32_t* smask,
                                               const float* sbound, float mu, float nq) {
  constexpr int C = EncCfg<D, BITS>::C;
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const float wj = scratch[lane];
  // the same f32 arithmetic as the main pass gives the same flags and cells
  const float q = fmaf(wj, srcR, qoff);
  const uint32_t qb = __float_as_uint(__fadd_rd(q, MAGIC_2P23));
  const uint2 ent = lds_u2(qb * 128u + lut_lane);
  const float dlj = __uint_as_float(ent.x) - q;
  const uint32_t cm = __ballot_sync(FULL, fabsf(dlj) < gq);
  // N in fp64 from the fp16 inputs still in the stage (the offset variant
  // compares against its stored fp16 scale instead)
  double n64 = (double)nq;
  if constexpr (!OS) {
    double sq = 0.0;
#pragma unroll
    for (int t = 0; t < D / 32; ++t) {
      const int k = lane + 32 * t;
      const double xk = (double)__half2float(__ushort_as_half(lds_u16(swz_addr(st_addr, row0 + k / C, k % C))));
      sq = fma(xk, xk, sq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(FULL, sq, o);
    n64 = sqrt(sq);
  }
  uint32_t code = 0;
  for (uint32_t c2 = cm; c2; c2 &= c2 - 1) {
    const int j = __ffs(c2) - 1;
    const int gi = gi0 + j;  // coordinate index in the vector
    // w_gi = sum_k s_k (-1)^popcount(gi & k) y_k with y = x (or x - offset):
    // exact in fp64 for fp16 x and offset
    double ps = 0.0;
#pragma unroll
    for (int t = 0; t < D / 32; ++t) {
      const int k = lane + 32 * t;
      double xk = (double)__half2float(__ushort_as_half(lds_u16(swz_addr(st_addr, row0 + k / C, k % C))));
      if constexpr (OS) xk -= (double)mu;
      const uint32_t sbit = (smask[k >> 1] >> (15 + 16 * (k & 1))) & 1u;
      const uint32_t neg = sbit ^ (uint32_t)(__popc(gi & k) & 1);
      ps += neg ? -xk : xk;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(FULL, ps, o);
    // the cell of coordinate j holds boundary number `below`; every other
    // boundary is decided with a margin of 1/64 cell
    const uint32_t below = __shfl_sync(FULL, ent.y, j);
    const uint32_t m = below + ((ps >= (double)sbound[below] * n64) ? 1u : 0u);
    if (lane == j) code = m;
  }
  __syncwarp();
  reinterpret_cast<uint32_t*>(scratch)[lane] = code;
  __syncwarp();
  return cm;
}

template <int D, int BITS, int W, bool OS>
__global__ void __launch_bounds__(W * 32, 1)
    encode_kernel(const __grid_constant__ tq_codec_tables T, const __grid_constant__ EncArgs a) {
  using Cfg = EncCfg<D, BITS>;
  using Sm = EncSmem<D, BITS, W>;
  constexpr int C = Cfg::C, NP = Cfg::NP, LPV = Cfg::LPV, WL = Cfg::WL, L = Cfg::L;
  constexpr int WARPS = W;
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // programmatic dependent launch: the next kernel may set up as CTAs exit
  if (threadIdx.x == 0) grid_dep_launch();
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t in_addr = (smem_base + Sm::HEADER + 1023u) & ~1023u;  // stages: 1024-byte aligned
  const uint32_t lut_addr = in_addr + Sm::IN_BYTES;

  // ---- cell table (built on the host): entry (cell, copy) = {boundary bits
  // or 3e38 if none, count of boundaries below}, 16 lane copies
  {
    uint2* lut = reinterpret_cast<uint2*>(smem + (lut_addr - smem_base));
    const int entries = T.lut_cells * ENC_LUT_COPIES;
    for (int e = threadIdx.x; e < entries; e += blockDim.x) {
      const int cell = e / ENC_LUT_COPIES;
      lut[e] = make_uint2(T.cell[cell][0], T.cell[cell][1]);
    }
  }
  float* sbound = reinterpret_cast<float*>(smem + Sm::BND);
  for (int j = threadIdx.x; j < L - 1; j += blockDim.x) sbound[j] = T.bounds[j];
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem + Sm::MASK);
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) smask[i] = T.sign_h2[i];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sm::BAR) + warp * ENC_STAGES;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < ENC_STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t stage0 = in_addr + (uint32_t)(warp * ENC_STAGES * Cfg::STAGE);
  float* scratch = reinterpret_cast<float*>(smem + Sm::SCR) + warp * 32;
  // (2^23 + cell) * 128 = 2^31 + cell * 128 (mod 2^32): the 2^31 is taken out here
  const uint32_t lut_lane = lut_addr + (uint32_t)(lane & (ENC_LUT_COPIES - 1)) * 8u - 0x80000000u;
  const int part = lane & (LPV - 1);  // which C-coordinate part of its vector this lane holds
  const uint32_t sw = (uint32_t)lane & 7u;
  const uint32_t row_off = (uint32_t)lane * 128u;

  // a launch covers fewer than 2^30 lane-rows: tile and row indices fit in int32
  const int n_rows = (int)(a.n * LPV);
  const int n_tiles1 = (n_rows + ENC_BOX_ROWS - 1) / ENC_BOX_ROWS;  // tiles per tensor
  const int n_tiles = a.two ? 2 * n_tiles1 : n_tiles1;
  // warps numbered SM-minor, so a partial last round of tiles spreads over all SMs
  const int gw = warp * (int)gridDim.x + (int)blockIdx.x;
  const int n_warps = (int)gridDim.x * WARPS;

  auto issue = [&](int tile, int stage) {  // called by the whole warp
    if (lane == 0) {
      const uint32_t bar = smem_u32(&bars[stage]);
      mbar_arrive_expect_tx(bar, (uint32_t)Cfg::STAGE);  // full boxes: rows past the end are zero-filled
      const bool second = tile >= n_tiles1;
      const CUtensorMap* tm = second ? &a.tm_x2 : &a.tm_x;
      const int lt = second ? tile - n_tiles1 : tile;
      if (!a.fault_inject) {
#pragma unroll
        for (int b = 0; b < Cfg::BOXES; ++b)
          tma_load_2d(stage0 + (uint32_t)(stage * Cfg::STAGE + b * ENC_BOX_BYTES), tm, b * ENC_BOX_COLS,
                      lt * ENC_BOX_ROWS, bar);
      }
    }
    __syncwarp();
  };

  grid_dep_wait();  // the previous kernel of the stream may still write the inputs
#pragma unroll
  for (int s = 0; s < ENC_STAGES; ++s) {
    const int t = gw + s * n_warps;
    if (t < n_tiles) issue(t, s);
  }

  const float Rscale = T.inv_delta;
  const float qoff = T.q_offset;
  const float gq = T.guard_q;

  int stage = 0;
  uint32_t parity = 0;  // bit s: parity of the next completion of stage s
  for (int tile = gw; tile < n_tiles; tile += n_warps) {
    const bool second = tile >= n_tiles1;  // a tile of the second tensor
    const int r0 = (second ? tile - n_tiles1 : tile) * ENC_BOX_ROWS;  // first lane-row of the tile
    const int valid_rows = min(ENC_BOX_ROWS, n_rows - r0);
    // every lane polls; the warp acts on one agreed outcome
    const bool ok = __all_sync(FULL, mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u, a.wait_limit));
    if (!ok) {
      if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
      // give the copies already issued into the other stage a bounded time to land
      const int os = stage ^ 1;
      if (tile + n_warps < n_tiles) (void)mbar_wait_bounded(smem_u32(&bars[os]), (parity >> os) & 1u, a.wait_limit);
      return;
    }
    parity ^= 1u << stage;
    const bool active = lane < valid_rows;
    const uint32_t st_addr = stage0 + (uint32_t)(stage * Cfg::STAGE);
    const uint32_t my_row = st_addr + row_off;

    // ---- offset variant: the vector's mean, rounded to fp16, is subtracted first
    float mu = 0.f;
    if constexpr (OS) {
      float sx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int b = 0; b < Cfg::BOXES; ++b) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 r = lds_u4(my_row + (uint32_t)(b * ENC_BOX_BYTES) + ((c ^ sw) << 4));
          const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) sx[q] = add_f16_pair(w4[q], sx[q]);
        }
      }
      float sum = (sx[0] + sx[1]) + (sx[2] + sx[3]);
#pragma unroll
      for (int m = 1; m < LPV; m <<= 1) sum += __shfl_xor_sync(FULL, sum, m);
      mu = __half2float(__float2half_rn(sum * (1.0f / (float)D)));
    }

    // ---- load, sign flip (XOR of fp16 sign bits), first butterfly stage
    f2 v[NP];
    f2 acc[4];
#pragma unroll
    for (int b = 0; b < Cfg::BOXES; ++b) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 r = lds_u4(my_row + (uint32_t)(b * ENC_BOX_BYTES) + ((c ^ sw) << 4));
        const int k0 = b * 32 + c * 4;  // first pair of the chunk
        uint32_t w4[4] = {r.x, r.y, r.z, r.w};
        if constexpr (OS) {
          // y = x - offset in f32, then the sign flip on the f32 values
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i0 = 2 * (k0 + q);  // coordinate within this lane's part
            uint32_t m0, m1;
            if constexpr (LPV == 1) {
              m0 = T.sign_f32[i0], m1 = T.sign_f32[i0 + 1];
            } else if constexpr (LPV == 2) {
              m0 = T.sign_f32[i0], m1 = T.sign_f32[i0 + 1];
              if (part) m0 ^= T.sign_f32_dx[i0], m1 ^= T.sign_f32_dx[i0 + 1];
            } else {
              const uint32_t mh = smask[part * NP + k0 + q];
              m0 = (mh << 16) & 0x80000000u, m1 = mh & 0x80000000u;
            }
            const f2 y = sub_offset_pair(w4[q], mu);
            const float y0 = __uint_as_float(__float_as_uint(y.x) ^ m0), y1 = __uint_as_float(__float_as_uint(y.y) ^ m1);
            v[k0 + q] = make_float2(y0 + y1, y0 - y1);
            acc[q] = (k0 == 0) ? mul2(v[q], v[q]) : fma2(v[k0 + q], v[k0 + q], acc[q]);
          }
          continue;
        }
        if constexpr (LPV <= 2) {  // masks from the constant bank
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            w4[q] ^= T.sign_h2[k0 + q];
            if (LPV == 2 && part) w4[q] ^= T.sign_h2_dx[k0 + q];
          }
        } else {
          const uint4 mk = *reinterpret_cast<const uint4*>(smask + part * NP + k0);
          w4[0] ^= mk.x, w4[1] ^= mk.y, w4[2] ^= mk.z, w4[3] ^= mk.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          v[k0 + q] = first_butterfly(w4[q]);
          // sum of squares as the pairs arrive: (x0+x1)^2 + (x0-x1)^2 = 2 (x0^2 + x1^2);
          // 8 chains of at most 16 terms
          acc[q] = (k0 == 0) ? mul2(v[q], v[q]) : fma2(v[k0 + q], v[k0 + q], acc[q]);
        }
      }
    }
    const f2 s4 = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
    float sum2 = s4.x + s4.y;
#pragma unroll
    for (int m = 1; m < LPV; m <<= 1) sum2 += __shfl_xor_sync(FULL, sum2, m);
    float nrm = sqrtf(0.5f * sum2);
    uint32_t side_word = 0;
    if constexpr (OS) {  // the scale is stored in fp16 and the codes are taken relative to it
      const __half n16 = __float2half_rn(nrm);
      nrm = __half2float(n16);
      side_word = (uint32_t)__half_as_ushort(__float2half_rn(mu)) | ((uint32_t)__half_as_ushort(n16) << 16);
    }

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

    // ---- quantize + pack, 32 coordinates (one guard group) at a time; a
    // group with a coordinate inside the guard band is redone at once, while
    // its rotated values are still in registers
    const bool special = !(nrm > 0.f) || !(nrm <= 3.0e38f);  // zero or non-finite vector (or fp16 scale)
    const float R = special ? 0.f : __fdiv_rn(Rscale, nrm);
    uint32_t words[WL];
#pragma unroll
    for (int w = 0; w < WL; ++w) words[w] = 0;
    const f2 R2 = make_float2(R, R), Q2 = make_float2(qoff, qoff), M2 = make_float2(MAGIC_2P23, MAGIC_2P23);
#pragma unroll
    for (int g = 0; g < Cfg::GROUPS; ++g) {
      float gmin = 3.0e38f;  // closest approach to a boundary in this group (q units)
      if (!special) {
#pragma unroll
        for (int k = g * 16; k < g * 16 + 16; ++k) {
          const f2 q2 = fma2(v[k], R2, Q2);
          const f2 qm = add2_rm(q2, M2);  // bits: 2^23 + floor(q)
          float dl[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float q = e ? q2.y : q2.x;
            const uint32_t qb = __float_as_uint(e ? qm.y : qm.x);
            const uint2 ent = lds_u2(qb * 128u + lut_lane);
            dl[e] = __uint_as_float(ent.x) - q;
            put_code<BITS>(words, 2 * k + e, ent.y + (__float_as_uint(dl[e]) >> 31));
          }
          gmin = fminf(gmin, fminf(fabsf(dl[0]), fabsf(dl[1])));
        }
      } else {
#pragma unroll
        for (int i = g * 32; i < g * 32 + 32; ++i) put_code<BITS>(words, i, (uint32_t)(L / 2));
      }
      // ---- exact recheck of the coordinates of this group inside the guard band (rare)
      uint32_t any = __ballot_sync(FULL, active && gmin < gq);
      while (any) {
        const int src = __ffs(any) - 1;
        any &= any - 1;
        const float srcR = __shfl_sync(FULL, R, src);
        const int src_part = src & (LPV - 1);
        const int row0 = src - src_part;  // lane-row of part 0 of the source vector
        // the source lane publishes the group's 32 rotated values
        if (lane == src) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            scratch[2 * k] = v[g * 16 + k].x;
            scratch[2 * k + 1] = v[g * 16 + k].y;
          }
        }
        __syncwarp();
        const float src_mu = __shfl_sync(FULL, mu, src), src_nq = __shfl_sync(FULL, nrm, src);
        const uint32_t cm = recheck_group<D, BITS, OS>(scratch, srcR, qoff, gq, lut_lane, st_addr, row0,
                                                       src_part * C + g * 32, smask, sbound, src_mu, src_nq);
        if (lane == src) {
          for (uint32_t c2 = cm; c2; c2 &= c2 - 1) {
            const int j = __ffs(c2) - 1;
            set_code<BITS>(words, g * 32 + j, reinterpret_cast<const uint32_t*>(scratch)[j]);
          }
        }
        __syncwarp();
      }
    }

    // ---- write the tile: each lane its packed row (rows of a tile are contiguous)
    if (a.slot == nullptr) {
      if (active) {
        uint8_t* dst = a.packed + (int64_t)(r0 + lane) * Cfg::PL;
        if constexpr (Cfg::PL % 16 == 0) {
#pragma unroll
          for (int w = 0; w < WL; w += 4)
            *reinterpret_cast<uint4*>(dst + 4 * w) = make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
        } else {
#pragma unroll
          for (int w = 0; w < WL; w += 2) *reinterpret_cast<uint2*>(dst + 4 * w) = make_uint2(words[w], words[w + 1]);
        }
        if (part == 0) {
          if constexpr (OS)
            a.side[(r0 + lane) / LPV] = side_word;
          else
            a.norms[(r0 + lane) / LPV] = nrm;
        }
      }
    } else if (active) {
      const int64_t r = a.vec_base + (r0 + lane) / LPV;
      const int64_t seq = r / a.h;
      const int head = (int)(r - seq * a.h);
      const int32_t s = a.slot[seq];
      if (s >= 0 && s < a.s_max) {
        const int64_t drow = (a.slot_abs ? (int64_t)s : seq * a.s_max + s) * a.h + head;
        uint8_t* dst = (second ? a.packed2 : a.packed) + drow * Cfg::P + part * Cfg::PL;
#pragma unroll
        for (int w = 0; w < WL; w += 2) *reinterpret_cast<uint2*>(dst + 4 * w) = make_uint2(words[w], words[w + 1]);
        if (part == 0) (second ? a.norms2 : a.norms)[drow] = nrm;
      } else if (part == 0 && !(a.slot_abs && s < 0)) {
        record_error(a.err, TQ_DEVERR_SLOT_RANGE);
      }
    }
    __syncwarp();

    // ---- refill this stage
    const int next = tile + ENC_STAGES * n_warps;
    if (next < n_tiles) issue(next, stage);
    stage ^= 1;
  }
}

// Warps per CTA: 16 (one persistent CTA per SM) for bulk work; 2 when the
// launch has at most two tiles per SM (a streaming append), so its few tiles
// spread over the SMs instead of sharing a few of them.
constexpr int ENC_WARPS_BULK = 16;
constexpr int ENC_WARPS_SMALL = 2;

template <int D, int BITS, int W, bool OS>
static cudaError_t configure_encode(size_t smem, int dev) {
  static std::atomic<uint64_t> configured{0};  // one bit per device
  const uint64_t bit = 1ull << (dev & 63);
  if (configured.load() & bit) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(encode_kernel<D, BITS, W, OS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) configured.fetch_or(bit);
  return e;
}

// OS: the offset + fp16-scale variant (bulk launches only, 16 warps).
template <int D, int BITS, bool OS>
static cudaError_t launch_encode_t(const tq_codec_tables& T, EncArgs a, const void* x, cudaStream_t st,
                                   const void* x2 = nullptr) {
  using Cfg = EncCfg<D, BITS>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const size_t smem_bulk = EncSmem<D, BITS, ENC_WARPS_BULK>::bytes(T.lut_cells);
  const size_t smem_small = EncSmem<D, BITS, ENC_WARPS_SMALL>::bytes(T.lut_cells);
  if ((e = configure_encode<D, BITS, ENC_WARPS_BULK, OS>(smem_bulk, dev)) != cudaSuccess) return e;
  if (!OS && (e = configure_encode<D, BITS, ENC_WARPS_SMALL, false>(smem_small, dev)) != cudaSuccess) return e;
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tq_tensor_map_encode_fn());
  if (!enc) return cudaErrorNotSupported;
  const int sms = tq_sm_count(dev);
  // launches of at most 2^30 lane-rows keep the copy coordinates in int32
  const int64_t max_vec = ((int64_t)1 << 30) / Cfg::LPV;
  const int64_t n_total = a.n;
  if (x2 && n_total > max_vec / 2) return cudaErrorNotSupported;  // two tensors: one launch of int32 rows
  uint8_t* packed0 = a.packed;
  float* norms0 = a.norms;
  uint32_t* side0 = a.side;
  for (int64_t off = 0; off < n_total; off += max_vec) {
    const int64_t n = std::min(max_vec, n_total - off);
    a.n = n;
    a.vec_base = off;
    if (a.slot == nullptr) {
      a.packed = packed0 + off * Cfg::P;
      if (OS)
        a.side = side0 + off;
      else
        a.norms = norms0 + off;
    }
    const cuuint64_t dims[2] = {(cuuint64_t)Cfg::C, (cuuint64_t)(n * Cfg::LPV)};
    const cuuint64_t strides[1] = {(cuuint64_t)Cfg::C * 2};
    const cuuint32_t box[2] = {(cuuint32_t)ENC_BOX_COLS, (cuuint32_t)ENC_BOX_ROWS};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&a.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
            const_cast<void*>(static_cast<const void*>(static_cast<const __half*>(x) + off * D)), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
    if (x2 && enc(&a.tm_x2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x2), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
    const int64_t tiles = (x2 ? 2 : 1) * ((n * Cfg::LPV + ENC_BOX_ROWS - 1) / ENC_BOX_ROWS);
    if (!OS && tiles <= (int64_t)ENC_WARPS_SMALL * sms) {
      const int grid = (int)((tiles + ENC_WARPS_SMALL - 1) / ENC_WARPS_SMALL);
      e = tq_launch_pdl(encode_kernel<D, BITS, ENC_WARPS_SMALL, false>, dim3(grid), dim3(ENC_WARPS_SMALL * 32),
                        smem_small, st, T, a);
    } else {
      const int64_t ctas_needed = (tiles + ENC_WARPS_BULK - 1) / ENC_WARPS_BULK;
      const int grid = (int)std::min<int64_t>(ctas_needed, (int64_t)sms);
      e = tq_launch_pdl(encode_kernel<D, BITS, ENC_WARPS_BULK, OS>, dim3(grid), dim3(ENC_WARPS_BULK * 32), smem_bulk,
                        st, T, a);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq

using namespace tq;

tq_status tq_launch_encode(const tq_ctx* ctx, const void* x, int64_t n, void* packed, float* norms,
                           const int32_t* slot, int h, int64_t s_max, void* stream, int fault_inject,
                           int slot_abs) {
  if (n == 0) return TQ_OK;
  EncArgs a;
  memset(&a, 0, sizeof(a));
  a.n = n;
  a.packed = static_cast<uint8_t*>(packed);
  a.norms = norms;
  a.slot = slot;
  a.h = h;
  a.s_max = s_max;
  a.slot_abs = slot_abs;
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.fault_inject = fault_inject;
  a.wait_limit = fault_inject ? 20000000LL : TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
  const tq_codec_tables& T = ctx->t;
#define TQ_ENC_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_encode_t<D_, B_, false>(T, a, x, st);
  TQ_ENC_CASE(64, 2) TQ_ENC_CASE(64, 3) TQ_ENC_CASE(64, 4)
  TQ_ENC_CASE(128, 2) TQ_ENC_CASE(128, 3) TQ_ENC_CASE(128, 4)
  TQ_ENC_CASE(256, 2) TQ_ENC_CASE(256, 3) TQ_ENC_CASE(256, 4)
#undef TQ_ENC_CASE
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_launch_encode_append2(const tq_ctx* ctx, const void* xk, const void* xv, int64_t n, void* k_packed,
                                  float* k_norms, void* v_packed, float* v_norms, const int32_t* slot, int h,
                                  int64_t s_max, void* stream) {
  if (n == 0) return TQ_OK;
  EncArgs a;
  memset(&a, 0, sizeof(a));
  a.n = n;
  a.packed = static_cast<uint8_t*>(k_packed);
  a.norms = k_norms;
  a.packed2 = static_cast<uint8_t*>(v_packed);
  a.norms2 = v_norms;
  a.two = 1;
  a.slot = slot;
  a.h = h;
  a.s_max = s_max;
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.wait_limit = TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
  const tq_codec_tables& T = ctx->t;
#define TQ_ENC_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_encode_t<D_, B_, false>(T, a, xk, st, xv);
  TQ_ENC_CASE(64, 2) TQ_ENC_CASE(64, 3) TQ_ENC_CASE(64, 4)
  TQ_ENC_CASE(128, 2) TQ_ENC_CASE(128, 3) TQ_ENC_CASE(128, 4)
  TQ_ENC_CASE(256, 2) TQ_ENC_CASE(256, 3) TQ_ENC_CASE(256, 4)
#undef TQ_ENC_CASE
  if (e == cudaErrorNotSupported) return TQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_launch_encode_os(const tq_ctx* ctx, const void* x, int64_t n, void* packed, uint32_t* side,
                              void* stream) {
  if (n == 0) return TQ_OK;
  EncArgs a;
  memset(&a, 0, sizeof(a));
  a.n = n;
  a.packed = static_cast<uint8_t*>(packed);
  a.side = side;
  a.h = 1;
  a.s_max = 1;
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.wait_limit = TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
  const tq_codec_tables& T = ctx->t;
#define TQ_ENCOS_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_encode_t<D_, B_, true>(T, a, x, st);
  TQ_ENCOS_CASE(64, 2) TQ_ENCOS_CASE(64, 3) TQ_ENCOS_CASE(64, 4)
  TQ_ENCOS_CASE(128, 2) TQ_ENCOS_CASE(128, 3) TQ_ENCOS_CASE(128, 4)
  TQ_ENCOS_CASE(256, 2) TQ_ENCOS_CASE(256, 3) TQ_ENCOS_CASE(256, 4)
#undef TQ_ENCOS_CASE
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
