// Decode-step attention over packed caches, specialised for 4-bit keys and
// 2-bit values (the asymmetric K/V split of the "KVarN" and "aither-kvcache"
// pages) at head_dim 128, and at 256 for more than 4 query heads per kv head
// (with fewer, the stages of a CTA's kv heads do not fit beside the table and
// the launch takes the generic kernel).
//
// Same mathematics as the generic kernel (tq_attend.cu, after the
// "aither-kvcache" page, section "Zero-buffer fused attention", and
// "TurboQuant efficient inference", section "2. A fused decode path"):
// scores against codebook values with a rotated query, values accumulated in
// the rotated domain, one inverse rotation in the split merge. What differs
// is how the work is laid out on the SM, which is bound by shared-memory
// wavefronts and instruction issue rather than by HBM unless both are kept
// small:
//
//  * One CTA of 16 warps per SM, 227 KB of shared memory: a 64 KB key table
//    region and as many tiles of 32 positions in flight as fit around it (4
//    at head_dim 128 with 8 kv heads per CTA). A tile arrives as four
//    tensor copies (TMA, no multicast): K codes as [kv head][position][row]
//    (a box whose position and head dimensions are swapped relative to
//    memory, so the 16-byte fragment loads of a warp fall in distinct banks),
//    V codes as [position][row of all the CTA's heads + 16 bytes] (the copy
//    box is wider than the tensor and the excess is zero-filled, again for
//    distinct banks), K norms and V norms as [position][head].
//  * A warp owns one kv head (and one group of 4 query heads); the warps of
//    a tile form a group, and with 8 warps per tile the two groups take
//    alternate tiles, each group owning half of the stages. The last warp of
//    a group to finish a stage refills it.
//  * Key levels: one PRMT + one LDS per fp16 pair. The table region starts at
//    a shared address that is a multiple of 65536 and entries are 256 bytes
//    apart, so the address of (code byte, lane copy) is region | byte << 8 |
//    lane * 4, and one byte permute merges the code byte into a per-lane
//    constant. 32 lane copies make every lookup conflict-free.
//  * Value levels take two routes, so that the shared-memory pipe (one
//    wavefront per clock) and the integer pipe (half rate) work in parallel:
//      - table: entry = two 2-bit codes of position 2t and two of position
//        2t+1 (two LOP3 build four index bytes from two position words) ->
//        the two fp16 pairs = two A-fragment registers of the value MMA, 16
//        lane copies in bytes [128, 256) of the 256-byte entries (LDS.64);
//      - registers: the four fp16 levels fit in two registers (low bytes,
//        high bytes) and one byte permute whose selector is built from two
//        codes (one IMAD per two selectors) returns the pair (c[code at
//        2t], c[code at 2t+1]).
//    FA_V_LUT_GROUPS of the four groups of m-blocks take the table.
//  * P (softmax weights x V norms, fp16 hi+lo) goes from the score MMA's
//    accumulator layout to the value MMA's B fragment with one movmatrix
//    transpose per 8 positions; no shared-memory round trip.
//  * The running max is raised only when a tile's max exceeds it by more
//    than 2^8 (exact: every weight and the accumulator use the same stale
//    max, and the weights stay below 2^8), so the accumulator is rarely
//    rescaled; the row sums stay per lane until the end.
// The partial (max, sum, accumulator) of each split goes to the same
// workspace as the generic kernel's and the same merge kernel finishes.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "tq_attend.cuh"

namespace tq {

constexpr int FA_WARPS = 16;
constexpr int FA_MAX_STAGES = 8;
constexpr int FA_TABLE_BYTES = 65536;
constexpr float FA_RESCALE_LOG2 = 8.f;  // raise the running max only past this margin
#ifndef FA_V_LUT_GROUPS
#define FA_V_LUT_GROUPS 3  // groups of value m-blocks (of 4) dequantised through the shared table
#endif

// Floats per staged norm row: the copy box is wider than the CTA's kv heads
// (the excess is zero-filled), so the norms of the 8 positions a warp reads
// at once fall in 8 different banks (a pitch of hw floats would put rows gq
// and gq + 4 in one bank for hw = 8).
__host__ __device__ constexpr int fa_norm_pitch(int hw) { return hw == 4 ? 12 : hw + 4; }

struct FastArgs {
  CUtensorMap tm_k;   // K codes  box (D/2 bytes, 32 positions, hw heads) -> [head][position][D/2]
  CUtensorMap tm_v;   // V codes  box (hw * D/4 + 16 bytes, 1 group, 32 positions)
  CUtensorMap tm_kn;  // K norms  box (hw, 1 group, 32 positions) f32
  CUtensorMap tm_vn;  // V norms
  AttnArgs a;
  uint32_t smem_base;  // shared address the dynamic region must start at
  int tb_off;          // offset of the table region (its shared address is a multiple of 65536)
  int kbuf[FA_MAX_STAGES], vbuf[FA_MAX_STAGES], knb[FA_MAX_STAGES], vnb[FA_MAX_STAGES];
  int n_stages;  // a multiple of n_groups
  int n_groups;  // warp groups taking alternate tiles
  int wpt;       // warps per tile: hw * nt
  int vpitch;    // bytes per V position row in shared memory (hw * D/4 + 16)
  int k_head_copies;  // 1: the K box is one head, issued hw times (no swapped-dimension map)
  int paged;          // 1: boxes of 16 positions, two per tile, rows from the block table
  int pg_off;         // paged: shared copy of the split's first block rows (int32), at this offset
  int pg_cap;         //        and this many entries (later blocks are read from the table)
  uint32_t tile_bytes;
};

TQ_DEV void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Table loads: the table is constant once built, so these need no ordering
// beyond their address dependencies.
TQ_DEV uint32_t lds_tab32(uint32_t addr) {
  uint32_t r;
  asm("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}

// 8x8 transpose of 16-bit elements across the warp (fragment layout in and out).
TQ_DEV uint32_t transpose8x8(uint32_t x) {
  uint32_t r;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

TQ_DEV float fast_exp2(float x) {  // the SFU's 2^x; 2^-inf = 0
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// fp16 hi + lo split of v packed as (lo half = hi part, high half = lo part).
TQ_DEV uint32_t split_hi_lo(float v) {
  const float r = v - __half2float(__float2half_rn(v));
  const __half2 p = __floats2half2_rn(v, r);  // (fp16(v), fp16(v - fp16(v)))
  return *reinterpret_cast<const uint32_t*>(&p);
}

TQ_DEV uint2 lds_tab64(uint32_t addr) {
  uint2 r;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

// Value-level pairs from two position words of 2-bit codes. `x` holds, in
// bits [1:0] of each byte, code cA (byte 0), cB (byte 1), cA' (byte 2), cB'
// (byte 3); the selector byte c * 0x11 + 0x40 picks (low byte of level c,
// high byte of level c) from the pool (v_lo, v_hi). Returns the fp16 pairs
// (c[cA], c[cB]) and (c[cA'], c[cB']).
TQ_DEV void value_pairs(uint32_t x, uint32_t v_lo, uint32_t v_hi, uint32_t& p0, uint32_t& p1) {
  const uint32_t sel = x * 0x11u + 0x40404040u;
  p0 = __byte_perm(v_lo, v_hi, sel);
  p1 = __byte_perm(v_lo, v_hi, sel >> 16);
}

template <int D, int HW>
__global__ void __launch_bounds__(FA_WARPS * 32, 1) attend_fast_kernel(const __grid_constant__ FastArgs f) {
  constexpr int PK = D / 2;   // K bytes per head row
  constexpr int PV = D / 4;   // V bytes per head row
  constexpr int NB = D / 16;  // k-blocks of the score MMA = m-blocks of the value MMA
  constexpr int KQW = D / 32; // words of a K row per lane (a quarter of the row)
  constexpr int VQW = D / 128;  // words of a V row per lane (an eighth)
  constexpr int VP = HW * PV + 16;  // shared pitch of a V position row
  constexpr int hw = HW;            // kv heads per CTA
  constexpr int NPITCH = fa_norm_pitch(HW);  // floats per staged norm row
  const AttnArgs& a = f.a;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) != f.smem_base) {  // the table addressing needs the planned addresses
    if (threadIdx.x == 0) record_error(a.err, TQ_DEVERR_SMEM_LAYOUT);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int split = blockIdx.x, b = blockIdx.y, hgrp = blockIdx.z;
  const int g = a.g, nt = a.nt, NS = f.n_stages, G = f.n_groups;
  const int grp = warp / f.wpt, wi = warp % f.wpt;
  const int hl = wi / nt, ct = wi % nt;  // local kv head and column tile of this warp
  const int hk = hgrp * hw + hl;

  int64_t pos = a.positions[b];
  if (pos > a.s_max) {
    if (threadIdx.x == 0 && split == 0 && hgrp == 0) record_error(a.err, TQ_DEVERR_POS_RANGE);
    pos = a.s_max;
  }
  const int64_t s0 = (int64_t)split * a.chunk;
  const int64_t s1 = min64(s0 + a.chunk, pos);
  const int64_t npos = s1 > s0 ? s1 - s0 : 0;
  const int ntiles = (int)((npos + ATT_TILE - 1) / ATT_TILE);
  const int nv_last = (int)(npos - (int64_t)(ntiles - 1) * ATT_TILE);  // positions in the last tile

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);          // full[stage]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + 64);      // warps done with the stage
  uint32_t* issued = reinterpret_cast<uint32_t*>(smem + 96);   // copies issued into the stage
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      cnt[s] = 0;
      issued[s] = 0;
    }
    fence_mbar_init();
  }
  const int row0 = f.paged ? 0 : (int)((int64_t)b * a.s_max + s0);  // first cache row of this split
  auto issue = [&](int tile, int s) {  // one thread
    const uint32_t bar = smem_u32(&bars[s]);
    mbar_arrive_expect_tx(bar, f.tile_bytes);
    if (f.paged) {
      // the tile's two blocks of 16 positions (rows of the split's first
      // blocks from the shared copy); a second block past the context
      // re-reads the first (its positions are masked out)
      const int64_t sa = s0 + (int64_t)tile * ATT_TILE;
      const int ja = 2 * tile;  // block index within the split
      const int* pg = reinterpret_cast<const int*>(smem + f.pg_off);
      const int ra = ja < f.pg_cap ? pg[ja] : (int)attn_pos_row(a, b, sa);
      const int rb = sa + ATT_BLOCK < pos ? (ja + 1 < f.pg_cap ? pg[ja + 1] : (int)attn_pos_row(a, b, sa + ATT_BLOCK))
                                          : ra;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = h ? rb : ra;
        tma_load_3d(smem_u32(smem + f.kbuf[s] + h * hw * ATT_BLOCK * PK), &f.tm_k, 0, row, hgrp * hw, bar);
        tma_load_3d(smem_u32(smem + f.vbuf[s] + h * ATT_BLOCK * VP), &f.tm_v, 0, hgrp, row, bar);
        tma_load_3d(smem_u32(smem + f.knb[s] + h * ATT_BLOCK * NPITCH * 4), &f.tm_kn, 0, hgrp, row, bar);
        tma_load_3d(smem_u32(smem + f.vnb[s] + h * ATT_BLOCK * NPITCH * 4), &f.tm_vn, 0, hgrp, row, bar);
      }
      issued[s] += 1;
      return;
    }
    const int row = row0 + tile * ATT_TILE;
    if (f.k_head_copies) {
      for (int h = 0; h < hw; ++h)
        tma_load_3d(smem_u32(smem + f.kbuf[s] + h * ATT_TILE * PK), &f.tm_k, 0, hgrp * hw + h, row, bar);
    } else {
      tma_load_3d(smem_u32(smem + f.kbuf[s]), &f.tm_k, 0, row, hgrp * hw, bar);
    }
    tma_load_3d(smem_u32(smem + f.vbuf[s]), &f.tm_v, 0, hgrp, row, bar);
    tma_load_3d(smem_u32(smem + f.knb[s]), &f.tm_kn, 0, hgrp, row, bar);
    tma_load_3d(smem_u32(smem + f.vnb[s]), &f.tm_vn, 0, hgrp, row, bar);
    issued[s] += 1;
  };
  if (f.paged) {  // the split's first block rows, before the first copies are issued
    int* pg = reinterpret_cast<int*>(smem + f.pg_off);
    const int nblk = (int)min64(f.pg_cap, (npos + ATT_BLOCK - 1) / ATT_BLOCK);
    for (int j = threadIdx.x; j < nblk; j += blockDim.x) pg[j] = (int)attn_pos_row(a, b, s0 + (int64_t)j * ATT_BLOCK);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    for (int t = 0; t < NS && t < ntiles; ++t) issue(t, t);
  }

  // rotated, scaled queries of the CTA's heads (q~ = H_pm D_K q), built in the
  // table region before the table
  float* qt = reinterpret_cast<float*>(smem + f.tb_off);
  const int nq = hw * g;
  for (int e = threadIdx.x; e < nq * D; e += blockDim.x) {
    const int i = e % D;
    const float x = __half2float(a.q[((int64_t)b * a.hq + (int64_t)hgrp * hw * g) * D + e]);
    const uint32_t sb = (a.k_sign_h2[i >> 1] >> (15 + 16 * (i & 1))) & 1u;
    qt[e] = sb ? -x : x;
  }
  __syncthreads();
  for (int h = 1; h < D; h <<= 1) {
    for (int e = threadIdx.x; e < nq * D / 2; e += blockDim.x) {
      const int r = e / (D / 2), k = e % (D / 2);
      const int i = (k / h) * 2 * h + (k % h);
      float* row = qt + r * D;
      const float u = row[i], w = row[i + h];
      row[i] = u + w;
      row[i + h] = u - w;
    }
    __syncthreads();
  }
  // B fragments of the score MMA: column gq = (query head ct*4 + gq/2, hi or
  // lo part); k rows 2tq, 2tq+1 | 2tq+8, 2tq+9 of block kb = dims
  // tq*D/4 + 4kb + {0,1} | {2,3} (a lane's K codes are a contiguous quarter row)
  uint32_t bq[NB][2];
  {
    const int j = ct * 4 + (gq >> 1);
    const bool lo = gq & 1;
    const float* qrow = qt + (hl * g + (j < g ? j : 0)) * D;
#pragma unroll
    for (int kb = 0; kb < NB; ++kb) {
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const int d0 = tq * (D / 4) + 4 * kb + 2 * e2;
        float v0 = 0.f, v1 = 0.f;
        if (j < g) {
          v0 = qrow[d0] * a.q_scale;
          v1 = qrow[d0 + 1] * a.q_scale;
        }
        if (lo) {
          v0 -= __half2float(__float2half_rn(v0));
          v1 -= __half2float(__float2half_rn(v1));
        }
        bq[kb][e2] = pack_half2(v0, v1);
      }
    }
  }
  __syncthreads();  // the query buffer becomes the key table

  const uint32_t tb = f.smem_base + (uint32_t)f.tb_off;  // a multiple of 65536
  {
    uint32_t* tw = reinterpret_cast<uint32_t*>(smem + f.tb_off);
    for (int e = threadIdx.x; e < 256 * 32; e += blockDim.x) {
      const int en = e >> 5;
      tw[en * 64 + (e & 31)] = pack_half2(a.k_levels[en & 15], a.k_levels[en >> 4]);
    }
    if (FA_V_LUT_GROUPS > 0) {
      for (int e = threadIdx.x; e < 256 * 16; e += blockDim.x) {
        const int en = e >> 4;
        // index bits: [1:0] dim d0 / position A, [3:2] d1 / A, [5:4] d0 / B, [7:6] d1 / B
        uint2* p = reinterpret_cast<uint2*>(smem + f.tb_off + en * 256 + 128 + (e & 15) * 8);
        *p = make_uint2(pack_half2(a.v_levels[en & 3], a.v_levels[(en >> 4) & 3]),
                        pack_half2(a.v_levels[(en >> 2) & 3], a.v_levels[en >> 6]));
      }
    }
  }
  // the 2-bit value levels as fp16: low bytes and high bytes
  uint32_t v_lo = 0, v_hi = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t h = __half_as_ushort(__float2half_rn(a.v_levels[c]));
    v_lo |= (h & 0xFFu) << (8 * c);
    v_hi |= (h >> 8) << (8 * c);
  }
  __syncthreads();

  const uint32_t LK = tb | (uint32_t)(lane * 4);  // byte 0 = lane copy, bytes 2-3 = region
  // K stage layout: [head][32 positions][row], or with paged boxes
  // [16-position box][head][16 positions][row]
  const int khs = f.paged ? ATT_BLOCK * PK : ATT_TILE * PK;     // head stride
  const int kbs = f.paged ? hw * ATT_BLOCK * PK : ATT_BLOCK * PK;  // stride of positions 16..31
  const int kcol = hl * khs + tq * (D / 8);  // this lane's quarter of its head's K rows
  const int vcol = hl * PV + gq * (D / 32);              // this lane's eighth of its head's V row
  const uint32_t LV = tb | (uint32_t)(128 + (lane & 15) * 8);

  float m_run = -INFINITY, l_run = 0.f;
  float acc[NB][4];
#pragma unroll
  for (int i = 0; i < NB; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;

  int s = grp;          // stage of this warp's current tile
  uint32_t phase = 0;   // parity of that stage's current fill
  for (int tile = grp; tile < ntiles; tile += G) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&bars[s]), phase, a.wait_limit));
    if (!ok) {
      if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
      break;
    }
    const uint8_t* kst = smem + f.kbuf[s] + kcol;
    const uint8_t* vst = smem + f.vbuf[s] + vcol;
    const float* kns = reinterpret_cast<const float*>(smem + f.knb[s]) + hl;
    const float* vns = reinterpret_cast<const float*>(smem + f.vnb[s]) + hl;
    const int nv = tile == ntiles - 1 ? nv_last : ATT_TILE;

    // ---- scores: rows = positions, columns = 4 query heads x (hi, lo)
    float sc[2][2];
#pragma unroll
    for (int mb16 = 0; mb16 < 2; ++mb16) {
      const int r0 = mb16 * 16 + gq;
      const uint8_t* krow = kst + mb16 * kbs + gq * PK;  // position r0 (r0 + 8 is 8 rows on)
      uint32_t kw0[KQW], kw1[KQW];
#pragma unroll
      for (int w = 0; w < KQW; w += 4) {
        const uint4 x0 = *reinterpret_cast<const uint4*>(krow + 4 * w);
        const uint4 x1 = *reinterpret_cast<const uint4*>(krow + 8 * PK + 4 * w);
        kw0[w] = x0.x, kw0[w + 1] = x0.y, kw0[w + 2] = x0.z, kw0[w + 3] = x0.w;
        kw1[w] = x1.x, kw1[w + 1] = x1.y, kw1[w + 2] = x1.z, kw1[w + 3] = x1.w;
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < NB; ++kb) {
        // code byte 2kb -> a0 (row r0) / a1 (row r0+8); byte 2kb+1 -> a2 / a3
        const uint32_t w0 = kw0[kb >> 1], w1 = kw1[kb >> 1];
        const uint32_t se = (kb & 1) ? 0x7624u : 0x7604u, so = (kb & 1) ? 0x7634u : 0x7614u;
        const uint32_t a0 = lds_tab32(__byte_perm(w0, LK, se));
        const uint32_t a1 = lds_tab32(__byte_perm(w1, LK, se));
        const uint32_t a2 = lds_tab32(__byte_perm(w0, LK, so));
        const uint32_t a3 = lds_tab32(__byte_perm(w1, LK, so));
        mma16816(c, a0, a1, a2, a3, bq[kb][0], bq[kb][1]);
      }
      sc[mb16][0] = (c[0] + c[1]) * kns[r0 * NPITCH];
      sc[mb16][1] = (c[2] + c[3]) * kns[(r0 + 8) * NPITCH];
    }
    const bool ragged = nv < ATT_TILE;
    if (ragged) {
#pragma unroll
      for (int mb16 = 0; mb16 < 2; ++mb16)
#pragma unroll
        for (int r = 0; r < 2; ++r)
          if (mb16 * 16 + gq + 8 * r >= nv) sc[mb16][r] = -INFINITY;
    }

    // ---- online softmax (log2 domain) for query head ct*4 + tq
    const float mx = warp_max8(fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1])));
    if (__any_sync(0xffffffffu, mx > m_run + FA_RESCALE_LOG2)) {
      const float mn = fmaxf(m_run, mx);
      const float alpha = fast_exp2(m_run - mn);
      l_run *= alpha;
#pragma unroll
      for (int i = 0; i < NB; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] *= alpha;
      m_run = mn;
    }
    uint32_t bp[2][2];  // B fragments of the value MMA (positions x columns)
#pragma unroll
    for (int mb16 = 0; mb16 < 2; ++mb16) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = mb16 * 16 + gq + 8 * r;
        const float p = fast_exp2(sc[mb16][r] - m_run);
        l_run += p;
        float pv = p * vns[row * NPITCH];
        if (ragged && row >= nv) pv = 0.f;
        bp[mb16][r] = transpose8x8(split_hi_lo(pv));
      }
    }

    // ---- values: acc[dims x columns] += V^T[dims x 16 positions] * P[16 positions x columns].
    // A-fragment register for (dim, positions 2tq | 2tq+1) = (c[code at 2tq], c[code at 2tq+1]);
    // the lane's codes are word(s) of its eighth of each position row, code k
    // of word w = dim D/8*gq + 16w + k, and code 2mb' (2mb'+1) feeds row gq (gq+8)
    // of m-block 8w + mb'.
#pragma unroll
    for (int mb16 = 0; mb16 < 2; ++mb16) {
      const uint8_t* ra = vst + (mb16 * 16 + 2 * tq) * VP;  // position 2tq of the block
      const uint32_t b0 = bp[mb16][0], b1 = bp[mb16][1];
#pragma unroll
      for (int w = 0; w < VQW; ++w) {
        const uint32_t wa0 = reinterpret_cast<const uint32_t*>(ra)[w];
        const uint32_t wb0 = reinterpret_cast<const uint32_t*>(ra + VP)[w];
        const uint32_t wa1 = reinterpret_cast<const uint32_t*>(ra + 8 * VP)[w];
        const uint32_t wb1 = reinterpret_cast<const uint32_t*>(ra + 9 * VP)[w];
        // table route: byte k = low nibble of A's byte k | low nibble of B's byte k << 4 (lo),
        // and the high nibbles (hi); m-block mb reads byte mb >> 1 of (mb & 1 ? hi : lo)
        const uint32_t lo0 = (wa0 & 0x0F0F0F0Fu) | ((wb0 << 4) & 0xF0F0F0F0u);
        const uint32_t hi0 = ((wa0 >> 4) & 0x0F0F0F0Fu) | (wb0 & 0xF0F0F0F0u);
        const uint32_t lo1 = (wa1 & 0x0F0F0F0Fu) | ((wb1 << 4) & 0xF0F0F0F0u);
        const uint32_t hi1 = ((wa1 >> 4) & 0x0F0F0F0Fu) | (wb1 & 0xF0F0F0F0u);
        // register route: bytes (A0, B0, A1, B1) and (A2, B2, A3, B3) of the two position words
        const uint32_t P0 = __byte_perm(wa0, wb0, 0x5140u), Q0 = __byte_perm(wa0, wb0, 0x7362u);
        const uint32_t P1 = __byte_perm(wa1, wb1, 0x5140u), Q1 = __byte_perm(wa1, wb1, 0x7362u);
        // group gi: m-blocks mlo and mlo + 2 (codes 2mb, 2mb+1 of the word share
        // selector words: codes e, 4+e of P (0..7) or 8+e, 12+e of Q)
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          const int mlo = 4 * (gi >> 1) + (gi & 1), mhi = mlo + 2;
          if (gi < FA_V_LUT_GROUPS) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int mb = t ? mhi : mlo;
              const uint32_t sel = 0x7604u | ((uint32_t)((mb >> 1) & 3) << 4);
              const uint2 x = lds_tab64(__byte_perm((mb & 1) ? hi0 : lo0, LV, sel));
              const uint2 y = lds_tab64(__byte_perm((mb & 1) ? hi1 : lo1, LV, sel));
              mma16816(acc[8 * w + mb], x.x, x.y, y.x, y.y, b0, b1);
            }
          } else {
            const uint32_t W0 = (gi >> 1) ? Q0 : P0, W1 = (gi >> 1) ? Q1 : P1;
            const int e0 = 2 * (gi & 1);
            uint32_t a_lo[2], a_hi[2], c_lo[2], c_hi[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              value_pairs((W0 >> (2 * (e0 + j))) & 0x03030303u, v_lo, v_hi, a_lo[j], a_hi[j]);
              value_pairs((W1 >> (2 * (e0 + j))) & 0x03030303u, v_lo, v_hi, c_lo[j], c_hi[j]);
            }
            mma16816(acc[8 * w + mlo], a_lo[0], a_lo[1], c_lo[0], c_lo[1], b0, b1);
            mma16816(acc[8 * w + mhi], a_hi[0], a_hi[1], c_hi[0], c_hi[1], b0, b1);
          }
        }
      }
    }

    // this warp is done with the stage; the group's last warp refills it
    __syncwarp();
    if (tile + NS < ntiles && lane == 0) {
      __threadfence_block();
      if (atomicAdd(&cnt[s], 1u) == (uint32_t)(f.wpt - 1)) {
        cnt[s] = 0;
        issue(tile + NS, s);
      }
    }
    s += G;
    if (s >= NS) {
      s -= NS;
      phase ^= 1u;
    }
  }
  // ---- this warp's partial for query head hk*g + ct*4 + tq; accumulator
  // row gq of m-block mb = dim D/8*gq + 2mb, row gq+8 = the next dim
  float o[2 * NB];
#pragma unroll
  for (int mb = 0; mb < NB; ++mb) {
    o[2 * mb] = acc[mb][0] + acc[mb][1];
    o[2 * mb + 1] = acc[mb][2] + acc[mb][3];
  }
  l_run = warp_sum8(l_run);
  __syncthreads();  // every warp is past the tables: the region holds the group merge
  constexpr int MS = 2 * NB + 2;  // floats per lane
  float* mg = reinterpret_cast<float*>(smem + f.tb_off);
  if (grp > 0) {
    float* dst = mg + ((size_t)((grp - 1) * f.wpt + wi) * 32 + lane) * MS;
    dst[0] = m_run;
    dst[1] = l_run;
#pragma unroll
    for (int i = 0; i < 2 * NB; ++i) dst[2 + i] = o[i];
  }
  __syncthreads();
  if (grp == 0) {
    for (int gr = 1; gr < f.n_groups; ++gr) {
      const float* src = mg + ((size_t)((gr - 1) * f.wpt + wi) * 32 + lane) * MS;
      const float m1 = src[0];
      const float M = fmaxf(m_run, m1);
      if (M != -INFINITY) {
        const float w0 = fast_exp2(m_run - M), w1 = fast_exp2(m1 - M);
        l_run = w0 * l_run + w1 * src[1];
#pragma unroll
        for (int i = 0; i < 2 * NB; ++i) o[i] = w0 * o[i] + w1 * src[2 + i];
        m_run = M;
      }
    }
    const int j = ct * 4 + tq;
    if (j < g) {
      const int h = hk * g + j;
      const int64_t idx = ((int64_t)b * a.hq + h) * a.n_split + split;
      if (gq == 0) {
        a.ws_m[idx] = m_run;
        a.ws_l[idx] = l_run;
      }
      float4* dst = reinterpret_cast<float4*>(a.ws_acc + idx * D + gq * (D / 8));
#pragma unroll
      for (int i = 0; i < NB / 2; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
  }

  // every copy issued into a stage has landed before the CTA exits (after a
  // time-out too, within the bound)
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      if (issued[s] > 0) (void)mbar_wait_bounded(smem_u32(&bars[s]), (issued[s] - 1) & 1u, a.wait_limit);
    }
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D tensor map: extents dims (innermost first), byte strides of dims 1
// and 2, box extents box. Returns false when the driver rejects it.
static bool encode_map(CUtensorMap* m, CUtensorMapDataType type, const void* base, const cuuint64_t (&dims)[3],
                       const cuuint64_t (&strides)[2], const cuuint32_t (&box)[3]) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, type, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared-memory plan: header [0, hdr) (barriers and counters; for a paged
// cache also the split's first block rows), tables [tb_off, tb_off + 64 KB)
// at the first shared address past the header that is a multiple of 65536,
// stage buffers (128-byte aligned) in the space below and above the tables.
// The most stages that fit, a multiple of the group count and at least two
// per group.
static bool plan_smem(FastArgs& f, int base, int max_dyn, int kbytes, int vbytes, int nbytes, int hdr) {
  const int tb_abs = (base + hdr + FA_TABLE_BYTES - 1) & ~(FA_TABLE_BYTES - 1);  // the first boundary past the header
  const int tb_off = tb_abs - base;
  if (tb_off + FA_TABLE_BYTES > max_dyn) return false;
  for (int ns = FA_MAX_STAGES; ns >= 2 * f.n_groups; --ns) {
    if (ns % f.n_groups) continue;
    int lo[2] = {hdr, tb_off + FA_TABLE_BYTES}, hi[2] = {tb_off, max_dyn};
    auto take = [&](int bytes, int* out) {
      for (int r = 0; r < 2; ++r) {
        const int at = (lo[r] + 127) & ~127;
        if (at + bytes <= hi[r]) {
          *out = at;
          lo[r] = at + bytes;
          return true;
        }
      }
      return false;
    };
    bool ok = true;
    for (int s = 0; s < ns && ok; ++s) ok = take(kbytes, &f.kbuf[s]);
    for (int s = 0; s < ns && ok; ++s) ok = take(vbytes, &f.vbuf[s]);
    for (int s = 0; s < ns && ok; ++s) ok = take(nbytes, &f.knb[s]);
    for (int s = 0; s < ns && ok; ++s) ok = take(nbytes, &f.vnb[s]);
    if (ok) {
      f.n_stages = ns;
      f.tb_off = tb_off;
      return true;
    }
  }
  return false;
}

// The launch geometry that depends only on the shapes and the device's
// shared memory: warps per tile and groups, the V row pitch, the paged
// block-row cache, the stage buffers and the table region. False when no plan
// of at least two stages per group fits.
static bool fast_plan(FastArgs& f, int d, int hw, int nt, bool paged, int reserved, int max_dyn) {
  const int pk = d / 2, pv = d / 4;
  f.wpt = hw * nt;
  f.n_groups = FA_WARPS / f.wpt;
  f.vpitch = hw * pv + 16;
  const int np = fa_norm_pitch(hw);
  const int kbytes = ATT_TILE * hw * pk, vbytes = ATT_TILE * f.vpitch, nbytes = ATT_TILE * np * 4;
  // paged: 2 KB after the 128-byte header hold the rows of the split's first
  // 512 blocks, so the issuing thread reads them from shared memory
  f.pg_off = 128;
  f.pg_cap = paged ? 512 : 0;
  if (!plan_smem(f, reserved, max_dyn, kbytes, vbytes, nbytes, 128 + 4 * f.pg_cap)) return false;
  f.smem_base = (uint32_t)reserved;
  f.tile_bytes = (uint32_t)(kbytes + vbytes + 2 * nbytes);
  return true;
}

}  // namespace tq

using namespace tq;

bool tq_attend_fast_plan(int d, int hw, int nt, int paged, int reserved, int max_dyn, int32_t* out) {
  if ((d != 128 && d != 256) || (hw != 4 && hw != 8 && hw != 16) || (nt != 1 && nt != 2) ||
      FA_WARPS % (hw * nt) != 0)
    return false;
  FastArgs f;
  if (!fast_plan(f, d, hw, nt, paged != 0, reserved, max_dyn)) return false;
  const int np = fa_norm_pitch(hw);
  out[0] = f.n_stages;
  out[1] = f.n_groups;
  out[2] = f.tb_off;
  out[3] = FA_TABLE_BYTES;
  out[4] = 128 + 4 * f.pg_cap;  // header and paged block-row cache
  out[5] = ATT_TILE * hw * (d / 2);
  out[6] = ATT_TILE * f.vpitch;
  out[7] = ATT_TILE * np * 4;
  for (int s = 0; s < FA_MAX_STAGES; ++s) {
    const bool used = s < f.n_stages;
    out[8 + s] = used ? f.kbuf[s] : -1;
    out[8 + FA_MAX_STAGES + s] = used ? f.vbuf[s] : -1;
    out[8 + 2 * FA_MAX_STAGES + s] = used ? f.knb[s] : -1;
    out[8 + 3 * FA_MAX_STAGES + s] = used ? f.vnb[s] : -1;
  }
  return true;
}

cudaError_t tq_launch_attend_fast(AttnArgs& a, int d, int k_bits, int v_bits, int sm_count, cudaStream_t st) {
  if (k_bits != 4 || v_bits != 2 || (d != 128 && d != 256)) return cudaErrorNotSupported;
  const int nt = a.g > 4 ? 2 : 1;
  // kv heads per CTA: 8 or 16 warps per tile, norm rows of whole 16-byte units
  int hw = 0;
  for (int cand : {8 / nt, 16 / nt}) {
    if (cand % 4 == 0 && a.hkv % cand == 0) {
      hw = cand;
      break;
    }
  }
  if (hw == 0) return cudaErrorNotSupported;
  const int pk = d / 2, pv = d / 4;
  const int hg = a.hkv / hw;
  const bool paged = a.block_tables != nullptr;
  const int64_t rows = paged ? a.num_blocks * ATT_BLOCK : (int64_t)a.B * a.s_max;
  if (rows + 2 * ATT_TILE >= ((int64_t)1 << 31)) return cudaErrorNotSupported;  // int32 coordinates
  for (const void* p : {(const void*)a.k_packed, (const void*)a.v_packed, (const void*)a.k_norms,
                        (const void*)a.v_norms})
    if (reinterpret_cast<uintptr_t>(p) % 16) return cudaErrorNotSupported;

  int dev = 0, reserved = 0, max_dyn = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorUnknown;
  if (cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_dyn, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return cudaErrorUnknown;

  FastArgs f;
  if (!fast_plan(f, d, hw, nt, paged, reserved, max_dyn)) return cudaErrorNotSupported;
  const int np = fa_norm_pitch(hw);
  // the rotated queries (before the tables) and the group merge (after) use the table region
  if (hw * a.g * d * 4 > FA_TABLE_BYTES) return cudaErrorNotSupported;
  if ((f.n_groups - 1) * f.wpt * 32 * (d / 8 + 2) * 4 > FA_TABLE_BYTES) return cudaErrorNotSupported;

  const cuuint64_t R = (cuuint64_t)rows, HG = (cuuint64_t)hg;
  // positions per box: a tile, or one block of a paged cache (two boxes per tile)
  const cuuint32_t BP = paged ? (cuuint32_t)ATT_BLOCK : (cuuint32_t)ATT_TILE;
  f.paged = paged ? 1 : 0;
  const auto U64 = CU_TENSOR_MAP_DATA_TYPE_UINT64, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // K: (row bytes, position, kv head) with the head stride inside the
  // position stride, so one box lands as [head][position][row]; where the
  // driver refuses that order, one (row, head, position) box per head.
  f.k_head_copies = 0;
  if (!encode_map(&f.tm_k, U64, a.k_packed, {(cuuint64_t)pk / 8, R, (cuuint64_t)a.hkv},
                  {(cuuint64_t)a.hkv * pk, (cuuint64_t)pk}, {(cuuint32_t)pk / 8, BP, (cuuint32_t)hw})) {
    if (paged) return cudaErrorNotSupported;  // the generic kernel takes it
    f.k_head_copies = 1;
    if (!encode_map(&f.tm_k, U64, a.k_packed, {(cuuint64_t)pk / 8, (cuuint64_t)a.hkv, R},
                    {(cuuint64_t)pk, (cuuint64_t)a.hkv * pk}, {(cuuint32_t)pk / 8, 1, ATT_TILE}))
      return cudaErrorNotSupported;
  }
  if (!encode_map(&f.tm_v, U64, a.v_packed, {(cuuint64_t)hw * pv / 8, HG, R},
                  {(cuuint64_t)hw * pv, (cuuint64_t)a.hkv * pv}, {(cuuint32_t)f.vpitch / 8, 1, BP}) ||
      !encode_map(&f.tm_kn, F32, a.k_norms, {(cuuint64_t)hw, HG, R}, {(cuuint64_t)hw * 4, (cuuint64_t)a.hkv * 4},
                  {(cuuint32_t)np, 1, BP}) ||
      !encode_map(&f.tm_vn, F32, a.v_norms, {(cuuint64_t)hw, HG, R}, {(cuuint64_t)hw * 4, (cuuint64_t)a.hkv * 4},
                  {(cuuint32_t)np, 1, BP}))
    return cudaErrorNotSupported;

  // the fast kernel's own split (one CTA per SM and kv-head group); the
  // workspace was laid out for the generic kernel's a.n_split, so a larger
  // split count would overrun it: leave such a launch to the generic kernel
  int n_split = 0, chunk = 0;
  attn_split_for(sm_count / hg, a.B, a.s_max, &n_split, &chunk);
  if (n_split > a.n_split) return cudaErrorNotSupported;
  a.nt = nt;
  a.hw_max = hw;
  a.n_split = n_split;
  a.chunk = chunk;
  f.a = a;
  void (*kern)(FastArgs) = nullptr;
  if (d == 128) kern = hw == 4 ? attend_fast_kernel<128, 4> : hw == 8 ? attend_fast_kernel<128, 8> : attend_fast_kernel<128, 16>;
  else kern = hw == 4 ? attend_fast_kernel<256, 4> : hw == 8 ? attend_fast_kernel<256, 8> : attend_fast_kernel<256, 16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.n_split, a.B, hg), FA_WARPS * 32, max_dyn, st>>>(f);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return tq_launch_attend_combine(a, d, st);
}
