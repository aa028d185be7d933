// Decode-step attention over packed caches, specialised for 4-bit keys and
// 2-bit values (the asymmetric K/V split of the "KVarN" and "aither-kvcache"
// pages) at head_dim 128 or 256.
//
// Same mathematics as the generic kernel (tq_attend.cu, after the
// "aither-kvcache" page, section "Zero-buffer fused attention", and
// "TurboQuant efficient inference", section "2. A fused decode path"):
// scores against codebook values with a rotated query, values accumulated in
// the rotated domain, one inverse rotation in the split merge. What differs
// is how the work is laid out on the SM:
//
//  * One CTA of 16 warps per SM, 227 KB of shared memory: a 64 KB lookup
//    table region and up to 8 tiles of 32 positions in flight. A tile (the
//    K codes, V codes, K norms and V norms of 32 positions x the CTA's kv
//    heads) arrives as four 3-D tensor copies (TMA, no multicast); V rows are
//    padded by 16 bytes (the copy box is wider than the tensor and the
//    excess is zero-filled) so that the fragment loads of a warp hit
//    distinct banks.
//  * A warp owns one kv head (and one group of 4 query heads); the warps of
//    a tile form a group, and with 8 warps per tile the two groups take
//    alternate tiles. The last warp of a group to finish a stage refills it.
//  * Table lookups cost one PRMT + one LDS: the 64 KB table region starts at
//    a shared address that is a multiple of 65536, entries are 256 bytes
//    apart, so the address is (region | code byte << 8 | lane offset), and
//    one byte permute merges a code byte with a per-lane constant holding
//    the region and lane bits.
//      - K: entry = one code byte (two 4-bit codes) -> fp16 pair, 32 lane
//        copies in bytes [0, 128) of the entry.
//      - V: entry = two 2-bit codes of one position | two of the next
//        position -> the two fp16 pairs (position 2t, 2t+1) of two dims,
//        i.e. two A-fragment registers of the value MMA, 16 lane copies in
//        bytes [128, 256). The index bytes come from two position words with
//        two LOP3 per four entries.
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

struct FastArgs {
  CUtensorMap tm_k;   // K codes  [rows][head groups][hw * D/2 bytes] as u64
  CUtensorMap tm_v;   // V codes  [rows][head groups][hw * D/4 bytes] as u64
  CUtensorMap tm_kn;  // K norms  [rows][head groups][hw] f32
  CUtensorMap tm_vn;  // V norms
  AttnArgs a;
  uint32_t smem_base;  // shared address the dynamic region must start at
  int tb_off;          // offset of the table region (its shared address is a multiple of 65536)
  int kbuf[FA_MAX_STAGES], vbuf[FA_MAX_STAGES], knb[FA_MAX_STAGES], vnb[FA_MAX_STAGES];
  int n_stages;  // a multiple of n_groups
  int n_groups;  // warp groups taking alternate tiles
  int wpt;       // warps per tile: hw * nt
  int vpitch;    // bytes per V position row in shared memory (hw * D/4 + 16)
  uint32_t tile_bytes;
};

TQ_DEV void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Table loads: the tables are constant once built, so these need no ordering
// beyond their address dependencies.
TQ_DEV uint32_t lds_tab32(uint32_t addr) {
  uint32_t r;
  asm("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}
TQ_DEV uint2 lds_tab64(uint32_t addr) {
  uint2 r;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
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
  const __half h = __float2half_rn(v);
  const __half l = __float2half_rn(v - __half2float(h));
  return (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
}

template <int D>
__global__ void __launch_bounds__(FA_WARPS * 32, 1) attend_fast_kernel(const __grid_constant__ FastArgs f) {
  constexpr int PK = D / 2;   // K bytes per head row
  constexpr int PV = D / 4;   // V bytes per head row
  constexpr int NB = D / 16;  // k-blocks of the score MMA = m-blocks of the value MMA
  constexpr int KQW = D / 32; // words of a K row per lane (a quarter of the row)
  constexpr int VQW = (D / 32 + 3) / 4;  // words of a V row per lane (an eighth)
  const AttnArgs& a = f.a;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) != f.smem_base) {  // the table trick needs the planned addresses
    if (threadIdx.x == 0) record_error(a.err, TQ_DEVERR_SMEM_LAYOUT);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int split = blockIdx.x, b = blockIdx.y, hgrp = blockIdx.z;
  const int hw = a.hw_max, g = a.g, nt = a.nt, NS = f.n_stages;
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
  const int row0 = (int)((int64_t)b * a.s_max + s0);  // first cache row of this split
  auto issue = [&](int tile) {  // one thread
    const int s = tile % NS;
    const uint32_t bar = smem_u32(&bars[s]);
    mbar_arrive_expect_tx(bar, f.tile_bytes);
    const int row = row0 + tile * ATT_TILE;
    tma_load_3d(smem_u32(smem + f.kbuf[s]), &f.tm_k, 0, hgrp, row, bar);
    tma_load_3d(smem_u32(smem + f.vbuf[s]), &f.tm_v, 0, hgrp, row, bar);
    tma_load_3d(smem_u32(smem + f.knb[s]), &f.tm_kn, 0, hgrp, row, bar);
    tma_load_3d(smem_u32(smem + f.vnb[s]), &f.tm_vn, 0, hgrp, row, bar);
    issued[s] += 1;
  };
  if (threadIdx.x == 0) {
    for (int t = 0; t < NS && t < ntiles; ++t) issue(t);
  }

  // rotated, scaled queries of the CTA's heads (q~ = H_pm D_K q), built in the
  // table region before the tables
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
  __syncthreads();  // the query buffer becomes the tables

  const uint32_t tb = f.smem_base + (uint32_t)f.tb_off;  // a multiple of 65536
  {
    uint32_t* tw = reinterpret_cast<uint32_t*>(smem + f.tb_off);
    for (int e = threadIdx.x; e < 256 * 32; e += blockDim.x) {
      const int en = e >> 5;
      tw[en * 64 + (e & 31)] = pack_half2(a.k_levels[en & 15], a.k_levels[en >> 4]);
    }
    for (int e = threadIdx.x; e < 256 * 16; e += blockDim.x) {
      const int en = e >> 4;
      // index bits: [1:0] dim d0 / position A, [3:2] d1 / A, [5:4] d0 / B, [7:6] d1 / B
      uint2* p = reinterpret_cast<uint2*>(smem + f.tb_off + en * 256 + 128 + (e & 15) * 8);
      *p = make_uint2(pack_half2(a.v_levels[en & 3], a.v_levels[(en >> 4) & 3]),
                      pack_half2(a.v_levels[(en >> 2) & 3], a.v_levels[en >> 6]));
    }
  }
  __syncthreads();

  const uint32_t LK = tb | (uint32_t)(lane * 4);                 // byte 0 = lane copy, bytes 2-3 = region
  const uint32_t LV = tb | (uint32_t)(128 + (lane & 15) * 8);
  const int kcol = hl * PK + tq * (D / 8);   // this lane's quarter of its head's K row
  const int vcol = hl * PV + gq * (D / 32);  // this lane's eighth of its head's V row
  const int vp = f.vpitch;

  float m_run = -INFINITY, l_run = 0.f;
  float acc[NB][4];
#pragma unroll
  for (int i = 0; i < NB; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;

  for (int tile = grp; tile < ntiles; tile += f.n_groups) {
    const int s = tile % NS;
    const bool ok =
        __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&bars[s]), (uint32_t)(tile / NS) & 1u, a.wait_limit));
    if (!ok) {
      if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
      break;
    }
    const uint8_t* kst = smem + f.kbuf[s];
    const uint8_t* vst = smem + f.vbuf[s];
    const float* kns = reinterpret_cast<const float*>(smem + f.knb[s]);
    const float* vns = reinterpret_cast<const float*>(smem + f.vnb[s]);
    const int nv = (int)min64(ATT_TILE, s1 - (s0 + (int64_t)tile * ATT_TILE));

    // ---- scores: rows = positions, columns = 4 query heads x (hi, lo)
    float sc[2][2];
#pragma unroll
    for (int mb16 = 0; mb16 < 2; ++mb16) {
      const int r0 = mb16 * 16 + gq;
      uint32_t kw0[KQW], kw1[KQW];
#pragma unroll
      for (int w = 0; w < KQW; w += 4) {
        const uint4 x0 = *reinterpret_cast<const uint4*>(kst + r0 * (hw * PK) + kcol + 4 * w);
        const uint4 x1 = *reinterpret_cast<const uint4*>(kst + (r0 + 8) * (hw * PK) + kcol + 4 * w);
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
      sc[mb16][0] = (c[0] + c[1]) * kns[r0 * hw + hl];
      sc[mb16][1] = (c[2] + c[3]) * kns[(r0 + 8) * hw + hl];
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
        float pv = p * vns[row * hw + hl];
        if (ragged && row >= nv) pv = 0.f;
        bp[mb16][r] = transpose8x8(split_hi_lo(pv));
      }
    }

    // ---- values: acc[dims x columns] += V^T[dims x 16 positions] * P[16 positions x columns]
#pragma unroll
    for (int mb16 = 0; mb16 < 2; ++mb16) {
      const uint8_t* ra = vst + (mb16 * 16 + 2 * tq) * vp + vcol;  // position 2tq of the block
      uint32_t lo0[VQW], hi0[VQW], lo1[VQW], hi1[VQW];
#pragma unroll
      for (int w = 0; w < VQW; ++w) {
        const uint32_t wa0 = reinterpret_cast<const uint32_t*>(ra)[w];
        const uint32_t wb0 = reinterpret_cast<const uint32_t*>(ra + vp)[w];
        const uint32_t wa1 = reinterpret_cast<const uint32_t*>(ra + 8 * vp)[w];
        const uint32_t wb1 = reinterpret_cast<const uint32_t*>(ra + 9 * vp)[w];
        // byte k: low nibble of A's byte k | low nibble of B's byte k << 4 (and the high nibbles)
        lo0[w] = (wa0 & 0x0F0F0F0Fu) | ((wb0 << 4) & 0xF0F0F0F0u);
        hi0[w] = ((wa0 >> 4) & 0x0F0F0F0Fu) | (wb0 & 0xF0F0F0F0u);
        lo1[w] = (wa1 & 0x0F0F0F0Fu) | ((wb1 << 4) & 0xF0F0F0F0u);
        hi1[w] = ((wa1 >> 4) & 0x0F0F0F0Fu) | (wb1 & 0xF0F0F0F0u);
      }
#pragma unroll
      for (int mb = 0; mb < NB; ++mb) {
        const int byte = mb >> 1, w = byte >> 2;
        const uint32_t sel = 0x7604u | ((uint32_t)(byte & 3) << 4);
        const uint2 x = lds_tab64(__byte_perm((mb & 1) ? hi0[w] : lo0[w], LV, sel));
        const uint2 y = lds_tab64(__byte_perm((mb & 1) ? hi1[w] : lo1[w], LV, sel));
        mma16816(acc[mb], x.x, x.y, y.x, y.y, bp[mb16][0], bp[mb16][1]);
      }
    }

    // this warp is done with the stage; the group's last warp refills it
    __syncwarp();
    if (tile + NS < ntiles && lane == 0) {
      __threadfence_block();
      if (atomicAdd(&cnt[s], 1u) == (uint32_t)(f.wpt - 1)) {
        cnt[s] = 0;
        issue(tile + NS);
      }
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

// 3-D map over [rows][head groups][inner] with the given element type; box =
// (box_inner, 1, ATT_TILE).
static bool encode_map(CUtensorMap* m, CUtensorMapDataType type, int esize, const void* base, uint64_t inner,
                       uint64_t groups, uint64_t rows, uint64_t group_stride, uint64_t row_stride,
                       uint32_t box_inner) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {inner, groups, rows};
  const cuuint64_t strides[2] = {group_stride, row_stride};
  const cuuint32_t box[3] = {box_inner, 1, ATT_TILE};
  const cuuint32_t estr[3] = {1, 1, 1};
  (void)esize;
  return enc(m, type, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared-memory plan: header [0, 128), tables [tb_off, tb_off + 64 KB) at a
// shared address that is a multiple of 65536, stage buffers (128-byte
// aligned) in the space below and above the tables. The most stages that
// fit, a multiple of the group count and at least two per group.
static bool plan_smem(FastArgs& f, int base, int max_dyn, int kbytes, int vbytes, int nbytes) {
  const int tb_abs = (base + FA_TABLE_BYTES - 1) & ~(FA_TABLE_BYTES - 1);
  const int tb_off = tb_abs - base;
  if (tb_off < 128 || tb_off + FA_TABLE_BYTES > max_dyn) return false;
  for (int ns = FA_MAX_STAGES; ns >= 2 * f.n_groups; --ns) {
    if (ns % f.n_groups) continue;
    int lo[2] = {128, tb_off + FA_TABLE_BYTES}, hi[2] = {tb_off, max_dyn};
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

}  // namespace tq

using namespace tq;

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
  const int64_t rows = (int64_t)a.B * a.s_max;
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
  f.wpt = hw * nt;
  f.n_groups = FA_WARPS / f.wpt;
  f.vpitch = hw * pv + 16;
  const int kbytes = ATT_TILE * hw * pk, vbytes = ATT_TILE * f.vpitch, nbytes = ATT_TILE * hw * 4;
  if (!plan_smem(f, reserved, max_dyn, kbytes, vbytes, nbytes)) return cudaErrorNotSupported;
  f.smem_base = (uint32_t)reserved;
  f.tile_bytes = (uint32_t)(kbytes + vbytes + 2 * nbytes);
  // the rotated queries (before the tables) and the group merge (after) use the table region
  if (hw * a.g * d * 4 > FA_TABLE_BYTES) return cudaErrorNotSupported;
  if ((f.n_groups - 1) * f.wpt * 32 * (d / 8 + 2) * 4 > FA_TABLE_BYTES) return cudaErrorNotSupported;

  if (!encode_map(&f.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, a.k_packed, (uint64_t)hw * pk / 8, hg, rows,
                  (uint64_t)hw * pk, (uint64_t)a.hkv * pk, (uint32_t)(hw * pk / 8)) ||
      !encode_map(&f.tm_v, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, a.v_packed, (uint64_t)hw * pv / 8, hg, rows,
                  (uint64_t)hw * pv, (uint64_t)a.hkv * pv, (uint32_t)(f.vpitch / 8)) ||
      !encode_map(&f.tm_kn, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.k_norms, (uint64_t)hw, hg, rows,
                  (uint64_t)hw * 4, (uint64_t)a.hkv * 4, (uint32_t)hw) ||
      !encode_map(&f.tm_vn, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.v_norms, (uint64_t)hw, hg, rows,
                  (uint64_t)hw * 4, (uint64_t)a.hkv * 4, (uint32_t)hw))
    return cudaErrorNotSupported;

  a.nt = nt;
  a.hw_max = hw;
  attn_split_for(sm_count / hg, a.B, a.s_max, &a.n_split, &a.chunk);
  f.a = a;
  auto kern = d == 128 ? attend_fast_kernel<128> : attend_fast_kernel<256>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.n_split, a.B, hg), FA_WARPS * 32, max_dyn, st>>>(f);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return tq_launch_attend_combine(a, d, st);
}
