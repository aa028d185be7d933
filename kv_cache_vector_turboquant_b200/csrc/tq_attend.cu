// Fused decode-step attention over packed K/V caches.
//
// Method ("aither-kvcache" PyPI page, section "Zero-buffer fused attention";
// "TurboQuant efficient inference", section "2. A fused decode path"): with
// k_hat_t = n_t D_K H (c_K[idx_t] / sqrt(d)), the score is
//   q . k_hat_t / sqrt(d) = (n_t / (d sqrt(d))) (H_pm D_K q) . c_K[idx_t],
// so the query is rotated once (q~ = H_pm D_K q) and scored against codebook
// values; the values are accumulated in the rotated domain,
//   acc = sum_t p_t n^V_t c_V[idx^V_t],   o = D_V H_pm (acc / l) / d,
// and rotated back once at the end.
//
// Split-S: the grid is (n_split, B, kv-head groups). Each CTA owns a chunk of
// cache positions of one sequence and a group of kv heads; each warp owns one
// kv head (and, for more than 4 query heads per kv head, one group of 4 query
// heads). Position rows of the group (contiguous in the [B, S, Hkv, P]
// layout) arrive in padded shared rows by 1-D bulk copies (TMA, no
// multicast) through a 2-stage mbarrier pipeline of 32-position tiles.
//
// Both contractions run on the tensor cores (mma.sync m16n8k16, fp16 inputs,
// f32 accumulation); the packed codes are turned into fp16 operand fragments
// in registers through lane-replicated shared tables indexed by two codes,
// never into fp16 tiles in memory:
//  * scores: A = 16 positions x 16 dims of K levels, B = 16 dims x 8 columns
//    holding the rotated query of 4 heads split as fp16 hi + lo parts (so the
//    query keeps ~22 bits); the two parts are summed from the accumulator.
//    The d dims are visited in a permuted order so that each thread's codes
//    are one contiguous quarter of the row; q~ uses the same order.
//  * values: A = 16 dims x 16 positions of V levels (dims permuted so each
//    thread's codes are a contiguous eighth of the row, and the accumulator
//    comes out in natural order), B = 16 positions x 8 columns of
//    p_t n^V_t split as fp16 hi + lo, transposed through a small per-warp
//    buffer.
// Online softmax in the exp2 domain per 32-position tile. The partial (max,
// sum, accumulator) of every split goes to the workspace; a second kernel
// merges the splits (log-sum-exp) and applies D_V H / d.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "tq_attend.cuh"

namespace tq {

template <int D, int KB, int VB>
struct AttCfg {
  static constexpr int PK = D * KB / 8;  // packed bytes of a K row (one head)
  static constexpr int PV = D * VB / 8;
  static constexpr int KT = PK / 4;  // K bytes per thread: a quarter of the row
  static constexpr int VT = PV / 8;  // V bytes per thread: an eighth of the row
  static constexpr int KW = (KT + 3) / 4 + 1;  // words holding a thread's K bits (+1 for straddling)
  static constexpr int VW = (VT + 3) / 4 + 1;
  static constexpr int KF = 2 * KB;  // bits of a two-code field
  static constexpr int VF = 2 * VB;
  static constexpr int LK2 = 1 << KF;  // two-code table entries
  static constexpr int LV2 = 1 << VF;
  static constexpr int NB = D / 16;  // k-blocks (scores) = m-blocks (values)
};

inline int round_units(int bytes, int unit, int mod, int rem) {
  int u = (bytes + unit - 1) / unit;
  while (u % mod != rem) ++u;
  return u * unit;
}

// Shared-memory layout of the partial kernel (bytes); identical on host and device.
struct AttSmem {
  int krow, vrow, stage, bar, cnt, st0, lutk, lutv, pw, nrm, qt, total;
  __host__ __device__ AttSmem(int D, int PK, int PV, int LK2, int lutv_bytes, int hw_max, int g) {
    // padded position rows: K rows a number of 16-byte units == 4 mod 8 apart,
    // V rows a number of words == 4 mod 16, so the fragment loads of a warp
    // fall in distinct banks
    int u = (hw_max * PK + 15) / 16;
    while (u % 8 != 4) ++u;
    krow = u * 16;
    int w = (hw_max * PV + 3) / 4;
    while (w % 16 != 4) ++w;
    vrow = w * 4;
    stage = ATT_TILE * (krow + vrow);
    bar = 0;                                   // full[stage] mbarriers
    cnt = 64;                                  // per stage: warps done with it
    st0 = 128;
    lutk = st0 + ATT_STAGES * stage;
    lutv = lutk + LK2 * 32 * 4;
    pw = lutv + lutv_bytes;                    // per warp: 2 blocks x 8 cols x 16 pos fp16
    nrm = pw + ATT_WARPS * 2 * 8 * 16 * 2;     // per warp: K and V norms of the tile
    // rotated queries of the CTA (f32), only needed before the tables are
    // built: they share the tables' space when it is large enough
    const int qbytes = hw_max * g * D * 4;
    const int tables = LK2 * 32 * 4 + lutv_bytes;
    qt = qbytes <= tables ? lutk : nrm + ATT_WARPS * 2 * ATT_TILE * 4;
    total = (qt == lutk ? nrm + ATT_WARPS * 2 * ATT_TILE * 4 : qt + qbytes);
  }
};

// Value table for 2-bit values: one entry per byte (4 codes) holding their 4
// fp16 levels, replicated 8 times (copy = lane & 7); other widths use a
// lane-replicated table of two-code entries.
template <int VB>
struct VTable {
  static constexpr bool BYTE = (VB == 2);
  static constexpr int BYTES = BYTE ? 256 * 8 * 8 : (1 << (2 * VB)) * 32 * 4;
};

// `NB` bits at bit offset `off` of a little-endian word stream.
template <int NB, int N>
TQ_DEV uint32_t bits_at(const uint32_t (&w)[N], int off) {
  uint32_t f = w[off >> 5] >> (off & 31);
  if ((off & 31) + NB > 32) f |= w[(off >> 5) + 1] << (32 - (off & 31));
  return f & ((1u << NB) - 1u);
}

// NBYTES bytes of shared memory starting at p (at least 2-byte aligned) as a
// little-endian word stream w[0..].
template <int NBYTES, int NW>
TQ_DEV void load_bytes(uint32_t (&w)[NW], const uint8_t* p) {
  if (NBYTES % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NBYTES / 16; ++i) {
      const uint4 r = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = r.x;
      w[4 * i + 1] = r.y;
      w[4 * i + 2] = r.z;
      w[4 * i + 3] = r.w;
    }
  } else if (NBYTES % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NBYTES / 8; ++i) {
      const uint2 r = reinterpret_cast<const uint2*>(p)[i];
      w[2 * i] = r.x;
      w[2 * i + 1] = r.y;
    }
  } else if (NBYTES % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NBYTES / 4; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  } else {
    const uintptr_t addr = reinterpret_cast<uintptr_t>(p);
    const uint32_t* base = reinterpret_cast<const uint32_t*>(addr & ~uintptr_t(3));
    const uint32_t sh = (uint32_t)(addr & 3) * 8u;
    uint32_t raw[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) raw[i] = base[i];
#pragma unroll
    for (int i = 0; i + 1 < NW; ++i) w[i] = __funnelshift_r(raw[i], raw[i + 1], sh);
    w[NW - 1] = raw[NW - 1] >> sh;
  }
}

template <int D, int KB, int VB>
__global__ void __launch_bounds__(ATT_WARPS * 32, 2) attend_partial_kernel(const __grid_constant__ AttnArgs a) {
  using Cfg = AttCfg<D, KB, VB>;
  constexpr int PK = Cfg::PK, PV = Cfg::PV, KT = Cfg::KT, VT = Cfg::VT, NB = Cfg::NB;
  constexpr int KF = Cfg::KF, VF = Cfg::VF;
  extern __shared__ __align__(128) uint8_t smem[];
  using VT_ = VTable<VB>;
  const AttSmem L(D, PK, PV, Cfg::LK2, VT_::BYTES, a.hw_max, a.g);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row group and column pair
  const int split = blockIdx.x, b = blockIdx.y;
  const int hk0 = blockIdx.z * a.hw_max;
  const int hw = min(a.hw_max, a.hkv - hk0);  // kv heads in this CTA
  const int g = a.g;
  const int hl = warp / a.nt, nt = warp % a.nt;  // this warp's kv head (local) and column tile
  const bool head_ok = hl < hw;
  const int hk = hk0 + hl;

  int64_t pos = a.positions[b];
  if (pos > a.s_max) {
    if (threadIdx.x == 0 && split == 0 && blockIdx.z == 0) record_error(a.err, TQ_DEVERR_POS_RANGE);
    pos = a.s_max;
  }
  const int64_t s0 = (int64_t)split * a.chunk;
  const int64_t s1 = min64(s0 + a.chunk, pos);
  const int64_t npos = s1 > s0 ? s1 - s0 : 0;
  const int ntiles = (int)((npos + ATT_TILE - 1) / ATT_TILE);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  float* qt = reinterpret_cast<float*>(smem + L.qt);
  __half* pwb = reinterpret_cast<__half*>(smem + L.pw) + warp * 2 * 8 * 16;
  float* nks = reinterpret_cast<float*>(smem + L.nrm) + warp * 2 * ATT_TILE;
  float* nvs = nks + ATT_TILE;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + L.cnt);
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      cnt[s] = 0;
    }
    fence_mbar_init();
  }
  __syncthreads();

  // producer: the issuing warp's lanes copy one K and one V row per position of a tile
  const uint32_t krow_bytes = (uint32_t)(hw * PK), vrow_bytes = (uint32_t)(hw * PV);
  auto issue = [&](int tile, int stage) {
    const int64_t t0 = s0 + (int64_t)tile * ATT_TILE;
    const int nv = (int)min64(ATT_TILE, s1 - t0);
    const uint32_t bar = smem_u32(&bars[stage]);
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)nv * (krow_bytes + vrow_bytes));
    __syncwarp();
    if (lane < nv) {
      const int64_t row = attn_pos_row(a, b, t0 + lane) * a.hkv + hk0;
      uint8_t* st = smem + L.st0 + stage * L.stage;
      bulk_g2s(smem_u32(st + lane * L.krow), a.k_packed + row * PK, krow_bytes, bar);
      bulk_g2s(smem_u32(st + ATT_TILE * L.krow + lane * L.vrow), a.v_packed + row * PV, vrow_bytes, bar);
    }
  };
  if (warp == 0) {
    for (int s = 0; s < ATT_STAGES && s < ntiles; ++s) issue(s, s);
  }

  // rotated, scaled queries of this CTA's heads: q~ = H_pm D_K q * q_scale
  const int nq = hw * g;
  const int qh0 = hk0 * g;
  for (int e = threadIdx.x; e < nq * D; e += blockDim.x) {
    const int i = e % D;
    const __half hv = a.q[((int64_t)b * a.hq + qh0) * D + e];
    const uint32_t sb = (a.k_sign_h2[i >> 1] >> (15 + 16 * (i & 1))) & 1u;
    const float x = __half2float(hv);
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

  // B fragments of the score MMA: column gq = (query head nt*4 + gq/2, hi or lo
  // part), rows = dims pi(kb, k) = tq*D/4 + 4*kb + k' for the fragment's k
  uint32_t bq[NB][2];
  {
    const int j = nt * 4 + (gq >> 1);
    const bool lo = gq & 1;
    const float* qrow = qt + (hl * g + (j < g ? j : 0)) * D;
#pragma unroll
    for (int kb = 0; kb < NB; ++kb) {
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const int d0 = tq * (D / 4) + 4 * kb + 2 * e2;
        float v0 = 0.f, v1 = 0.f;
        if (head_ok && j < g) {
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

  __syncthreads();  // every warp has its query fragments: the query buffer may be reused
  {
    // two-code K table: entry f = code_lo | code_hi << bits -> fp16 pair (c[lo], c[hi])
    uint32_t* lk = reinterpret_cast<uint32_t*>(smem + L.lutk);
    for (int e = threadIdx.x; e < Cfg::LK2 * 32; e += blockDim.x) {
      const int f = e >> 5;
      lk[e] = pack_half2(a.k_levels[f & ((1 << KB) - 1)], a.k_levels[f >> KB]);
    }
    if (VT_::BYTE) {
      uint2* lv = reinterpret_cast<uint2*>(smem + L.lutv);
      for (int e = threadIdx.x; e < 256 * 8; e += blockDim.x) {
        const int f = e >> 3;
        lv[e] = make_uint2(pack_half2(a.v_levels[f & 3], a.v_levels[(f >> 2) & 3]),
                           pack_half2(a.v_levels[(f >> 4) & 3], a.v_levels[f >> 6]));
      }
    } else {
      uint32_t* lv = reinterpret_cast<uint32_t*>(smem + L.lutv);
      for (int e = threadIdx.x; e < Cfg::LV2 * 32; e += blockDim.x) {
        const int f = e >> 5;
        lv[e] = pack_half2(a.v_levels[f & ((1 << VB) - 1)], a.v_levels[f >> VB]);
      }
    }
  }
  __syncthreads();

  const uint32_t lutk_lane = smem_u32(smem + L.lutk) + lane * 4u;
  const uint32_t lutv_lane = smem_u32(smem + L.lutv) + (VT_::BYTE ? (lane & 7) * 8u : lane * 4u);
  float m_run = -INFINITY, l_run = 0.f;
  float acc[NB][4];
#pragma unroll
  for (int i = 0; i < NB; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;

  // norms of the first tile (lane = position), then prefetched one tile ahead
  float nk_next = 0.f, nv_next = 0.f;
  if (head_ok && ntiles > 0 && lane < min64(ATT_TILE, npos)) {
    const int64_t row = attn_pos_row(a, b, s0 + lane) * a.hkv + hk;
    nk_next = __ldg(a.k_norms + row);
    nv_next = __ldg(a.v_norms + row);
  }

  uint32_t parity = 0;
  for (int tile = 0; tile < ntiles; ++tile) {
    const int stage = tile % ATT_STAGES;
    const int64_t t0 = s0 + (int64_t)tile * ATT_TILE;
    const int nv = (int)min64(ATT_TILE, s1 - t0);
    nks[lane] = nk_next;
    nvs[lane] = nv_next;
    if (head_ok && tile + 1 < ntiles) {
      const int64_t t1 = t0 + ATT_TILE;
      if (lane < min64(ATT_TILE, s1 - t1)) {
        const int64_t row = attn_pos_row(a, b, t1 + lane) * a.hkv + hk;
        nk_next = __ldg(a.k_norms + row);
        nv_next = __ldg(a.v_norms + row);
      }
    }
    // each warp waits for the tile on its own (no CTA-wide barrier in the
    // loop); its lanes act on one agreed outcome
    const bool ok =
        __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u, a.wait_limit));
    if (!ok) {
      // the stage never filled: record it and leave the loop; the other warps
      // then find their next stage unfilled too, since this warp never
      // releases it
      if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
      break;
    }
    parity ^= 1u << stage;
    const uint8_t* kst = smem + L.st0 + stage * L.stage;
    const uint8_t* vst = kst + ATT_TILE * L.krow;

    if (head_ok) {
      // ---- scores on the tensor cores: 2 blocks of 16 positions
      float sc[2][2];
#pragma unroll
      for (int mb16 = 0; mb16 < 2; ++mb16) {
        const int r0 = mb16 * 16 + gq, r1 = r0 + 8;
        uint32_t kw0[Cfg::KW], kw1[Cfg::KW];
        load_bytes<KT>(kw0, kst + r0 * L.krow + hl * PK + tq * KT);
        load_bytes<KT>(kw1, kst + r1 * L.krow + hl * PK + tq * KT);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kb = 0; kb < NB; ++kb) {
          const uint32_t a0 = lds32(bits_at<KF>(kw0, (2 * kb) * KF) * 128u + lutk_lane);
          const uint32_t a1 = lds32(bits_at<KF>(kw1, (2 * kb) * KF) * 128u + lutk_lane);
          const uint32_t a2 = lds32(bits_at<KF>(kw0, (2 * kb + 1) * KF) * 128u + lutk_lane);
          const uint32_t a3 = lds32(bits_at<KF>(kw1, (2 * kb + 1) * KF) * 128u + lutk_lane);
          mma16816(c, a0, a1, a2, a3, bq[kb][0], bq[kb][1]);
        }
        sc[mb16][0] = (r0 < nv) ? (c[0] + c[1]) * nks[r0] : -INFINITY;
        sc[mb16][1] = (r1 < nv) ? (c[2] + c[3]) * nks[r1] : -INFINITY;
      }
      // ---- online softmax (log2 domain) for query head nt*4 + tq
      const float mx = warp_max8(fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1])));
      const float mn = fmaxf(m_run, mx);
      float alpha = 1.f, p[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      if (mn != -INFINITY) {
        alpha = exp2f(m_run - mn);
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int r = 0; r < 2; ++r) p[i][r] = exp2f(sc[i][r] - mn);  // exp2(-inf) = 0
      }
      l_run = l_run * alpha + warp_sum8(p[0][0] + p[0][1] + p[1][0] + p[1][1]);
      m_run = mn;
#pragma unroll
      for (int i = 0; i < NB; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] *= alpha;
      // p * n^V as fp16 hi + lo, stored column-major [block][col][position]
#pragma unroll
      for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int pr = gq + 8 * r;
          const float pv = (i * 16 + pr < nv) ? p[i][r] * nvs[i * 16 + pr] : 0.f;
          const __half hi = __float2half_rn(pv);
          const __half lo = __float2half_rn(pv - __half2float(hi));
          pwb[(i * 8 + 2 * tq) * 16 + pr] = hi;
          pwb[(i * 8 + 2 * tq + 1) * 16 + pr] = lo;
        }
      }
      __syncwarp();
      // ---- values on the tensor cores: acc[dims x cols] += V^T[dims x 16 pos] * P'[16 pos x cols]
#pragma unroll
      for (int mb16 = 0; mb16 < 2; ++mb16) {
        const uint32_t* pcol = reinterpret_cast<const uint32_t*>(pwb + (mb16 * 8 + gq) * 16);
        const uint32_t bp0 = pcol[tq], bp1 = pcol[tq + 4];
        uint32_t vw[4][Cfg::VW];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = mb16 * 16 + 2 * tq + (j & 1) + 8 * (j >> 1);
          load_bytes<VT>(vw[j], vst + r * L.vrow + hl * PV + gq * VT);
        }
        if (VT_::BYTE) {
          // one byte = the 4 codes of M-blocks 2m (low pair) and 2m+1 (high pair)
#pragma unroll
          for (int m = 0; m < NB / 2; ++m) {
            uint2 lv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t byte = bits_at<8>(vw[j], 8 * m);
              asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lv[j].x), "=r"(lv[j].y) : "r"(byte * 64u + lutv_lane));
            }
            mma16816(acc[2 * m], __byte_perm(lv[0].x, lv[1].x, 0x5410), __byte_perm(lv[0].x, lv[1].x, 0x7632),
                     __byte_perm(lv[2].x, lv[3].x, 0x5410), __byte_perm(lv[2].x, lv[3].x, 0x7632), bp0, bp1);
            mma16816(acc[2 * m + 1], __byte_perm(lv[0].y, lv[1].y, 0x5410), __byte_perm(lv[0].y, lv[1].y, 0x7632),
                     __byte_perm(lv[2].y, lv[3].y, 0x5410), __byte_perm(lv[2].y, lv[3].y, 0x7632), bp0, bp1);
          }
        } else {
#pragma unroll
          for (int mb = 0; mb < NB; ++mb) {
            const uint32_t l0 = lds32(bits_at<VF>(vw[0], mb * VF) * 128u + lutv_lane);
            const uint32_t l1 = lds32(bits_at<VF>(vw[1], mb * VF) * 128u + lutv_lane);
            const uint32_t l2 = lds32(bits_at<VF>(vw[2], mb * VF) * 128u + lutv_lane);
            const uint32_t l3 = lds32(bits_at<VF>(vw[3], mb * VF) * 128u + lutv_lane);
            mma16816(acc[mb], __byte_perm(l0, l1, 0x5410), __byte_perm(l0, l1, 0x7632), __byte_perm(l2, l3, 0x5410),
                     __byte_perm(l2, l3, 0x7632), bp0, bp1);
          }
        }
      }
    }
    // this warp is done with the stage; the last of the CTA's warps to finish
    // it issues its refill
    __syncwarp();
    if (tile + ATT_STAGES < ntiles) {
      uint32_t last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(&cnt[stage], 1u) == ATT_WARPS - 1;
        if (last) cnt[stage] = 0;
      }
      if (__shfl_sync(0xffffffffu, last, 0)) issue(tile + ATT_STAGES, stage);
    }
  }

  // ---- partial results of this split: query head hk*g + nt*4 + tq
  const int j = nt * 4 + tq;
  if (head_ok && j < g) {
    const int h = hk * g + j;
    const int64_t idx = ((int64_t)b * a.hq + h) * a.n_split + split;
    if (gq == 0) {
      a.ws_m[idx] = m_run;
      a.ws_l[idx] = l_run;
    }
    float* dst = a.ws_acc + idx * D + gq * (D / 8);
#pragma unroll
    for (int mb = 0; mb < NB; ++mb) {
      dst[2 * mb] = acc[mb][0] + acc[mb][1];
      dst[2 * mb + 1] = acc[mb][2] + acc[mb][3];
    }
  }
}


// Merge the splits of one (sequence, query head) and rotate back:
// M = max_s m_s, w_s = 2^(m_s - M), o~ = sum_s w_s acc_s / sum_s w_s l_s,
// o = D_V H_pm o~ / d, rounded to fp16. One CTA of d threads per row.
template <int D>
__global__ void __launch_bounds__(D) attend_combine_kernel(const __grid_constant__ AttnArgs a) {
  // launched as a programmatic dependent of the partial kernel: wait until
  // that grid has completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float o[D];
  const int h = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
  const int64_t base = ((int64_t)b * a.hq + h) * a.n_split;
  float M = -INFINITY;
  for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, a.ws_m[base + s]);
  float lsum = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.n_split; ++s) {
      const float ms = a.ws_m[base + s];
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      lsum = fmaf(w, a.ws_l[base + s], lsum);
      acc = fmaf(w, a.ws_acc[(base + s) * D + i], acc);
    }
  }
  o[i] = lsum > 0.f ? acc / lsum : 0.f;
  __syncthreads();
#pragma unroll
  for (int hh = 1; hh < D; hh <<= 1) {
    float val = 0.f;
    const int partner = i ^ hh;
    const float mine = o[i], other = o[partner];
    val = (i & hh) ? other - mine : mine + other;
    __syncthreads();
    o[i] = val;
    __syncthreads();
  }
  const uint32_t sb = (a.v_sign_h2[i >> 1] >> (15 + 16 * (i & 1))) & 1u;
  const float r = o[i] * (1.0f / (float)D);
  a.out[((int64_t)b * a.hq + h) * D + i] = __float2half_rn(sb ? -r : r);
}

template <int D, int KB, int VB>
static cudaError_t launch_attend_t(const AttnArgs& a, cudaStream_t st, int dev) {
  using Cfg = AttCfg<D, KB, VB>;
  const AttSmem L(D, Cfg::PK, Cfg::PV, Cfg::LK2, VTable<VB>::BYTES, a.hw_max, a.g);
  cudaError_t e = cudaFuncSetAttribute(attend_partial_kernel<D, KB, VB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.n_split, a.B, (a.hkv + a.hw_max - 1) / a.hw_max);
  attend_partial_kernel<D, KB, VB><<<grid, ATT_WARPS * 32, L.total, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  (void)dev;
  return tq_launch_attend_combine(a, D, st);
}

}  // namespace tq

using namespace tq;

cudaError_t tq_launch_attend_combine(const AttnArgs& a, int d, cudaStream_t st) {
  const dim3 grid(a.hq, a.B);
  // programmatic dependent launch: the merge grid is set up while the
  // partial kernel runs and starts as its CTAs retire (it waits for the
  // partial grid's completion before reading the workspace)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(d);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (d == 64) return cudaLaunchKernelEx(&cfg, attend_combine_kernel<64>, a);
  if (d == 128) return cudaLaunchKernelEx(&cfg, attend_combine_kernel<128>, a);
  if (d == 256) return cudaLaunchKernelEx(&cfg, attend_combine_kernel<256>, a);
  return cudaErrorInvalidValue;
}

size_t tq_attend_workspace_bytes_impl(int B, int hq, int head_dim, int64_t s_max) {
  int ns = 0, chunk = 0;
  attn_split(B, s_max, &ns, &chunk);
  const size_t rows = (size_t)B * hq * ns;
  return 2 * align16(rows * 4) + rows * (size_t)head_dim * 4;
}

static tq_status launch_attend(const tq_ctx* k, const tq_ctx* v, const void* q, int B, int hq, int hkv,
                               const void* k_packed, const float* k_norms, const void* v_packed,
                               const float* v_norms, int64_t s_max, const int32_t* positions,
                               const int32_t* block_tables, int max_blocks, int64_t num_blocks, void* out,
                               void* workspace, size_t ws_bytes, void* stream) {
  const int d = k->d;
  const int g = hq / hkv;
  if (g > ATT_MAXG) return TQ_ERR_UNSUPPORTED;
  const int pk = d * k->bits / 8, pv = d * v->bits / 8;
  // position rows of a kv-head group are copied with 1-D bulk copies: their
  // byte counts and offsets must be multiples of 16
  if ((pk % 16 && hkv % 2) || (pv % 16 && hkv % 2)) return TQ_ERR_UNSUPPORTED;
  if ((pk * (hkv % 8)) % 16 || (pv * (hkv % 8)) % 16 || (pk * (hkv % 4)) % 16 || (pv * (hkv % 4)) % 16)
    return TQ_ERR_UNSUPPORTED;
  AttnArgs a{};
  for (int i = 0; i < TQ_MAX_D / 2; ++i) {
    a.k_sign_h2[i] = k->t.sign_h2[i];
    a.v_sign_h2[i] = v->t.sign_h2[i];
  }
  for (int i = 0; i < TQ_MAX_L; ++i) {
    a.k_levels[i] = k->t.levels[i];
    a.v_levels[i] = v->t.levels[i];
  }
  a.q = static_cast<const __half*>(q);
  a.k_packed = static_cast<const uint8_t*>(k_packed);
  a.k_norms = k_norms;
  a.v_packed = static_cast<const uint8_t*>(v_packed);
  a.v_norms = v_norms;
  a.positions = positions;
  a.block_tables = block_tables;
  a.max_blocks = max_blocks;
  a.num_blocks = num_blocks;
  a.out = static_cast<__half*>(out);
  a.B = B;
  a.hq = hq;
  a.hkv = hkv;
  a.g = g;
  a.s_max = s_max;
  a.nt = g > 4 ? 2 : 1;
  a.hw_max = ATT_WARPS / a.nt;
  attn_split(B, s_max, &a.n_split, &a.chunk);
  const size_t rows = (size_t)B * hq * a.n_split;
  if (ws_bytes < 2 * align16(rows * 4) + rows * (size_t)d * 4) return TQ_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.ws_m = reinterpret_cast<float*>(ws);
  a.ws_l = reinterpret_cast<float*>(ws + align16(rows * 4));
  a.ws_acc = reinterpret_cast<float*>(ws + 2 * align16(rows * 4));
  a.q_scale = (float)(1.4426950408889634 / ((double)d * std::sqrt((double)d)));
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.wait_limit = TQ_WAIT_LIMIT_CYCLES;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // 4-bit keys with 2-bit values: the fast kernel, when it takes the shapes
  cudaError_t e = tq_launch_attend_fast(a, d, k->bits, v->bits, tq_sm_count(dev), st);
  if (e != cudaErrorNotSupported) return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
  e = cudaErrorInvalidValue;
#define TQ_ATT_CASE(D_, KB_, VB_) \
  if (d == D_ && k->bits == KB_ && v->bits == VB_) e = launch_attend_t<D_, KB_, VB_>(a, st, dev);
#define TQ_ATT_D(D_)                                                                  \
  TQ_ATT_CASE(D_, 2, 2) TQ_ATT_CASE(D_, 2, 3) TQ_ATT_CASE(D_, 2, 4) TQ_ATT_CASE(D_, 3, 2) \
  TQ_ATT_CASE(D_, 3, 3) TQ_ATT_CASE(D_, 3, 4) TQ_ATT_CASE(D_, 4, 2) TQ_ATT_CASE(D_, 4, 3) \
  TQ_ATT_CASE(D_, 4, 4)
  TQ_ATT_D(64) TQ_ATT_D(128) TQ_ATT_D(256)
#undef TQ_ATT_D
#undef TQ_ATT_CASE
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_launch_attend(const tq_ctx* k, const tq_ctx* v, const void* q, int B, int hq, int hkv,
                           const void* k_packed, const float* k_norms, const void* v_packed,
                           const float* v_norms, int64_t s_max, const int32_t* positions, void* out,
                           void* workspace, size_t ws_bytes, void* stream) {
  return launch_attend(k, v, q, B, hq, hkv, k_packed, k_norms, v_packed, v_norms, s_max, positions, nullptr, 0, 0,
                       out, workspace, ws_bytes, stream);
}

tq_status tq_launch_attend_paged(const tq_ctx* k, const tq_ctx* v, const void* q, int B, int hq, int hkv,
                                 const void* k_cache, const float* k_norms, const void* v_cache,
                                 const float* v_norms, int64_t num_blocks, const int32_t* block_tables,
                                 int max_blocks, const int32_t* context_lens, void* out, void* workspace,
                                 size_t ws_bytes, void* stream) {
  return launch_attend(k, v, q, B, hq, hkv, k_cache, k_norms, v_cache, v_norms, (int64_t)max_blocks * ATT_BLOCK,
                       context_lens, block_tables, max_blocks, num_blocks, out, workspace, ws_bytes, stream);
}
