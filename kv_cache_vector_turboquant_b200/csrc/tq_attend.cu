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
// Split-S: the grid is (n_split, B, kv-head groups of 8). Each CTA owns a
// chunk of cache positions of one sequence and up to 8 kv heads (one warp
// each). Position rows (all heads of one position, contiguous in the
// [B, S, Hkv, P] layout) are brought into padded shared rows by 1-D bulk
// copies (TMA, no multicast) through a 3-stage mbarrier pipeline; tiles are 32
// positions. Per tile and kv head: scores with lane = position, online softmax
// in the exp2 domain, value accumulation with lane = coordinate block. The
// partial (max, sum, accumulator) of every split goes to the workspace; a
// second kernel merges the splits (log-sum-exp) and applies D_V H / d.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "tq_common.cuh"

namespace tq {

constexpr int ATT_WARPS = 8;   // kv heads per CTA (one warp each)
constexpr int ATT_STAGES = 3;  // position tiles in flight
constexpr int ATT_TILE = 32;   // positions per tile
constexpr int ATT_MAXG = 8;    // query heads per kv head supported
constexpr int ATT_TARGET_CTAS = 296;

struct AttnArgs {
  uint32_t k_sign_h2[TQ_MAX_D / 2];
  uint32_t v_sign_h2[TQ_MAX_D / 2];
  float k_levels[TQ_MAX_L];
  float v_levels[TQ_MAX_L];
  const __half* q;
  const uint8_t* k_packed;
  const float* k_norms;
  const uint8_t* v_packed;
  const float* v_norms;
  const int32_t* positions;
  __half* out;
  float* ws_m;    // [B, Hq, n_split]  running max (log2 domain)
  float* ws_l;    // [B, Hq, n_split]  sum of weights
  float* ws_acc;  // [B, Hq, n_split, D] rotated accumulator
  uint32_t* err;
  long long wait_limit;
  int B, hq, hkv, g;
  int64_t s_max;
  int n_split;
  int chunk;  // positions per split (multiple of ATT_TILE)
  float q_scale;  // log2(e) / (d sqrt(d))
};

// Split count and chunk for a batch: about ATT_TARGET_CTAS CTAs per kv-head
// group, chunks a multiple of the tile. Depends only on (B, s_max), so the
// workspace size does too.
inline void attn_split(int B, int64_t s_max, int* n_split, int* chunk) {
  const int64_t tiles = (s_max + ATT_TILE - 1) / ATT_TILE;
  int64_t ns = (ATT_TARGET_CTAS + (int64_t)B - 1) / (int64_t)B;
  ns = std::max<int64_t>(1, std::min<int64_t>(ns, tiles));
  const int64_t tiles_per = (tiles + ns - 1) / ns;
  *chunk = (int)(tiles_per * ATT_TILE);
  *n_split = (int)((tiles + tiles_per - 1) / tiles_per);
}

template <int D, int KB, int VB>
struct AttCfg {
  static constexpr int PK = D * KB / 8;
  static constexpr int PV = D * VB / 8;
  static constexpr int LK = 1 << KB;
  static constexpr int LV = 1 << VB;
  static constexpr int CPL = D / 32;  // coordinates per lane in the value phase
};


// Shared-memory layout of the partial kernel (bytes); identical on host and device.
struct AttSmem {
  int bar, qt, kst, vst, pw, lutk, lutv, total;
  int krow, vrow, stage;
  __host__ __device__ AttSmem(int D, int PK, int PV, int LK, int LV, int g) {
    krow = ATT_WARPS * PK + 16;  // padded position row of K (all heads of the group)
    vrow = ATT_WARPS * PV + 16;
    stage = ATT_TILE * (krow + vrow);
    bar = 0;
    qt = 128;
    kst = qt + ATT_WARPS * g * D * 4;
    vst = kst + ATT_TILE * krow;  // stage s: kst + s*stage (K rows), then V rows
    pw = kst + ATT_STAGES * stage;
    lutk = pw + ATT_WARPS * ATT_TILE * ATT_MAXG * 4;
    lutv = lutk + LK * 32 * 4;
    total = lutv + LV * 32 * 4;
  }
};

TQ_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
TQ_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Extract `NB` bits at bit offset `off` of a little-endian word stream.
template <int NB>
TQ_DEV uint32_t bits_at(const uint32_t* w, int off) {
  uint32_t f = w[off >> 5] >> (off & 31);
  if ((off & 31) + NB > 32) f |= w[(off >> 5) + 1] << (32 - (off & 31));
  return f & ((1u << NB) - 1u);
}

template <int D, int KB, int VB>
__global__ void __launch_bounds__(ATT_WARPS * 32, 2) attend_partial_kernel(const __grid_constant__ AttnArgs a) {
  using Cfg = AttCfg<D, KB, VB>;
  constexpr int PK = Cfg::PK, PV = Cfg::PV, CPL = Cfg::CPL;
  extern __shared__ __align__(128) uint8_t smem[];
  const AttSmem L(D, PK, PV, Cfg::LK, Cfg::LV, a.g);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const int hk0 = blockIdx.z * ATT_WARPS;
  const int hw = min(ATT_WARPS, a.hkv - hk0);  // kv heads in this CTA
  const int g = a.g;

  int64_t pos = a.positions[b];
  if (pos > a.s_max) {
    if (threadIdx.x == 0 && split == 0) record_error(a.err, TQ_DEVERR_POS_RANGE);
    pos = a.s_max;
  }
  const int64_t s0 = (int64_t)split * a.chunk;
  const int64_t s1 = min64(s0 + a.chunk, pos);
  const int64_t npos = s1 > s0 ? s1 - s0 : 0;
  const int ntiles = (int)((npos + ATT_TILE - 1) / ATT_TILE);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  float* qt = reinterpret_cast<float*>(smem + L.qt);
  float* pw = reinterpret_cast<float*>(smem + L.pw) + warp * ATT_TILE * ATT_MAXG;
  {
    float* lk = reinterpret_cast<float*>(smem + L.lutk);
    for (int e = threadIdx.x; e < Cfg::LK * 32; e += blockDim.x) lk[e] = a.k_levels[e >> 5];
    float* lv = reinterpret_cast<float*>(smem + L.lutv);
    for (int e = threadIdx.x; e < Cfg::LV * 32; e += blockDim.x) lv[e] = a.v_levels[e >> 5];
  }
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < ATT_STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();

  // producer: warp 0 issues one K row copy and one V row copy per position
  const uint32_t krow_bytes = (uint32_t)(hw * PK), vrow_bytes = (uint32_t)(hw * PV);
  auto issue = [&](int tile, int stage) {
    const int64_t t0 = s0 + (int64_t)tile * ATT_TILE;
    const int nv = (int)min64(ATT_TILE, s1 - t0);
    const uint32_t bar = smem_u32(&bars[stage]);
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)nv * (krow_bytes + vrow_bytes));
    __syncwarp();
    if (lane < nv) {
      const int64_t row = ((int64_t)b * a.s_max + t0 + lane) * a.hkv + hk0;
      uint8_t* st = smem + L.kst + stage * L.stage;
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
  for (int e = threadIdx.x; e < nq * D; e += blockDim.x) qt[e] *= a.q_scale;
  __syncthreads();

  const bool head_ok = warp < hw;
  const int hk = hk0 + warp;
  const float* qw = qt + warp * g * D;  // this warp's g query heads
  const uint32_t lutk_lane = smem_u32(smem + L.lutk) + lane * 4u;
  const uint32_t lutv_lane = smem_u32(smem + L.lutv) + lane * 4u;
  float m[ATT_MAXG], l[ATT_MAXG], acc[ATT_MAXG][CPL];
#pragma unroll
  for (int j = 0; j < ATT_MAXG; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[j][c] = 0.f;
  }

  uint32_t parity = 0;
  for (int tile = 0; tile < ntiles; ++tile) {
    const int stage = tile % ATT_STAGES;
    const int64_t t0 = s0 + (int64_t)tile * ATT_TILE;
    const int nv = (int)min64(ATT_TILE, s1 - t0);
    // all threads poll the barrier; the CTA acts on one agreed outcome
    const bool ok = __syncthreads_and(mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u,
                                                        a.wait_limit) ? 1 : 0) != 0;
    if (!ok) {
      if (threadIdx.x == 0) {
        record_error(a.err, TQ_DEVERR_TIMEOUT);
        // drain the other stages already issued, bounded, then leave
        for (int s = 1; s < ATT_STAGES; ++s) {
          const int os = (stage + s) % ATT_STAGES;
          if (tile + s < ntiles) (void)mbar_wait_bounded(smem_u32(&bars[os]), (parity >> os) & 1u, a.wait_limit);
        }
      }
      return;
    }
    parity ^= 1u << stage;
    const uint8_t* kst = smem + L.kst + stage * L.stage;
    const uint8_t* vst = kst + ATT_TILE * L.krow;

    if (head_ok) {
      // ---- scores, lane = position
      const bool valid = lane < nv;
      float sc[ATT_MAXG];
#pragma unroll
      for (int j = 0; j < ATT_MAXG; ++j) sc[j] = 0.f;
      float nk = 0.f, nvn = 0.f;
      if (valid) {
        const int64_t row = ((int64_t)b * a.s_max + t0 + lane) * a.hkv + hk;
        nk = __ldg(a.k_norms + row);
        nvn = __ldg(a.v_norms + row);
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(kst + lane * L.krow + warp * PK);
        uint32_t words[PK / 4];
#pragma unroll
        for (int w = 0; w < PK / 4; ++w) words[w] = kw[w];
        constexpr int CH = 32;  // coordinates per chunk held in registers
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += CH) {
          float lv[CH];
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const uint32_t code = bits_at<KB>(words, (c0 + i) * KB);
            float val;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(val) : "r"(code * 128u + lutk_lane));
            lv[i] = val;
          }
#pragma unroll
          for (int j = 0; j < ATT_MAXG; ++j) {
            if (j < g) {
              const float4* qv = reinterpret_cast<const float4*>(qw + j * D + c0);
              float s = 0.f;
#pragma unroll
              for (int i4 = 0; i4 < CH / 4; ++i4) {
                const float4 qq = qv[i4];
                s = fmaf(qq.x, lv[4 * i4], s);
                s = fmaf(qq.y, lv[4 * i4 + 1], s);
                s = fmaf(qq.z, lv[4 * i4 + 2], s);
                s = fmaf(qq.w, lv[4 * i4 + 3], s);
              }
              sc[j] += s;
            }
          }
        }
      }
      // ---- online softmax (log2 domain), per query head of the group
      float alpha[ATT_MAXG];
#pragma unroll
      for (int j = 0; j < ATT_MAXG; ++j) {
        alpha[j] = 1.f;
        if (j < g) {
          const float s = valid ? sc[j] * nk : -INFINITY;
          const float mx = warp_max(s);
          const float mn = fmaxf(m[j], mx);
          float p = 0.f;
          if (mn != -INFINITY) {
            alpha[j] = exp2f(m[j] - mn);
            p = valid ? exp2f(s - mn) : 0.f;
          }
          l[j] = l[j] * alpha[j] + warp_sum(p);
          m[j] = mn;
          pw[lane * ATT_MAXG + j] = p * nvn;
        }
      }
      __syncwarp();
      // ---- values, lane = block of CPL coordinates
#pragma unroll
      for (int j = 0; j < ATT_MAXG; ++j)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[j][c] *= alpha[j];
      for (int t = 0; t < nv; ++t) {
        const uint32_t* vw = reinterpret_cast<const uint32_t*>(vst + t * L.vrow + warp * PV);
        const int off = lane * CPL * VB;
        uint32_t two[2];
        two[0] = vw[off >> 5];
        two[1] = ((off & 31) + CPL * VB > 32) ? vw[(off >> 5) + 1] : 0u;
        float lvv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const uint32_t code = bits_at<VB>(two, (off & 31) + c * VB);
          float val;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(val) : "r"(code * 128u + lutv_lane));
          lvv[c] = val;
        }
        const float* pt = pw + t * ATT_MAXG;
#pragma unroll
        for (int j = 0; j < ATT_MAXG; ++j) {
          if (j < g) {
            const float pj = pt[j];
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[j][c] = fmaf(pj, lvv[c], acc[j][c]);
          }
        }
      }
    }
    __syncthreads();  // every warp is done with this stage
    if (warp == 0 && tile + ATT_STAGES < ntiles) issue(tile + ATT_STAGES, stage);
  }

  // ---- partial results of this split
  if (head_ok) {
#pragma unroll
    for (int j = 0; j < ATT_MAXG; ++j) {
      if (j < g) {
        const int h = hk * g + j;
        const int64_t idx = ((int64_t)b * a.hq + h) * a.n_split + split;
        if (lane == 0) {
          a.ws_m[idx] = m[j];
          a.ws_l[idx] = l[j];
        }
        float* dst = a.ws_acc + idx * D + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; ++c) dst[c] = acc[j][c];
      }
    }
  }
}


// Merge the splits of one (sequence, query head) and rotate back:
// M = max_s m_s, w_s = 2^(m_s - M), o~ = sum_s w_s acc_s / sum_s w_s l_s,
// o = D_V H_pm o~ / d, rounded to fp16. One CTA of d threads per row.
template <int D>
__global__ void __launch_bounds__(D) attend_combine_kernel(const __grid_constant__ AttnArgs a) {
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

inline size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

template <int D, int KB, int VB>
static cudaError_t launch_attend_t(const AttnArgs& a, cudaStream_t st, int dev) {
  using Cfg = AttCfg<D, KB, VB>;
  const AttSmem L(D, Cfg::PK, Cfg::PV, Cfg::LK, Cfg::LV, a.g);
  cudaError_t e = cudaFuncSetAttribute(attend_partial_kernel<D, KB, VB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.n_split, a.B, (a.hkv + ATT_WARPS - 1) / ATT_WARPS);
  attend_partial_kernel<D, KB, VB><<<grid, ATT_WARPS * 32, L.total, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attend_combine_kernel<D><<<dim3(a.hq, a.B), D, 0, st>>>(a);
  (void)dev;
  return cudaGetLastError();
}

}  // namespace tq

using namespace tq;

size_t tq_attend_workspace_bytes_impl(int B, int hq, int head_dim, int64_t s_max) {
  int ns = 0, chunk = 0;
  attn_split(B, s_max, &ns, &chunk);
  const size_t rows = (size_t)B * hq * ns;
  return 2 * align16(rows * 4) + rows * (size_t)head_dim * 4;
}

tq_status tq_launch_attend(const tq_ctx* k, const tq_ctx* v, const void* q, int B, int hq, int hkv,
                           const void* k_packed, const float* k_norms, const void* v_packed,
                           const float* v_norms, int64_t s_max, const int32_t* positions, void* out,
                           void* workspace, size_t ws_bytes, void* stream) {
  const int d = k->d;
  const int g = hq / hkv;
  if (g > ATT_MAXG) return TQ_ERR_UNSUPPORTED;
  const int pk = d * k->bits / 8, pv = d * v->bits / 8;
  // position rows of a kv-head group are copied with 1-D bulk copies: their
  // byte counts and offsets must be multiples of 16
  if ((pk % 16 && hkv % 2) || (pv % 16 && hkv % 2)) return TQ_ERR_UNSUPPORTED;
  AttnArgs a;
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
  a.out = static_cast<__half*>(out);
  a.B = B;
  a.hq = hq;
  a.hkv = hkv;
  a.g = g;
  a.s_max = s_max;
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
  cudaError_t e = cudaErrorInvalidValue;
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
