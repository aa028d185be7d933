// Encode on the fifth-generation tensor cores: fp16 vectors -> (packed
// Lloyd-Max codes, f32 norms), the same outputs as encode_kernel, for bulk
// launches.
//
// Method ("aither-kvcache" PyPI page, section "Algorithm", steps 1-5): per
// vector x of length d, N = ||x||_2; z = H D x / N with D the seeded sign
// flip and H the natural-order (Sylvester) Walsh-Hadamard matrix with +-1
// entries; index_i = #{j : z_i >= t_j}; indices packed little-endian.
//
// Factorisation used: H_d = H_{d/16} (x) H_16 (Sylvester's construction), so
// coordinate 16 b' + j of H D x is sum_b (-1)^popc(b' & b) S[b][j] with
// S[b] = H_16 D_b x_b the 16-point transform of block b. The tensor cores
// compute every S[b] of a 128-vector tile as one MMA each; the rest runs on
// the CUDA cores.
//
// B200 mapping (one persistent CTA per SM, warp-specialised):
//  * one thread of warp 0 streams 128-vector tiles into a ring of
//    shared-memory stages (4 at d = 128) with 2-D tensor copies (64-column
//    boxes, 128-byte swizzle, no multicast), refilling a stage as soon as its
//    MMAs are done and the norm warps have read it;
//  * one thread of warp 1 issues per tile d/16 tcgen05 MMAs of M = 128
//    vectors by N = K = 16 (A: the tile's columns of block b; B: H_16 with
//    block b's signs folded in, fp16 +-1, built in shared memory once). The
//    f32 results live in tensor memory: d columns per tile, 512/d tiles in
//    flight;
//  * two norm warps read each tile's fp16 rows from its shared-memory stage
//    (before the stage is refilled) and sum x^2 on the CUDA cores, one
//    mixed-precision FMA (fp16 inputs, f32 accumulator) per element in 8
//    or 16 chains; the square root goes to the epilogue through a small
//    per-accumulator buffer in shared memory;
//  * three epilogue warpgroups (two at d = 256) take turns on the tiles, one
//    vector per thread (TMEM lane = tile row); at d <= 128 setmaxnreg moves
//    registers from warpgroup 0 (copies, MMAs, norms: 56 each) to them (152
//    each), so more table lookups stay in flight: the remaining log2(d/16)
//    butterfly stages run in registers with packed f32x2 on 4 positions j at
//    a time (2 at d = 256), two such chunks per loop iteration; the
//    quantiser, guard band and fp64 recheck are those of encode_kernel; each
//    thread stores its packed row and norm.
//
// Exactness: the tensor core's arithmetic for kind::f16 with f32 accumulation
// was measured on B200 (every product exact; each addend's magnitude cut to a
// multiple of 2^(E-25), E the largest addend exponent; the sum rounded toward
// zero). For one 16-term block that bounds the error of S[b][j] by
// 7.5 u max_k |x_k| + 2 u |S[b][j]| (u = 2^-24); with the f32 stages, the
// norm (at most 9.5 u relative at d <= 128, 10 u at 256: squares of fp16
// values are exact in f32, chains of at most 16 terms and a tree of at most
// 4 levels) and the scaling, the error of q stays below the guard band of
// encode_kernel (7.4e-6 at d = 128 against 1e-5; 1.1e-5 at d = 256 against
// 2e-5), so unflagged decisions are the exact ones and flagged coordinates
// are recomputed in fp64 from the fp16 inputs.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "tq_common.cuh"
#include "tq_umma.cuh"

namespace tq {

constexpr int TC_ROWS = 128;   // vectors per tile (MMA M, TMEM lanes)
constexpr int TC_GROUPS = 3;   // epilogue warpgroups at most
// lane copies of the cell table, one per lane (measured against 16 copies:
// fewer shared-memory bank conflicts and 1.2-1.9 us less per launch over a
// layer's K and V; with 4 stages at d = 128 the larger table still fits)
constexpr int TC_LUT_COPIES = 32;
constexpr int TC_TMEM_COLS = 512;
constexpr float TC_MAGIC_2P23 = 8388608.0f;

template <int D, int BITS>
struct TcCfg {
  static constexpr int NB = D / 16;                  // 16-point blocks per vector
  static constexpr int BOXES = D / 64;               // 64-column copy boxes per tile
  static constexpr int BOX_BYTES = TC_ROWS * 128;    // 16 KB
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  static constexpr int STAGES = D == 256 ? 2 : (D == 128 ? 4 : 8);
  static constexpr int NACC = TC_TMEM_COLS / D;      // tiles in flight in tensor memory
  // epilogue warpgroups in use: at most one per accumulator, so that a group
  // waiting for use k of an accumulator's barrier always finds use k - 1
  // complete (a parity wait cannot tell use k from use k - 2)
  static constexpr int GROUPS = NACC < TC_GROUPS ? NACC : TC_GROUPS;
  // warpgroup 0: copies, MMAs and the two norm warps; then the epilogue warpgroups
  static constexpr int NW0 = 2;                      // first of the two norm warps
  static constexpr int EPI0 = 4;                     // first epilogue warp
  static constexpr int WARPS = EPI0 + 4 * GROUPS;
  // registers per thread after the split (launch: 128 per thread at 16 warps)
  static constexpr int REG_CTRL = 56, REG_EPI = 152;
  static constexpr bool SPLIT = WARPS == 16;  // (d = 256 runs 12 warps at their launch registers)
  // f32 chains of the sum of squares (at most 16 terms each)
  static constexpr int NCH = D == 256 ? 16 : 8;
  static constexpr int JC = D == 256 ? 2 : 4;        // positions j per epilogue chunk
  static constexpr int CHUNKS = 16 / JC;
  static constexpr int NV = NB * JC;                 // values per chunk (16 or 32)
  static constexpr int P = D * BITS / 8;             // packed bytes per vector
  static constexpr int WORDS = D * BITS / 32;
  static constexpr int L = 1 << BITS;
  // JC codes 2^(BITS-1) (the code of a zero or non-finite vector), BITS apart
  static constexpr uint32_t HALF_FIELD = (uint32_t)(L / 2) * (JC == 4 ? (1u | 1u << BITS | 1u << 2 * BITS | 1u << 3 * BITS)
                                                                      : (1u | 1u << BITS));
  // shared memory, from a 1024-aligned base: the stages first
  static constexpr int BREG = STAGES * TILE_BYTES;   // NB/4 regions of 16 rows x 128 B
  static constexpr int BAR = BREG + NB / 4 * 2048;   // full, empty, tfull, tempty, nfull, done
  static constexpr int NBARS = 2 * STAGES + 3 * NACC + 1;
  static constexpr int NRM = BAR + NBARS * 8;        // per accumulator: the tile's 128 norms
  static constexpr int SLOT = NRM + NACC * TC_ROWS * 4;  // TMEM base address
  static constexpr int SIGN = SLOT + 16;             // D sign bits (bit l of word t: coordinate 32 t + l)
  static constexpr int BND = SIGN + 32;              // the 2^BITS - 1 boundaries, z units
  static constexpr int SCR = (BND + 64 + 127) & ~127;  // per epilogue warp: 32 words
  static constexpr int LUT = SCR + 4 * TC_GROUPS * 128;
  static size_t bytes(int cells) { return 1024 + (size_t)LUT + (size_t)cells * TC_LUT_COPIES * 8; }
};

struct TcArgs {
  CUtensorMap tm_x;      // x as [n rows, d cols] fp16, box 64 x 128, 128-byte swizzle
  const __half* x;       // the same rows (fp64 recheck)
  int64_t n;             // vectors
  uint8_t* packed;
  float* norms;
  uint32_t* err;
  int fault_inject;      // test hook: 1 = never issue the tile copies
  long long wait_limit;  // bound on each mbarrier wait, SM cycles
};

// 32-byte store (sm_100): one instruction writes 8 words of a thread's row
TQ_DEV void tc_stg_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

TQ_DEV uint2 tc_lds_u2(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

TQ_DEV uint4 tc_lds_u4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}

// a0 += lo(w)^2, a1 += hi(w)^2 for the fp16 pair w: mixed-precision FMAs of
// sm_100 (fp16 operands, f32 addend and result). The square of an fp16 value
// is exact in f32, so each step rounds once.
TQ_DEV void tc_sq_acc2(float& a0, float& a1, uint32_t w) {
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "fma.rn.f32.f16 %0, lo, lo, %0;\n\tfma.rn.f32.f16 %1, hi, hi, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(w));
}

// sqrt(sum x^2) of row r of a tile staged in shared memory at `st` (boxes of
// 64 columns, 128-byte swizzle: 16-byte chunk c of row r at c ^ (r % 8)), in
// NCH f32 chains of at most 16 terms and a tree
template <int D, int NCH>
TQ_DEV float tc_row_norm(uint32_t st, int r) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  float ch[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) ch[c] = 0.f;
  // the row's 8 swizzled chunk addresses (the swizzle depends only on r % 8)
  uint32_t off[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) off[c] = st + r * 128 + (uint32_t)((c ^ (r & 7)) << 4);
#pragma unroll
  for (int c = 0; c < CPR; ++c) {
    const uint4 v = tc_lds_u4(off[c & 7] + (c >> 3) * (TC_ROWS * 128));
    float* cc = ch + ((c >> 3) & (NCH / 8 - 1)) * 8;
    tc_sq_acc2(cc[0], cc[1], v.x);
    tc_sq_acc2(cc[2], cc[3], v.y);
    tc_sq_acc2(cc[4], cc[5], v.z);
    tc_sq_acc2(cc[6], cc[7], v.w);
  }
#pragma unroll
  for (int w = NCH / 2; w > 0; w >>= 1)
#pragma unroll
    for (int c = 0; c < w; ++c) ch[c] += ch[c + w];
  return sqrtf(ch[0]);
}

TQ_DEV void tc_tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Exact codes of the values of one epilogue chunk of the source lane that lie
// inside the guard band. On entry scratch[0..NV-1] holds the chunk's rotated
// f32 values (value e is coordinate 16 (e / JC) + j0 + e % JC of the source
// vector, whose fp16 row is xrow); on return scratch[e] holds, as a uint32,
// the exact code of value e for every bit e of the returned mask. Called by
// the whole warp; rare, so kept out of line.
template <int D, int BITS>
__device__ __noinline__ uint32_t tc_recheck(float* scratch, float srcR, float qoff, float gq, uint32_t lut_lane,
                                            const __half* xrow, const uint32_t* sgn, int j0, const float* sbound) {
  using Cfg = TcCfg<D, BITS>;
  constexpr int NV = Cfg::NV, JC = Cfg::JC;
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  // the same f32 arithmetic as the main pass gives the same flags and cells
  uint2 ent = make_uint2(0u, 0u);
  bool band = false;
  if (lane < NV) {
    const float q = fmaf(scratch[lane], srcR, qoff);
    const uint32_t qb = __float_as_uint(__fadd_rd(q, TC_MAGIC_2P23));
    ent = tc_lds_u2(qb * (uint32_t)(TC_LUT_COPIES * 8) + lut_lane);
    band = fabsf(__uint_as_float(ent.x) - q) < gq;
  }
  const uint32_t cm = __ballot_sync(FULL, band);
  // N in fp64 from the fp16 inputs (products and sums exact)
  double xk[D / 32];
  double sq = 0.0;
#pragma unroll
  for (int t = 0; t < D / 32; ++t) {
    xk[t] = (double)__half2float(xrow[lane + 32 * t]);
    sq = fma(xk[t], xk[t], sq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(FULL, sq, o);
  const double n64 = sqrt(sq);
  uint32_t code = 0;
  for (uint32_t c2 = cm; c2; c2 &= c2 - 1) {
    const int e = __ffs(c2) - 1;
    const int i = 16 * (e / JC) + j0 + (e % JC);  // coordinate of value e
    // w_i = sum_k s_k (-1)^popcount(i & k) x_k, exact in fp64 (fp16 terms)
    double ps = 0.0;
#pragma unroll
    for (int t = 0; t < D / 32; ++t) {
      const int k = lane + 32 * t;
      const uint32_t neg = ((sgn[t] >> lane) & 1u) ^ (uint32_t)(__popc(i & k) & 1);
      ps += neg ? -xk[t] : xk[t];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(FULL, ps, o);
    // the cell of value e holds boundary number `below`; every other
    // boundary is decided with a margin of 1/64 cell
    const uint32_t below = __shfl_sync(FULL, ent.y, e);
    const uint32_t m = below + ((ps >= (double)sbound[below] * n64) ? 1u : 0u);
    if (lane == e) code = m;
  }
  __syncwarp();
  reinterpret_cast<uint32_t*>(scratch)[lane] = code;
  __syncwarp();
  return cm;
}

template <int JC>
TQ_DEV void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[JC]) {
  if constexpr (JC == 4)
    tmem_ld4(taddr, r);
  else
    tmem_ld2(taddr, r);
}

template <int D, int BITS>
__global__ void __launch_bounds__(TcCfg<D, BITS>::WARPS * 32, 1)
    encode_tc_kernel(const __grid_constant__ tq_codec_tables T, const __grid_constant__ TcArgs a) {
  using Cfg = TcCfg<D, BITS>;
  constexpr int NB = Cfg::NB, JC = Cfg::JC, S = Cfg::STAGES, NACC = Cfg::NACC, WORDS = Cfg::WORDS;
  constexpr int L = Cfg::L;
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the next kernel of the stream may start its own set-up as this grid's
  // CTAs exit (it waits for this grid before touching global memory)
  if (tid == 0) grid_dep_launch();

  const int64_t n_tiles = (a.n + TC_ROWS - 1) / TC_ROWS;
  const int cnt = (int64_t)blockIdx.x < n_tiles ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

  const uint32_t bar0 = base + Cfg::BAR;
  const uint32_t done_bar = bar0 + 8u * (2 * S + 3 * NACC);
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar0 + 8u * s, 1);             // full: tile landed
      mbar_init(bar0 + 8u * (S + s), 1 + 64);  // empty: its MMAs done, its rows read by the norm warps
    }
    for (int q = 0; q < NACC; ++q) {
      mbar_init(bar0 + 8u * (2 * S + q), 1);             // tfull: accumulator written
      mbar_init(bar0 + 8u * (2 * S + NACC + q), 4);      // tempty: its 4 warps read it (and its norms)
      mbar_init(bar0 + 8u * (2 * S + 2 * NACC + q), 64);  // nfull: the tile's norms written
    }
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + Cfg::SLOT, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + Cfg::SLOT);
  uint32_t* sgn = reinterpret_cast<uint32_t*>(sm + Cfg::SIGN);
  float* sbound = reinterpret_cast<float*>(sm + Cfg::BND);

  // ---- tables, built by warps 1 ... while warp 0 already streams the first
  // tiles in:
  //  * B operands: block b holds H_16[j][k] * s_{16 b + k} as fp16 +-1 in the
  //    K-major 128-byte-swizzled layout, four blocks side by side in one
  //    16-row region (block b: region b / 4, bytes 32 (b % 4) ... + 31 of row j);
  //  * the D sign bits (word t, bit l: coordinate 32 t + l), one ballot each;
  //  * the boundaries in z units (fp64 recheck);
  //  * the cell table: entry (cell, copy) = {boundary bits, count below}.
  if (warp >= 1) {
    const int t = tid - 32, nt = (int)blockDim.x - 32;
    for (int e = t; e < NB * 256; e += nt) {
      const int b = e >> 8, j = (e >> 4) & 15, k = e & 15, i = 16 * b + k;
      const uint32_t neg = ((T.sign_h2[i >> 1] >> (15 + 16 * (i & 1))) & 1u) ^ (uint32_t)(__popc(j & k) & 1);
      const int kb = 32 * (b & 3) + 2 * k;  // byte of the element within the row
      const uint32_t off = Cfg::BREG + (b >> 2) * 2048 + j * 128 + (((kb >> 4) ^ (j & 7)) << 4) + (kb & 15);
      *reinterpret_cast<uint16_t*>(sm + off) = neg ? (uint16_t)0xBC00u : (uint16_t)0x3C00u;
    }
    fence_proxy_async_smem();  // the B operands are read by the tensor cores
    for (int w = warp - 1; w < D / 32; w += Cfg::WARPS - 1) {
      const int i = 32 * w + lane;
      const uint32_t word = __ballot_sync(FULL, (T.sign_h2[i >> 1] >> (15 + 16 * (i & 1))) & 1u);
      if (lane == 0) sgn[w] = word;
    }
    if (t < L - 1) sbound[t] = T.bounds[t];
    uint2* lut = reinterpret_cast<uint2*>(sm + Cfg::LUT);
    const int entries = T.lut_cells * TC_LUT_COPIES;
    for (int e = t; e < entries; e += nt) {
      const int cell = e / TC_LUT_COPIES;
      lut[e] = make_uint2(T.cell[cell][0], T.cell[cell][1]);
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory");  // the tables are complete
  }

  if (warp < Cfg::EPI0) {
    // warpgroup 0: copies (warp 0), MMAs (warp 1), norms (warps 2, 3)
    if constexpr (Cfg::SPLIT) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Cfg::REG_CTRL));
    if (warp == 0) {
      // ---- producer: tile i of this CTA into stage i % S as soon as the MMAs
      // and the norm warps of tile i - S have released it
      if (lane == 0 && !a.fault_inject) {
        grid_dep_wait();  // the previous kernel of the stream may still write x
        for (int i = 0; i < cnt; ++i) {
          const int s = i % S;
          if (i >= S && !mbar_wait_bounded(bar0 + 8u * (S + s), ((i / S) - 1) & 1, a.wait_limit)) {
            record_error(a.err, TQ_DEVERR_TIMEOUT);
            break;
          }
          const int y = (int)(((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * TC_ROWS);
          mbar_arrive_expect_tx(bar0 + 8u * s, Cfg::TILE_BYTES);
  #pragma unroll
          for (int bx = 0; bx < Cfg::BOXES; ++bx)
            tc_tma_load_2d(base + s * Cfg::TILE_BYTES + bx * Cfg::BOX_BYTES, &a.tm_x, 64 * bx, y, bar0 + 8u * s);
        }
      }
    } else if (warp == 1) {
      // ---- MMA issuer: S[b] = A_b * B_b^T for the d/16 blocks of tile i
      if (lane == 0) {
        grid_dep_wait();  // (its only global access is the error word)
        constexpr uint32_t IDESC = umma_idesc_f16(TC_ROWS, 16);
        for (int i = 0; i < cnt; ++i) {
          const int s = i % S, q = i % NACC;
          if (!mbar_wait_bounded(bar0 + 8u * s, (i / S) & 1, a.wait_limit) ||
              (i >= NACC && !mbar_wait_bounded(bar0 + 8u * (2 * S + NACC + q), ((i / NACC) - 1) & 1, a.wait_limit))) {
            record_error(a.err, TQ_DEVERR_TIMEOUT);
            break;
          }
          tc_fence_after();
          const uint32_t st = base + s * Cfg::TILE_BYTES;
  #pragma unroll
          for (int b = 0; b < NB; ++b) {
            const uint64_t ad = umma_desc_sw128(st + (b >> 2) * Cfg::BOX_BYTES + (b & 3) * 32);
            const uint64_t bd = umma_desc_sw128(base + Cfg::BREG + (b >> 2) * 2048 + (b & 3) * 32);
            umma_f16(tmem + (uint32_t)(q * D + 16 * b), ad, bd, IDESC, false);
          }
          umma_commit(bar0 + 8u * (S + s));      // the stage may be refilled
          umma_commit(bar0 + 8u * (2 * S + q));  // the accumulator may be read
        }
        // every MMA issued has completed before tensor memory is freed
        umma_commit(done_bar);
        if (!mbar_wait_bounded(done_bar, 0, a.wait_limit)) record_error(a.err, TQ_DEVERR_TIMEOUT);
      }
    } else {
      // ---- norm warps: rows 64 k + lane and 64 k + 32 + lane of every tile,
      // read from the tile's stage as soon as it lands; N = sqrt(sum x^2) in
      // NCH f32 chains (at most 16 terms each, then a tree), written to the
      // accumulator's norm buffer once the epilogue has taken the previous
      // tile's norms from it
      const int k = warp - Cfg::NW0;
      float* nbuf = reinterpret_cast<float*>(sm + Cfg::NRM);
      for (int i = 0; i < cnt; ++i) {
        const int s = i % S, q = i % NACC;
        bool ok = mbar_wait_bounded(bar0 + 8u * s, (i / S) & 1, a.wait_limit);
        if (ok && i >= NACC) ok = mbar_wait_bounded(bar0 + 8u * (2 * S + NACC + q), ((i / NACC) - 1) & 1, a.wait_limit);
        if (!__all_sync(FULL, ok)) {
          if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
          break;
        }
        const uint32_t st = base + s * Cfg::TILE_BYTES;
  #pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int r = 64 * k + 32 * rr + lane;
          nbuf[q * TC_ROWS + r] = tc_row_norm<D, Cfg::NCH>(st, r);
        }
        // every thread arrives: its reads of the stage are done and its norms written
        mbar_arrive(bar0 + 8u * (S + s));
        mbar_arrive(bar0 + 8u * (2 * S + 2 * NACC + q));
      }
    }
  } else {
    // the epilogue warpgroups; registers from warpgroup 0 move here:
    // 3 x 128 x 152 + 128 x 56 = 512 x 128, the launch's total
    if constexpr (Cfg::SPLIT) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Cfg::REG_EPI));
    // ---- epilogue warpgroup g (warps 4g + 2 ... 4g + 5, which cover the four
    // lane quarters of tensor memory): tiles g, g + GROUPS, ...; one vector per thread
    const int g = (warp - Cfg::EPI0) >> 2, quarter = warp & 3;
    float* scratch = reinterpret_cast<float*>(sm + Cfg::SCR + (warp - Cfg::EPI0) * 128);
    // the bits of 2^23 + cell times 256 are cell * 256 (mod 2^32)
    static_assert(TC_LUT_COPIES * 8 == 256, "cell stride of the table addressing");
    const uint32_t lut_lane = base + Cfg::LUT + (uint32_t)(lane & (TC_LUT_COPIES - 1)) * 8u;
    const float Rscale = T.inv_delta, qoff = T.q_offset, gq = T.guard_q;
    const f2 Q2 = make_float2(qoff, qoff), M2 = make_float2(TC_MAGIC_2P23, TC_MAGIC_2P23);
    grid_dep_wait();  // before the first store and the first recheck load
    const float* nbuf = reinterpret_cast<const float*>(sm + Cfg::NRM);
    for (int i = g; i < cnt; i += Cfg::GROUPS) {
      const int q = i % NACC;
      // warp-uniform decision: the tensor-memory loads below are warp-collective
      const bool ok = mbar_wait_bounded(bar0 + 8u * (2 * S + q), (i / NACC) & 1, a.wait_limit) &&
                      mbar_wait_bounded(bar0 + 8u * (2 * S + 2 * NACC + q), (i / NACC) & 1, a.wait_limit);
      if (!__all_sync(FULL, ok)) {
        if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int64_t tile = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
      const int64_t row = tile * TC_ROWS + 32 * quarter + lane;
      const bool active = row < a.n;
      const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(q * D);

      // ---- norm of this thread's vector, from the norm warps
      const float nrm = nbuf[q * TC_ROWS + 32 * quarter + lane];
      const bool special = !(nrm > 0.f) || !(nrm <= 3.0e38f);  // zero or non-finite vector
      const float R = special ? 0.f : __fdiv_rn(Rscale, nrm);
      const f2 R2 = make_float2(R, R);

      // Codes of output block b' (coordinates 16 b' + j) collect in a
      // 16*BITS-bit shift register (clo: bits 0-31, chi: the rest). A loop
      // iteration handles two chunks of JC positions (compile-time code
      // positions within a 2*JC*BITS-bit field per block), then shifts the
      // field in on top, so after the last iteration every code sits at its
      // stream position.
      uint32_t clo[NB], chi[NB];
#pragma unroll
      for (int bp = 0; bp < NB; ++bp) clo[bp] = chi[bp] = 0u;

#pragma unroll 1
      for (int c2 = 0; c2 < Cfg::CHUNKS; c2 += 2) {
        uint32_t fld[NB];  // 2 JC codes of block b', code jj at bits BITS * jj
#pragma unroll
        for (int bp = 0; bp < NB; ++bp) fld[bp] = 0u;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int j0 = (c2 + u) * JC;
          uint32_t r[NB][JC];
#pragma unroll
          for (int b = 0; b < NB; ++b) tmem_ld_chunk<JC>(tl + (uint32_t)(16 * b + j0), r[b]);
          tmem_wait_ld();
#pragma unroll
          for (int b = 0; b < NB; ++b) tmem_regs_after_wait(r[b]);
          if (u == 1 && c2 + 2 >= Cfg::CHUNKS) {  // every load of this accumulator is done: free it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar0 + 8u * (2 * S + NACC + q));
          }
          // v[h][b'] = positions (j0 + 2h, j0 + 2h + 1) of output block b'
          f2 v[JC / 2][NB];
#pragma unroll
          for (int h = 0; h < JC / 2; ++h) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
              v[h][b] = make_float2(__uint_as_float(r[b][2 * h]), __uint_as_float(r[b][2 * h + 1]));
            wht_pairs<NB>(v[h]);
          }
          float gmin = 3.0e38f;  // closest approach to a boundary in this chunk (q units)
          if (!special) {
#pragma unroll
            for (int h = 0; h < JC / 2; ++h) {
#pragma unroll
              for (int bp = 0; bp < NB; ++bp) {
                const f2 q2 = fma2(v[h][bp], R2, Q2);
                const f2 qm = add2_rm(q2, M2);  // bits: 2^23 + floor(q)
                float dl[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const float qq = e ? q2.y : q2.x;
                  const uint32_t qb = __float_as_uint(e ? qm.y : qm.x);
                  const uint2 ent = tc_lds_u2(qb * (uint32_t)(TC_LUT_COPIES * 8) + lut_lane);
                  dl[e] = __uint_as_float(ent.x) - qq;
                  fld[bp] += (ent.y + (__float_as_uint(dl[e]) >> 31)) << (BITS * (u * JC + 2 * h + e));
                }
                gmin = fminf(gmin, fminf(fabsf(dl[0]), fabsf(dl[1])));
              }
            }
          } else {
#pragma unroll
            for (int bp = 0; bp < NB; ++bp) fld[bp] += Cfg::HALF_FIELD << (BITS * u * JC);
          }
          // ---- exact recheck of the values of this chunk inside the guard band (rare)
          uint32_t any = __ballot_sync(FULL, active && gmin < gq);
          while (any) {
            const int src = __ffs(any) - 1;
            any &= any - 1;
            const float srcR = __shfl_sync(FULL, R, src);
            if (lane == src) {
#pragma unroll
              for (int h = 0; h < JC / 2; ++h)
#pragma unroll
                for (int bp = 0; bp < NB; ++bp) {
                  scratch[bp * JC + 2 * h] = v[h][bp].x;
                  scratch[bp * JC + 2 * h + 1] = v[h][bp].y;
                }
            }
            __syncwarp();
            const int64_t srow = tile * TC_ROWS + 32 * quarter + src;
            const uint32_t cm =
                tc_recheck<D, BITS>(scratch, srcR, qoff, gq, lut_lane, a.x + srow * D, sgn, j0, sbound);
            if (lane == src) {
              for (uint32_t cc = cm; cc; cc &= cc - 1) {
                const int e = __ffs(cc) - 1;
                const uint32_t sh = (uint32_t)(BITS * (u * JC + e % JC)),
                               m = reinterpret_cast<const uint32_t*>(scratch)[e];
                const int eb = e / JC;
#pragma unroll
                for (int bp = 0; bp < NB; ++bp) {
                  const uint32_t mk = bp == eb ? ((1u << BITS) - 1u) << sh : 0u;
                  fld[bp] = (fld[bp] & ~mk) | ((m << sh) & mk);
                }
              }
            }
            __syncwarp();
          }
        }
        // ---- shift the 2 JC codes in on top of each block's register
#pragma unroll
        for (int bp = 0; bp < NB; ++bp) {
          constexpr int FW = 2 * JC * BITS, CW = 16 * BITS;
          if constexpr (CW == 32) {
            clo[bp] = FW == 32 ? fld[bp] : __funnelshift_r(clo[bp], fld[bp], FW);
          } else if constexpr (FW == 32) {  // 4 bits, 4 positions: whole words
            clo[bp] = chi[bp];
            chi[bp] = fld[bp];
          } else if constexpr (CW - FW >= 32) {  // the new field lies within chi
            clo[bp] = __funnelshift_r(clo[bp], chi[bp], FW);
            chi[bp] = (chi[bp] >> FW) | (fld[bp] << (CW - FW - 32));
          } else {  // the new field straddles clo and chi; the old bits end in clo
            clo[bp] = __funnelshift_r(clo[bp], chi[bp], FW) | (fld[bp] << (CW - FW));
            chi[bp] = fld[bp] >> (32 - (CW - FW));
          }
        }
      }

      // ---- the packed row: block b' holds stream bits [16 BITS b', 16 BITS (b' + 1))
      uint32_t words[WORDS];
#pragma unroll
      for (int bp = 0; bp < NB; ++bp) {
        if constexpr (BITS == 2) {
          words[bp] = clo[bp];
        } else if constexpr (BITS == 4) {
          words[2 * bp] = clo[bp];
          words[2 * bp + 1] = chi[bp];
        } else {  // 48 bits per block: pairs of blocks fill three words
          const int k = 3 * (bp >> 1);
          if ((bp & 1) == 0) {
            words[k] = clo[bp];
            words[k + 1] = chi[bp];
          } else {
            words[k + 1] |= clo[bp] << 16;
            words[k + 2] = (clo[bp] >> 16) | (chi[bp] << 16);
          }
        }
      }

      // ---- this thread's packed row and norm
      if (active) {
        uint8_t* dst = a.packed + row * Cfg::P;
        // rows of a multiple of 32 bytes from a 32-byte aligned base: 32-byte
        // stores (a warp's store then touches half as many cache lines)
        bool stored = false;
        if constexpr (Cfg::P % 32 == 0) {
          if ((reinterpret_cast<uintptr_t>(a.packed) & 31u) == 0) {
#pragma unroll
            for (int w = 0; w < WORDS; w += 8) tc_stg_v8(dst + 4 * w, words + w);
            stored = true;
          }
        }
        if (!stored) {
          if constexpr (Cfg::P % 16 == 0) {
#pragma unroll
            for (int w = 0; w < WORDS; w += 4)
              *reinterpret_cast<uint4*>(dst + 4 * w) = make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
          } else {
#pragma unroll
            for (int w = 0; w < WORDS; w += 2)
              *reinterpret_cast<uint2*>(dst + 4 * w) = make_uint2(words[w], words[w + 1]);
          }
        }
        a.norms[row] = nrm;
      }
    }
  }
  // ---- teardown: every role is done (or gave up); free the tensor memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
}

template <int D, int BITS>
static cudaError_t launch_encode_tc_t(const tq_codec_tables& T, TcArgs a, const void* x, cudaStream_t st) {
  using Cfg = TcCfg<D, BITS>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const size_t smem = Cfg::bytes(T.lut_cells);
  static std::atomic<uint64_t> configured{0};  // one bit per device
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(encode_tc_kernel<D, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Cfg::bytes(TQ_MAX_CELLS));
    if (e != cudaSuccess) return e;
    if constexpr (Cfg::SPLIT) {
      // the epilogue's setmaxnreg.inc waits until warpgroup 0 has released
      // enough registers: it can only complete if the launch holds the whole
      // split (3 x 128 x REG_EPI + 128 x REG_CTRL registers), so check the
      // registers the kernel is launched with before the first launch
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, encode_tc_kernel<D, BITS>);
      if (e != cudaSuccess) return e;
      if ((int64_t)fa.numRegs * Cfg::WARPS * 32 < (int64_t)128 * (3 * Cfg::REG_EPI + Cfg::REG_CTRL))
        return cudaErrorNotSupported;
    }
    configured.fetch_or(bit);
  }
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tq_tensor_map_encode_fn());
  if (!enc) return cudaErrorNotSupported;
  const int sms = tq_sm_count(dev);
  // launches of at most 2^30 rows keep the copy coordinates in int32
  const int64_t max_rows = (int64_t)1 << 30;
  const int64_t n_total = a.n;
  uint8_t* packed0 = a.packed;
  float* norms0 = a.norms;
  for (int64_t off = 0; off < n_total; off += max_rows) {
    const int64_t n = std::min(max_rows, n_total - off);
    const __half* xs = static_cast<const __half*>(x) + off * D;
    a.n = n;
    a.x = xs;
    a.packed = packed0 + off * Cfg::P;
    a.norms = norms0 + off;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)n};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)TC_ROWS};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&a.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(static_cast<const void*>(xs)), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
    const int64_t tiles = (n + TC_ROWS - 1) / TC_ROWS;
    const int grid = (int)std::min<int64_t>(tiles, (int64_t)sms);
    e = tq_launch_pdl(encode_tc_kernel<D, BITS>, dim3(grid), dim3(Cfg::WARPS * 32), smem, st, T, a);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq

using namespace tq;

int64_t tq_encode_tc_min_rows(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  return (int64_t)TC_ROWS * tq_sm_count(dev);
}

tq_status tq_launch_encode_tc(const tq_ctx* ctx, const void* x, int64_t n, void* packed, float* norms, void* stream,
                              int fault_inject) {
  if (n == 0) return TQ_OK;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.n = n;
  a.packed = static_cast<uint8_t*>(packed);
  a.norms = norms;
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.fault_inject = fault_inject;
  a.wait_limit = fault_inject ? 20000000LL : TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
  const tq_codec_tables& T = ctx->t;
#define TQ_ENCTC_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_encode_tc_t<D_, B_>(T, a, x, st);
  TQ_ENCTC_CASE(64, 2) TQ_ENCTC_CASE(64, 3) TQ_ENCTC_CASE(64, 4)
  TQ_ENCTC_CASE(128, 2) TQ_ENCTC_CASE(128, 3) TQ_ENCTC_CASE(128, 4)
  TQ_ENCTC_CASE(256, 2) TQ_ENCTC_CASE(256, 3) TQ_ENCTC_CASE(256, 4)
#undef TQ_ENCTC_CASE
  // cudaErrorNotSupported: a launch this kernel cannot make (the caller
  // takes the CUDA-core kernel)
  return e == cudaSuccess ? TQ_OK : e == cudaErrorNotSupported ? TQ_ERR_UNSUPPORTED : TQ_ERR_CUDA;
}
