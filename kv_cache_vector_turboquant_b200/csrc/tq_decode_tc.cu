// Decode on the fifth-generation tensor cores: (packed codes, f32 norms) ->
// fp16 vectors, the same outputs as decode_kernel, for bulk launches at
// head_dim 64 and 128.
//
// Method ("aither-kvcache" PyPI page, section "Algorithm": decoding reverses
// steps 4-1): x_hat = D (H_pm c[idx]) * (N / d), H_pm the +-1 natural-order
// Walsh-Hadamard matrix, D the seeded sign flip, c the codebook levels.
//
// Transform: H_d = H_{d/32} (x) H_32 (Sylvester), so coordinate 32 b' + j of
// H_pm c is sum_b (-1)^popc(b' & b) S[b][j] with S[b] = H_32 c_b the 32-point
// transform of block b. The tensor cores compute every S[b] of a 128-vector
// tile (M = 128, N = 32, two K-steps of 16 per block); the remaining
// log2(d/32) stages run as f32 butterflies in the epilogue. The levels lie on
// the 2^-14 grid (16 significant bits), so each level is split into an fp16
// value and an fp16 remainder (both exact) and both parts are multiplied
// (four MMAs per block into its accumulator columns). Every product and every
// partial sum is a multiple of 2^-14 below 2^9 (|H_pm c| <= d max|c| < 2^9),
// so it is exact in f32: the tensor core cuts addends only below 2^(E-25)
// with E <= 7 and rounds an exact sum to itself, and the f32 butterflies add
// exact values whose sums are exact. The only roundings are the product by
// N / d and the fp16 conversion, as in decode_kernel (outputs bit-identical).
//
// Why 32-point blocks and not the whole transform on the tensor cores: the
// whole transform (N = d) is 8 times the tensor-core work of these blocks
// (256 multiply-adds per coordinate at d = 128, about 1 PFLOP/s of fp16 at
// the streaming rate) and ran the GPU into its power limit on its own (about
// 1500 MHz); 32-point blocks cost one f32x2 add per coordinate more and keep
// the clock near 1800 MHz, so a decode or the whole codec step is faster at
// the power limit and no slower at full clock. 16-point blocks (three f32
// stages) and 64-point blocks (one stage) measured slower.
//
// B200 mapping (one persistent CTA of 18 warps per SM, warp-specialised):
//  * warp 0: 1-D bulk copies of each full tile's packed rows into a ring of
//    shared-memory stages (a partial last tile is read with plain loads);
//  * warps 2-9 (two builder warpgroups taking alternate tiles, one row per
//    thread): each pair of codes (each code byte at 2 bits) indexes a
//    lane-replicated table of value pairs and remainder pairs (packed fp16),
//    which go straight into tensor memory with tcgen05.st (A operand: row m
//    in lane m, two fp16 per 32-bit column, 8 columns per 16-element K-step);
//  * warp 1: per tile 2 d/16 MMAs (M = 128, N = 32, K = 16) with A from
//    tensor memory ([a-tmem] form) and B = H_32 (fp16 +-1, shared memory,
//    built once per CTA), f32 accumulators in tensor memory: two A operands
//    (the builders refill a half as soon as the MMAs that read it commit)
//    and one accumulator per epilogue warpgroup;
//  * warps 10-17 (two epilogue warpgroups, one row per thread): the
//    remaining butterfly stages across the 32-point blocks, the scale N / d,
//    the fp16 conversion and the sign flip on fp16 pairs, staged in the
//    group's 128-byte-swizzled tile and written by 2-D tensor stores (which
//    clip a partial last tile).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "tq_common.cuh"
#include "tq_umma.cuh"

namespace tq {

constexpr int DT_ROWS = 128;
constexpr int DT_WARPS = 18;  // copies, MMAs, 2 builder and 2 epilogue warpgroups
constexpr int DT_TMEM_COLS = 512;
constexpr size_t DT_SMEM_MAX = 232448;

template <int D, int BITS>
struct DtCfg {
  static constexpr int NB = D / 16;                 // 16-element K-steps per vector
  static constexpr int NB32 = D / 32;               // 32-point transform blocks per vector
  static constexpr int JP = 32 / NB32;              // positions per epilogue chunk (all blocks: 32 values)
  static constexpr int BOXES = D / 64;              // 64-column store boxes per tile
  static constexpr int P = D * BITS / 8;            // packed bytes per vector
  static constexpr int WORDS = P / 4;
  static constexpr int TILE_P = DT_ROWS * P;        // packed bytes of a full tile
  // 2 bits: one table entry per code byte (four codes, two A columns);
  // otherwise one per pair of codes (one A column)
  static constexpr bool QUAD = BITS == 2;
  static constexpr int E = QUAD ? 256 : 1 << (2 * BITS);  // table entries
  // tensor memory: NA A operands (values d/2 + remainders d/2 columns each),
  // then one accumulator (d columns) per epilogue warpgroup
  static constexpr int NA = 2;
  static constexpr int ACC0 = NA * D;
  static constexpr int STAGES = 8;
  // shared memory, from a 1024-aligned base
  static constexpr int OUT = 0;                     // 2 groups x BOXES x [128 rows x 128 B]
  static constexpr int OUT_BYTES = BOXES * DT_ROWS * 128;
  static constexpr int BREG = OUT + 2 * OUT_BYTES;  // H_32: 32 rows x 128 B (k < 32 used)
  static constexpr int IN = BREG + 32 * 128;        // STAGES x TILE_P
  static constexpr int LUT = IN + STAGES * TILE_P;  // E entries of 256 B (lane copies of values, remainders)
  static constexpr int BAR = LUT + E * 256;
  // full[S], empty[S], aready[NA][2], aempty[NA][2], tfull[2], tempty[2], done
  static constexpr int NBARS = 2 * STAGES + 4 * NA + 4 + 1;
  static constexpr int SLOT = BAR + NBARS * 8;
  // at 3 bits the table (64 entries of 256 B) starts at a shared address that
  // is a multiple of its 16 KB size, so an entry's address is the code pair's
  // bits shifted into place OR'd with the lane's offset (the base moves by up
  // to 15 KB for it); otherwise the base is 1024-aligned
  static constexpr uint32_t LUT_ALIGN = BITS == 3 ? 16384u : 1024u;
  static constexpr size_t BYTES = LUT_ALIGN + (size_t)SLOT + 16;
};

struct DtArgs {
  CUtensorMap tm_out;  // output as [n rows, d cols] fp16, box 64 x 128, 128-byte swizzle
  const uint8_t* packed;
  const float* norms;  // the offset variant: its side words (fp16 offset | fp16 scale << 16)
  int64_t n;
  uint32_t* err;
  long long wait_limit;
};

TQ_DEV uint2 dt_lds_u2(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

TQ_DEV uint32_t dt_lds_u32(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}

TQ_DEV void dt_tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}

TQ_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
TQ_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[bdesc]^T (A in tensor memory), one thread.
TQ_DEV void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// OS: the offset + fp16-scale variant (x_hat = offset + (scale / d) D H_pm c,
// the sign applied in f32 and the offset added before the fp16 rounding, as
// decode_kernel's offset instance does)
template <int D, int BITS, bool OS>
__global__ void __launch_bounds__(DT_WARPS * 32, 1)
    decode_tc_kernel(const __grid_constant__ tq_codec_tables T, const __grid_constant__ DtArgs a) {
  using Cfg = DtCfg<D, BITS>;
  constexpr int NB = Cfg::NB, S = Cfg::STAGES, NA = Cfg::NA, WORDS = Cfg::WORDS;
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  static_assert(Cfg::LUT % 1024 == 0, "the table offset keeps the base 1024-aligned");
  const uint32_t base = ((raw + (uint32_t)Cfg::LUT + Cfg::LUT_ALIGN - 1u) & ~(Cfg::LUT_ALIGN - 1u)) - (uint32_t)Cfg::LUT;
  uint8_t* sm = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the next kernel of the stream may start its own set-up as this grid's
  // CTAs exit (it waits for this grid before touching global memory)
  if (tid == 0) grid_dep_launch();

  const int64_t n_tiles = (a.n + DT_ROWS - 1) / DT_ROWS;
  const int cnt = (int64_t)blockIdx.x < n_tiles ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  auto tile_of = [&](int i) { return (int64_t)blockIdx.x + (int64_t)i * gridDim.x; };
  auto full_tile = [&](int i) { return (tile_of(i) + 1) * DT_ROWS <= a.n; };

  const uint32_t bar0 = base + Cfg::BAR;
  // full[s]: stage s holds tile i's rows; empty[s]: the builders read it;
  // aready[a][h] / aempty[a][h]: half h (blocks h d/32 ...) of A operand a
  // written / read by its MMAs;
  // tfull[g] / tempty[g]: accumulator g written / read by epilogue group g;
  // done: every MMA is done
  const uint32_t full0 = bar0, empty0 = bar0 + 8u * S, aready0 = bar0 + 16u * S, aempty0 = aready0 + 16u * NA,
                 tfull0 = aempty0 + 16u * NA, tempty0 = tfull0 + 16u, done_b = tempty0 + 16u;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 4);
    }
    for (int q = 0; q < 2 * NA; ++q) {
      mbar_init(aready0 + 8u * q, 4);
      mbar_init(aempty0 + 8u * q, 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(tfull0 + 8u * g, 1);
      mbar_init(tempty0 + 8u * g, 4);
    }
    mbar_init(done_b, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + Cfg::SLOT, DT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + Cfg::SLOT);
  // A operand k: values at columns k d + [0, d/2), remainders at + [d/2, d);
  // accumulator of epilogue group g at columns NA d + g d + [0, d).
  // The tables are filled after this point, so the first copies are in
  // flight meanwhile.

  // ---- code table, built by warps 2-17 (the epilogue warps have nothing to
  // do before the first accumulator). At 3 and 4 bits entry f = code_a |
  // code_b << BITS is 256 bytes: the A-operand column value_a | value_b << 16
  // for each of the 32 lanes, then the column remainder_a | remainder_b << 16
  // for each lane (fp16; value + remainder = level exactly: a 2^-14-grid
  // level below 4 has at most 16 significant bits, its fp16 remainder is a
  // multiple of 2^-14 below 2^-9). A lookup is two 4-byte loads (one
  // wavefront each, no bank conflict), so each word lands in the register
  // that its tensor-memory store reads, with no register moves between the
  // loads and the stores. At 2 bits an entry covers a whole code byte (two
  // columns) and a lookup is two 8-byte loads. Each thread computes one
  // entry and writes its share of the lane copies with 16-byte stores,
  // rotated so a warp's stores spread over banks.
  if (warp >= 2) {
    constexpr int E = Cfg::E, PER = 512 / E, LANES = 32 / PER;
    static_assert(E <= 512 && 512 % E == 0 && PER * LANES == 32, "one thread per entry and lane group");
    const int t = tid - 64, f = t / PER, part = t % PER;
    // the value word and the remainder word of the pair of codes pc
    auto pair_words = [&](int pc, uint32_t& ev, uint32_t& er) {
      const float ca = T.levels[pc & ((1 << BITS) - 1)], cb = T.levels[pc >> BITS];
      const __half va = __float2half_rn(ca), vb = __float2half_rn(cb);
      const __half ra = __float2half_rn(ca - __half2float(va)), rb = __float2half_rn(cb - __half2float(vb));
      ev = (uint32_t)__half_as_ushort(va) | ((uint32_t)__half_as_ushort(vb) << 16);
      er = (uint32_t)__half_as_ushort(ra) | ((uint32_t)__half_as_ushort(rb) << 16);
    };
    if constexpr (Cfg::QUAD) {
      // entry f = a code byte (pairs f & 15, f >> 4): 16 lane copies of its
      // two value words, then 16 of its two remainder words (8 bytes each;
      // an 8-byte load is served per half-warp, so 16 copies are enough for
      // conflict-free lookups); each of the two threads of an entry writes 8
      uint32_t ev0, er0, ev1, er1;
      pair_words(f & 15, ev0, er0);
      pair_words(f >> 4, ev1, er1);
      uint8_t* row = sm + Cfg::LUT + f * 256 + part * 64;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int jj = (j + t) & 3;
        *reinterpret_cast<uint4*>(row + jj * 16) = make_uint4(ev0, ev1, ev0, ev1);
        *reinterpret_cast<uint4*>(row + 128 + jj * 16) = make_uint4(er0, er1, er0, er1);
      }
    } else {
      uint32_t ev, er;
      pair_words(f, ev, er);
      uint8_t* row = sm + Cfg::LUT + f * 256 + part * LANES * 4;
      if constexpr (LANES < 4) {
#pragma unroll
        for (int j = 0; j < LANES; ++j) {
          reinterpret_cast<uint32_t*>(row)[j] = ev;
          reinterpret_cast<uint32_t*>(row + 128)[j] = er;
        }
      } else {
#pragma unroll
        for (int j = 0; j < LANES / 4; ++j) {
          const int jj = (j + t) % (LANES / 4);
          *reinterpret_cast<uint4*>(row + jj * 16) = make_uint4(ev, ev, ev, ev);
          *reinterpret_cast<uint4*>(row + 128 + jj * 16) = make_uint4(er, er, er, er);
        }
      }
    }
    // B = H_32 (natural order, +-1; the signs are applied to the fp16 output)
    // as an N = 32 by K = 32 operand, K-major with the 128-byte swizzle: row n
    // at n * 128 bytes, its 16-byte chunk c at c ^ (n % 8); K-step kh of a
    // block reads elements 16 kh ... 16 kh + 15 (descriptor start + 32 kh bytes)
    for (int e = t; e < 32 * 32; e += 512) {
      const int n = e >> 5, k = e & 31;
      const uint32_t off = Cfg::BREG + n * 128 + ((((k * 2) >> 4) ^ (n & 7)) << 4) + ((k * 2) & 15);
      *reinterpret_cast<uint16_t*>(sm + off) = (__popc(n & k) & 1) ? (uint16_t)0xBC00u : (uint16_t)0x3C00u;
    }
    fence_proxy_async_smem();  // B is read by the tensor cores
    asm volatile("bar.sync 3, 544;" ::: "memory");  // the table and B are complete (warps 1-17)
  }

  if (warp == 0) {
    // ---- producer: full tiles by one bulk copy each; the partial last tile
    // only completes the stage's phase (the builders load it themselves)
    if (lane == 0) {
      grid_dep_wait();  // the previous kernel of the stream may still write the codes
      for (int i = 0; i < cnt; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait_bounded(empty0 + 8u * s, ((i / S) - 1) & 1, a.wait_limit)) {
          record_error(a.err, TQ_DEVERR_TIMEOUT);
          break;
        }
        if (full_tile(i)) {
          mbar_arrive_expect_tx(full0 + 8u * s, Cfg::TILE_P);
          bulk_g2s(base + Cfg::IN + s * Cfg::TILE_P, a.packed + tile_of(i) * Cfg::TILE_P, Cfg::TILE_P, full0 + 8u * s);
        } else {
          mbar_arrive(full0 + 8u * s);
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: the 32-point block transforms S[b] = (A_value +
    // A_remainder)_b H_32^T, each accumulated over its two K-steps of both
    // parts (exact: see the top)
    asm volatile("bar.sync 3, 544;" ::: "memory");  // B (and the table) are built
    if (lane == 0) {
      grid_dep_wait();  // (its only global access is the error word)
      constexpr uint32_t IDESC = umma_idesc_f16(DT_ROWS, 32);
      bool ok = true;
      for (int i = 0; i < cnt && ok; ++i) {
        const int k = i % NA, g = i & 1;
        const uint32_t ab = tmem + (uint32_t)(k * D), db = tmem + (uint32_t)(Cfg::ACC0 + g * D);
        // each half of the A operand is multiplied as soon as it is written
        // and handed back as soon as its MMAs complete
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait_bounded(aready0 + 8u * (2 * k + h), (i / NA) & 1, a.wait_limit) ||
              (h == 0 && i >= 2 && !mbar_wait_bounded(tempty0 + 8u * g, ((i >> 1) - 1) & 1, a.wait_limit))) {
            record_error(a.err, TQ_DEVERR_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ks = h * NB / 2; ks < (h + 1) * NB / 2; ++ks) {
            // K-step ks: coordinates 16 ks ... 16 ks + 15 of the levels, half
            // ks % 2 of 32-point block ks / 2, whose S goes to columns 32 (ks / 2) ...
            const uint64_t bdesc = umma_desc_sw128(base + Cfg::BREG + 32 * (ks & 1));
            const uint32_t dcol = db + (uint32_t)(32 * (ks >> 1));
            umma_f16_ts(dcol, ab + (uint32_t)(8 * ks), bdesc, IDESC, (ks & 1) != 0);
            umma_f16_ts(dcol, ab + (uint32_t)(D / 2 + 8 * ks), bdesc, IDESC, true);
          }
          umma_commit(aempty0 + 8u * (2 * k + h));  // this half may be rewritten
        }
        if (ok) umma_commit(tfull0 + 8u * g);  // the accumulator may be read
      }
      umma_commit(done_b);
      if (!mbar_wait_bounded(done_b, 0, a.wait_limit)) record_error(a.err, TQ_DEVERR_TIMEOUT);
    }
  } else if (warp < 10) {
    // ---- builder warpgroup bg (warps 2 + 4 bg ... 5 + 4 bg): tiles bg, bg + 2,
    // ... into A operand bg; one row per thread (tensor-memory lane = tile row)
    const int bg = (warp - 2) >> 2, quarter = warp & 3, r = 32 * quarter + lane;
    const uint32_t lanebase = (uint32_t)(32 * quarter) << 16;
    const uint32_t lut_lane = base + Cfg::LUT + (Cfg::QUAD ? (uint32_t)(lane & 15) * 8u : (uint32_t)lane * 4u);
    grid_dep_wait();  // a partial tile's rows are read from global memory
    bool alive = true;
    for (int i = bg; i < cnt && alive; i += 2) {
      const int s = i % S, k = i % NA;
      if (!__all_sync(FULL, mbar_wait_bounded(full0 + 8u * s, (i / S) & 1, a.wait_limit))) {
        if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
        break;
      }
      const int64_t row = tile_of(i) * DT_ROWS + r;
      uint32_t words[WORDS];
      if (full_tile(i)) {
        const uint8_t* src = sm + Cfg::IN + s * Cfg::TILE_P + r * Cfg::P;
        if constexpr (Cfg::P % 16 == 0) {
#pragma unroll
          for (int w = 0; w < WORDS; w += 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + 4 * w);
            words[w] = v.x, words[w + 1] = v.y, words[w + 2] = v.z, words[w + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int w = 0; w < WORDS; w += 2) {
            const uint2 v = *reinterpret_cast<const uint2*>(src + 4 * w);
            words[w] = v.x, words[w + 1] = v.y;
          }
        }
      } else {
#pragma unroll
        for (int w = 0; w < WORDS; ++w) words[w] = 0u;
        if (row < a.n) {
          const uint32_t* src = reinterpret_cast<const uint32_t*>(a.packed + row * Cfg::P);
#pragma unroll
          for (int w = 0; w < WORDS; ++w) words[w] = __ldg(src + w);
        }
      }
      const uint32_t sb = tmem + lanebase + (uint32_t)(k * D);
      // A column p = pair of coordinates (2p, 2p + 1), 16 columns per store;
      // half h = value (and remainder) columns [h d/4, (h + 1) d/4)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (i >= NA &&
            !__all_sync(FULL, mbar_wait_bounded(aempty0 + 8u * (2 * k + h), ((i / NA) - 1) & 1, a.wait_limit))) {
          if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
          alive = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c0 = h * D / 4; c0 < (h + 1) * D / 4; c0 += 16) {
          uint32_t vv[16], rr[16];
          if constexpr (Cfg::QUAD) {
            // code byte c0 / 2 + j -> columns c0 + 2j, c0 + 2j + 1, by two
            // 8-byte loads (values, remainders) into consecutive registers
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int byte = c0 / 2 + j;
              const uint32_t f = __byte_perm(words[byte >> 2], 0u, 0x4440u | (uint32_t)(byte & 3));
              const uint2 v2 = dt_lds_u2(f * 256u + lut_lane), r2 = dt_lds_u2(f * 256u + lut_lane + 128u);
              vv[2 * j] = v2.x, vv[2 * j + 1] = v2.y;
              rr[2 * j] = r2.x, rr[2 * j + 1] = r2.y;
            }
          } else {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              constexpr int FB = 2 * BITS;
              const int off = (c0 + t) * FB;
              uint32_t addr;  // the code pair's table entry for this lane
              if constexpr (FB == 8) {  // 4 bits: a pair is a byte
                const uint32_t f = __byte_perm(words[off >> 5], 0u, 0x4440u | (uint32_t)((off >> 3) & 3));
                addr = f * 256u + lut_lane;
              } else {  // 3 bits: the 6-bit pair shifted to bits 8-13, OR'd with the aligned lane offset
                static_assert(Cfg::E == 64 && Cfg::LUT_ALIGN == 16384u, "aligned 3-bit table");
                const int sh = off & 31;
                uint32_t g;
                if (sh + FB > 32)
                  g = __funnelshift_r(words[off >> 5], words[(off >> 5) + 1], sh - 8);
                else
                  g = sh >= 8 ? words[off >> 5] >> (sh - 8) : words[off >> 5] << (8 - sh);
                addr = (g & 0x3F00u) | lut_lane;
              }
              // the value pair and the remainder pair by two 4-byte loads, so
              // each lands in the register its tensor-memory store reads
              vv[t] = dt_lds_u32(addr);
              rr[t] = dt_lds_u32(addr + 128u);
            }
          }
          tmem_st16(sb + (uint32_t)c0, vv);
          tmem_st16(sb + (uint32_t)(D / 2 + c0), rr);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(aready0 + 8u * (2 * k + h));
      }
      // The stage is handed back only once every word read from it has been
      // consumed by a tensor-memory store that has completed: a release right
      // after the loads let the next tile's copy land before loads that the
      // compiler had scheduled later (seen at 4 bits, d = 128).
      if (alive && lane == 0) mbar_arrive(empty0 + 8u * s);
    }
  } else {
    // ---- epilogue warpgroup g (warps 10 + 4g ... 13 + 4g): tiles g, g + 2, ...
    const int g = (warp - 10) >> 2, quarter = warp & 3, r = 32 * quarter + lane;
    const bool leader = warp == 10 + 4 * g && lane == 0;
    const uint32_t lanebase = (uint32_t)(32 * quarter) << 16;
    const uint32_t stage_out = base + Cfg::OUT + (uint32_t)(g * Cfg::OUT_BYTES);
    uint8_t* out_sm = sm + Cfg::OUT + g * Cfg::OUT_BYTES;
    bool stored_once = false;
    // norms are loaded one tile ahead, so their latency is off the chain
    auto load_norm = [&](int i) {
      const int64_t row = tile_of(i) * DT_ROWS + r;
      return (i < cnt && row < a.n) ? __ldg(a.norms + row) : 0.f;
    };
    grid_dep_wait();  // before the first norm load and the first store
    float nrm_next = load_norm(g);
    for (int i = g; i < cnt; i += 2) {
      const float nrm = nrm_next;
      nrm_next = load_norm(i + 2);
      const bool ok = mbar_wait_bounded(tfull0 + 8u * g, (i >> 1) & 1, a.wait_limit);
      if (!__all_sync(FULL, ok)) {
        if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int64_t tile = tile_of(i);
      float scale = nrm, mu = 0.f;
      if constexpr (OS) {
        const uint32_t sw32 = __float_as_uint(nrm);
        mu = __half2float(__ushort_as_half((unsigned short)(sw32 & 0xffffu)));
        scale = __half2float(__ushort_as_half((unsigned short)(sw32 >> 16)));
      }
      const float sc = scale * (1.0f / (float)D);
      const f2 sc2 = make_float2(sc, sc), mu2 = make_float2(mu, mu);
      // the group's staging tile must have been read by its previous store
      if (leader && stored_once) bulk_wait_read<0>();
      asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory");
      const uint32_t tl = tmem + lanebase + (uint32_t)(Cfg::ACC0 + g * D);
      // column 32 b + j of the accumulator is S[b][j]; per tensor-memory wait
      // positions JP c ... JP c + JP - 1 of every block (32 values), then the
      // log2(d / 32) remaining stages of the transform across the blocks in
      // f32 pairs, which gives coordinates 32 b' + JP c ... of H_pm c
      constexpr int NB32 = Cfg::NB32, JP = Cfg::JP;
#pragma unroll
      for (int c = 0; c < 32 / JP; ++c) {
        uint32_t rv[NB32][JP];
#pragma unroll
        for (int b = 0; b < NB32; ++b) {
          if constexpr (JP == 8)
            tmem_ld8(tl + (uint32_t)(32 * b + JP * c), rv[b]);
          else
            tmem_ld16(tl + (uint32_t)(32 * b + JP * c), rv[b]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int b = 0; b < NB32; ++b) tmem_regs_after_wait(rv[b]);
        if (c == 32 / JP - 1) {  // every load of the accumulator is done: free the slot
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8u * g);
        }
        f2 x[JP / 2][NB32];  // x[p][b] = S[b][JP c + 2p], S[b][JP c + 2p + 1]
#pragma unroll
        for (int p = 0; p < JP / 2; ++p) {
#pragma unroll
          for (int b = 0; b < NB32; ++b)
            x[p][b] = make_float2(__uint_as_float(rv[b][2 * p]), __uint_as_float(rv[b][2 * p + 1]));
          wht_pairs<NB32>(x[p]);  // exact: sums of multiples of 2^-14 below 2^9
        }
#pragma unroll
        for (int b = 0; b < NB32; ++b) {
          const int k0 = 32 * b + JP * c;  // first coordinate of these JP
          uint32_t hw[JP / 2];
#pragma unroll
          for (int p = 0; p < JP / 2; ++p) {
            const f2 y = mul2(x[p][b], sc2);
            if constexpr (OS) {
              const uint32_t m0 = T.sign_f32[k0 + 2 * p], m1 = T.sign_f32[k0 + 2 * p + 1];
              const f2 ys = add2(make_float2(__uint_as_float(__float_as_uint(y.x) ^ m0),
                                             __uint_as_float(__float_as_uint(y.y) ^ m1)),
                                 mu2);
              const __half2 hv = __floats2half2_rn(ys.x, ys.y);
              hw[p] = *reinterpret_cast<const uint32_t*>(&hv);
            } else {
              const __half2 hv = __floats2half2_rn(y.x, y.y);
              hw[p] = *reinterpret_cast<const uint32_t*>(&hv) ^ T.sign_h2[(k0 >> 1) + p];
            }
          }
          // 16 bytes of the swizzled staging row per 8 coordinates
#pragma unroll
          for (int q = 0; q < JP / 8; ++q) {
            const int kk = k0 + 8 * q, box = kk >> 6, col = kk & 63;
            const uint32_t off = (uint32_t)(box * DT_ROWS * 128 + r * 128) + ((uint32_t)((col >> 3) ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(out_sm + off) = make_uint4(hw[4 * q], hw[4 * q + 1], hw[4 * q + 2], hw[4 * q + 3]);
          }
        }
      }
      fence_proxy_async_smem();
      asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory");
      if (leader) {
        // rows past the end of a partial tile are clipped by the tensor store
#pragma unroll
        for (int bx = 0; bx < Cfg::BOXES; ++bx)
          dt_tma_store_2d(&a.tm_out, 64 * bx, (int)(tile * DT_ROWS), stage_out + (uint32_t)(bx * DT_ROWS * 128));
        bulk_commit();
        stored_once = true;
      }
    }
    if (leader) bulk_wait_all<0>();
  }
  // ---- teardown: every role is done (or gave up); free the tensor memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, DT_TMEM_COLS);
  }
}

template <int D, int BITS, bool OS>
static cudaError_t launch_decode_tc_t(const tq_codec_tables& T, DtArgs a, void* x, cudaStream_t st) {
  using Cfg = DtCfg<D, BITS>;
  static_assert(Cfg::BYTES <= DT_SMEM_MAX, "shared memory of the tensor-core decode");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> configured{0};  // one bit per device
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(decode_tc_kernel<D, BITS, OS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::BYTES);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tq_tensor_map_encode_fn());
  if (!enc) return cudaErrorNotSupported;
  const int sms = tq_sm_count(dev);
  // launches of at most 2^30 rows keep the store coordinates in int32
  const int64_t max_rows = (int64_t)1 << 30;
  const int64_t n_total = a.n;
  const uint8_t* packed0 = a.packed;
  const float* norms0 = a.norms;
  for (int64_t off = 0; off < n_total; off += max_rows) {
    const int64_t n = std::min(max_rows, n_total - off);
    a.n = n;
    a.packed = packed0 + off * Cfg::P;
    a.norms = norms0 + off;
    __half* xo = static_cast<__half*>(x) + off * D;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)n};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)DT_ROWS};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&a.tm_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, static_cast<void*>(xo), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
    const int64_t tiles = (n + DT_ROWS - 1) / DT_ROWS;
    const int grid = (int)std::min<int64_t>(tiles, (int64_t)sms);
    e = tq_launch_pdl(decode_tc_kernel<D, BITS, OS>, dim3(grid), dim3(DT_WARPS * 32), Cfg::BYTES, st, T, a);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq

using namespace tq;

namespace {

tq_status launch_decode_tc_any(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x,
                               void* stream, bool os) {
  if (n == 0) return TQ_OK;
  if (ctx->d > 128) return TQ_ERR_UNSUPPORTED;  // one tile would fill tensor memory
  DtArgs a;
  memset(&a, 0, sizeof(a));
  a.n = n;
  a.packed = static_cast<const uint8_t*>(packed);
  a.norms = norms;
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.wait_limit = TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
  const tq_codec_tables& T = ctx->t;
#define TQ_DECTC_CASE(D_, B_)                                                       \
  if (ctx->d == D_ && ctx->bits == B_)                                              \
    e = os ? launch_decode_tc_t<D_, B_, true>(T, a, x, st) : launch_decode_tc_t<D_, B_, false>(T, a, x, st);
  TQ_DECTC_CASE(64, 2) TQ_DECTC_CASE(64, 3) TQ_DECTC_CASE(64, 4)
  TQ_DECTC_CASE(128, 2) TQ_DECTC_CASE(128, 3) TQ_DECTC_CASE(128, 4)
#undef TQ_DECTC_CASE
  if (e == cudaErrorNotSupported) return TQ_ERR_UNSUPPORTED;
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace

tq_status tq_launch_decode_tc(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x,
                              void* stream) {
  return launch_decode_tc_any(ctx, packed, norms, n, x, stream, false);
}

tq_status tq_launch_decode_tc_os(const tq_ctx* ctx, const void* packed, const uint32_t* side, int64_t n, void* x,
                                 void* stream) {
  return launch_decode_tc_any(ctx, packed, reinterpret_cast<const float*>(side), n, x, stream, true);
}
