// Decode kernel: (packed codes, f32 norms) -> fp16 vectors.
//
// Method ("aither-kvcache" PyPI page, section "Algorithm": decoding reverses
// steps 4-1): unpack the indices, look up the levels c[idx], undo the scaled
// rotation and multiply by the norm:
//   x_hat = N * D H (c[idx] / sqrt(d)) = D (H_pm c[idx]) * (N / d),
// H_pm the unnormalised +-1 Walsh-Hadamard matrix. The levels lie on the
// 2^-14 grid and |H_pm c| < 2^10, so H_pm c is exact in f32 in any order; the
// only roundings are the product by N/d (a power-of-two scaling of N, exact)
// in f32 and the final fp16 conversion.
//
// B200 mapping: every lane owns 64 coordinates (1, 2 or 4 lanes per vector),
// 16 warps per SM. Each warp runs a 3-stage pipeline of 1-D bulk copies (TMA)
// bringing its tile of packed rows and norms into shared memory (one copy each
// per tile); a lane-replicated table indexed by two codes returns
// (c[a] + c[b], c[a] - c[b]), the levels already through the first
// butterfly; the other stages run in registers with f32x2 add/sub and
// shuffles across the lanes of a vector. The fp16 rows are staged in the
// warp's 4 KB output tile in the 128-byte swizzled layout (16-byte chunk c of
// row r at position c ^ (r % 8): conflict-free stores of natural chunks) and
// leave through one 2-D tensor store (TMA) per tile, which also clips a
// partial last tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "tq_common.cuh"

namespace tq {

constexpr int DEC_WARPS = 16;
constexpr int DEC_STAGES = 3;
constexpr int DEC_C = 64;

template <int D, int BITS>
struct DecCfg {
  static constexpr int C = DEC_C;
  static constexpr int LPV = D / C;
  static constexpr int NP = C / 2;
  static constexpr int VPW = 32 / LPV;
  static constexpr int P = D * BITS / 8;
  static constexpr int PL = C * BITS / 8;  // packed bytes per lane: 16, 24, 32
  static constexpr int WL = PL / 4;
  static constexpr int E = 1 << (2 * BITS);  // pair-table entries
  static constexpr int TILE_P = 32 * PL;     // packed bytes of a full tile
  static constexpr int PACK_BYTES = TILE_P;   // lane rows contiguous, as in memory
  static constexpr int IN_STAGE = PACK_BYTES + VPW * 4;  // packed rows + norms
  static constexpr int OUT = 32 * 2 * C;                  // the warp's output tile (4 KB)
};

// Shared memory: header, input stages, then (1024-byte aligned, for the
// swizzle pattern of the tensor store) the warps' output tiles and the pair
// table. The dynamic window's base is only 16-byte aligned, so the kernel
// rounds the output region up at run time (1 KB of slack is reserved).
template <int D, int BITS>
struct DecSmem {
  using Cfg = DecCfg<D, BITS>;
  static constexpr int BAR = 0;     // warps x stages u64
  static constexpr int MASK = 512;  // sign masks, up to 128 u32
  static constexpr int IN = MASK + 512;
  static constexpr int STAGE = (Cfg::IN_STAGE + 15) / 16 * 16;
  static constexpr int OUT = IN + DEC_WARPS * DEC_STAGES * STAGE;  // before rounding up to 1024
  static constexpr int OUT_BYTES = DEC_WARPS * Cfg::OUT;
  static constexpr size_t BYTES = (size_t)OUT + 1024 + OUT_BYTES + (size_t)Cfg::E * 32 * 8;
};

struct DecArgs {
  CUtensorMap tm_x;  // output as [n * lanes-per-vector rows, 64] fp16, box 64 x 32, 128-byte swizzle
  const uint8_t* packed;
  const float* norms;
  int64_t n;
  __half* x;
  uint32_t* err;
  long long wait_limit;
  int norms_bulk;  // norms pointer 16-byte aligned: norms tiles come by bulk copy
};

TQ_DEV void tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}

TQ_DEV f2 lds_f2(uint32_t addr) {
  f2 r;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(r.x), "=f"(r.y) : "r"(addr));
  return r;
}

template <int D, int BITS, bool OS>
__global__ void __launch_bounds__(DEC_WARPS * 32, 1)
    decode_kernel(const __grid_constant__ tq_codec_tables T, const __grid_constant__ DecArgs a) {
  using Cfg = DecCfg<D, BITS>;
  using Sm = DecSmem<D, BITS>;
  constexpr int C = Cfg::C, NP = Cfg::NP, LPV = Cfg::LPV, VPW = Cfg::VPW, WL = Cfg::WL;
  constexpr int E = Cfg::E;
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // programmatic dependent launch: the next kernel may set up as CTAs exit
  if (threadIdx.x == 0) grid_dep_launch();
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t out_addr = (smem_base + Sm::OUT + 1023u) & ~1023u;
  const uint32_t lut_addr = out_addr + Sm::OUT_BYTES;

  // pair table: entry (f, lane) with f = code_a | code_b << BITS holds
  // (c[a] + c[b], c[a] - c[b]) -- exact in f32 (2^-14 grid).
  {
    f2* lut = reinterpret_cast<f2*>(smem + (lut_addr - smem_base));
    for (int e = threadIdx.x; e < E * 32; e += blockDim.x) {
      const int f = e >> 5;
      const float ca = T.levels[f & ((1 << BITS) - 1)];
      const float cb = T.levels[f >> BITS];
      lut[e] = make_float2(ca + cb, ca - cb);
    }
  }
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem + Sm::MASK);
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) smask[i] = T.sign_h2[i];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sm::BAR) + warp * DEC_STAGES;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < DEC_STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();

  uint8_t* in0 = smem + Sm::IN + warp * DEC_STAGES * Sm::STAGE;
  const uint32_t otile = out_addr + (uint32_t)(warp * Cfg::OUT);
  uint8_t* orow = smem + (otile - smem_base) + lane * 2 * C;
  const uint32_t sw = (uint32_t)lane & 7u;  // swizzle of this lane's output row
  const uint32_t lut_lane = lut_addr + lane * 8u;
  const int part = lane & (LPV - 1);
  const uint4* my_masks = reinterpret_cast<const uint4*>(smask + part * NP);

  const int64_t n_tiles = (a.n + VPW - 1) / VPW;
  const int64_t gw = (int64_t)blockIdx.x * DEC_WARPS + warp;
  const int64_t n_warps = (int64_t)gridDim.x * DEC_WARPS;
  constexpr int NORM_OFF = Cfg::PACK_BYTES;

  // Full tiles come through bulk copies; the last, partial tile (if any) is
  // read with plain loads (its byte count need not be a multiple of 16).
  auto full_tile = [&](int64_t tile) { return (tile + 1) * VPW <= a.n; };
  auto issue = [&](int64_t tile, int stage) {  // called by the whole warp
    if (!full_tile(tile)) return;
    const uint32_t bar = smem_u32(&bars[stage]);
    uint8_t* dst = in0 + stage * Sm::STAGE;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, (uint32_t)(Cfg::TILE_P + (a.norms_bulk ? VPW * 4 : 0)));
      if (a.norms_bulk) bulk_g2s(smem_u32(dst + NORM_OFF), a.norms + tile * VPW, VPW * 4, bar);
      bulk_g2s(smem_u32(dst), a.packed + tile * Cfg::TILE_P, Cfg::TILE_P, bar);
    }
    __syncwarp();
  };

  grid_dep_wait();  // the previous kernel of the stream may still write the codes
#pragma unroll
  for (int s = 0; s < DEC_STAGES; ++s) {
    const int64_t t = gw + s * n_warps;
    if (t < n_tiles) issue(t, s);
  }

  int stage = 0;
  uint32_t parity = 0;
  bool stored_once = false;
  for (int64_t tile = gw; tile < n_tiles; tile += n_warps) {
    const int64_t v0 = tile * VPW;
    const int valid_lanes = (int)min64(VPW, a.n - v0) * LPV;
    const bool active = lane < valid_lanes;
    const int vl = lane / LPV;  // vector within the tile
    uint32_t words[WL];
    float nrm = 0.f;
    if (full_tile(tile)) {
      const bool ok =
          __all_sync(FULL, mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u, a.wait_limit));
      if (!ok) {
        if (lane == 0) record_error(a.err, TQ_DEVERR_TIMEOUT);
#pragma unroll
        for (int s = 1; s < DEC_STAGES; ++s) {
          const int os = (stage + s) % DEC_STAGES;
          if (tile + s * n_warps < n_tiles && full_tile(tile + s * n_warps))
            (void)mbar_wait_bounded(smem_u32(&bars[os]), (parity >> os) & 1u, a.wait_limit);
        }
        if (lane == 0) bulk_wait_all<0>();
        return;
      }
      parity ^= 1u << stage;
      const uint8_t* st = in0 + stage * Sm::STAGE;
      const uint8_t* row = st + lane * Cfg::PL;
      if (Cfg::PL % 16 == 0) {
#pragma unroll
        for (int w = 0; w < WL / 4; ++w) {
          const uint4 r = reinterpret_cast<const uint4*>(row)[w];
          words[4 * w] = r.x;
          words[4 * w + 1] = r.y;
          words[4 * w + 2] = r.z;
          words[4 * w + 3] = r.w;
        }
      } else {
#pragma unroll
        for (int w = 0; w < WL / 2; ++w) {
          const uint2 r = reinterpret_cast<const uint2*>(row)[w];
          words[2 * w] = r.x;
          words[2 * w + 1] = r.y;
        }
      }
      nrm = a.norms_bulk ? reinterpret_cast<const float*>(st + NORM_OFF)[vl] : __ldg(a.norms + v0 + vl);
    } else {
#pragma unroll
      for (int w = 0; w < WL; ++w) words[w] = 0;
      if (active) {
        const uint32_t* row = reinterpret_cast<const uint32_t*>(a.packed + v0 * Cfg::P) + lane * WL;
#pragma unroll
        for (int w = 0; w < WL; ++w) words[w] = __ldg(row + w);
        nrm = __ldg(a.norms + v0 + vl);
      }
    }
    __syncwarp();
    // the stage has been read into registers: refill it
    {
      const int64_t next = tile + DEC_STAGES * n_warps;
      if (next < n_tiles) issue(next, stage);
    }

    // ---- unpack pairs of codes -> levels through the first butterfly
    f2 v[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      constexpr int FB = 2 * BITS;
      const int off = j * FB;
      uint32_t f = words[off >> 5] >> (off & 31);
      if ((off & 31) + FB > 32) f |= words[(off >> 5) + 1] << (32 - (off & 31));
      f &= (uint32_t)(E - 1);
      v[j] = lds_f2(f * 256u + lut_lane);
    }
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

    // ---- scale by N/d, round to fp16, apply the signs, stage the tile. The
    // offset variant's side word is fp16 offset | fp16 scale << 16: it
    // scales by scale/d, flips signs in f32 and adds the offset before the
    // rounding.
    float mu = 0.f;
    if constexpr (OS) {
      const uint32_t sw32 = __float_as_uint(nrm);
      mu = __half2float(__ushort_as_half((unsigned short)(sw32 & 0xffffu)));
      nrm = __half2float(__ushort_as_half((unsigned short)(sw32 >> 16)));
    }
    const float sc = nrm * (1.0f / (float)D);
    const f2 sc2 = make_float2(sc, sc);
    // the previous tile's bulk store must have finished reading the buffer
    if (lane == 0 && stored_once) bulk_wait_read<0>();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < C / 8; ++c) {
      uint32_t h[4];
      if constexpr (OS) {
        const f2 mu2 = make_float2(mu, mu);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i0 = 2 * (4 * c + q);  // coordinate within this lane's part
          uint32_t m0, m1;
          if constexpr (LPV == 1) {
            m0 = T.sign_f32[i0], m1 = T.sign_f32[i0 + 1];
          } else if constexpr (LPV == 2) {
            m0 = T.sign_f32[i0], m1 = T.sign_f32[i0 + 1];
            if (part) m0 ^= T.sign_f32_dx[i0], m1 ^= T.sign_f32_dx[i0 + 1];
          } else {
            const uint32_t mh = reinterpret_cast<const uint32_t*>(my_masks)[4 * c + q];
            m0 = (mh << 16) & 0x80000000u, m1 = mh & 0x80000000u;
          }
          f2 y = mul2(v[4 * c + q], sc2);
          y = make_float2(__uint_as_float(__float_as_uint(y.x) ^ m0), __uint_as_float(__float_as_uint(y.y) ^ m1));
          y = add2(y, mu2);
          const __half2 hv = __floats2half2_rn(y.x, y.y);
          h[q] = *reinterpret_cast<const uint32_t*>(&hv);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const f2 y = mul2(v[4 * c + q], sc2);
          const __half2 hv = __floats2half2_rn(y.x, y.y);
          h[q] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        if constexpr (LPV <= 2) {  // masks from the constant bank
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            h[q] ^= T.sign_h2[4 * c + q];
            if (LPV == 2 && part) h[q] ^= T.sign_h2_dx[4 * c + q];
          }
        } else {
          const uint4 mk = my_masks[c];
          h[0] ^= mk.x, h[1] ^= mk.y, h[2] ^= mk.z, h[3] ^= mk.w;
        }
      }
      *reinterpret_cast<uint4*>(orow + 16 * (c ^ sw)) = make_uint4(h[0], h[1], h[2], h[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      // rows past the end of a partial tile are clipped by the tensor store
      tma_store_2d(&a.tm_x, 0, (int)(tile * 32), otile);
      bulk_commit();
      stored_once = true;
    }
    if (++stage == DEC_STAGES) stage = 0;
  }
  if (lane == 0) bulk_wait_all<0>();
}

template <int D, int BITS, bool OS>
static cudaError_t launch_decode_t(const tq_codec_tables& T, DecArgs a, cudaStream_t st) {
  using Cfg = DecCfg<D, BITS>;
  constexpr size_t smem = DecSmem<D, BITS>::BYTES;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> configured{0};
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(decode_kernel<D, BITS, OS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tq_tensor_map_encode_fn());
  if (!enc) return cudaErrorNotSupported;
  // launches of at most 2^30 lane-rows keep the store coordinates in int32
  const int64_t max_vec = ((int64_t)1 << 30) / Cfg::LPV;
  const int64_t n_total = a.n;
  const uint8_t* packed0 = a.packed;
  const float* norms0 = a.norms;
  __half* x0 = a.x;
  for (int64_t off = 0; off < n_total; off += max_vec) {
    const int64_t n = std::min(max_vec, n_total - off);
    a.n = n;
    a.packed = packed0 + off * Cfg::P;
    a.norms = norms0 + off;
    a.x = x0 + off * D;
    a.norms_bulk = (reinterpret_cast<uintptr_t>(a.norms) & 15u) == 0;
    const cuuint64_t dims[2] = {(cuuint64_t)Cfg::C, (cuuint64_t)(n * Cfg::LPV)};
    const cuuint64_t strides[1] = {(cuuint64_t)Cfg::C * 2};
    const cuuint32_t box[2] = {(cuuint32_t)Cfg::C, 32u};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&a.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, static_cast<void*>(a.x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
    const int64_t tiles = (n + Cfg::VPW - 1) / Cfg::VPW;
    const int64_t ctas = (tiles + DEC_WARPS - 1) / DEC_WARPS;
    const int grid = (int)std::min<int64_t>(ctas, (int64_t)tq_sm_count(dev));
    e = tq_launch_pdl(decode_kernel<D, BITS, OS>, dim3(grid), dim3(DEC_WARPS * 32), smem, st, T, a);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq

using namespace tq;

tq_status tq_launch_decode(const tq_ctx* ctx, const void* packed, const float* norms, int64_t n, void* x,
                           void* stream) {
  if (n == 0) return TQ_OK;
  DecArgs a;
  memset(&a, 0, sizeof(a));
  a.packed = static_cast<const uint8_t*>(packed);
  a.norms = norms;
  a.n = n;
  a.x = static_cast<__half*>(x);
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.wait_limit = TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
#define TQ_DEC_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_decode_t<D_, B_, false>(ctx->t, a, st);
  TQ_DEC_CASE(64, 2) TQ_DEC_CASE(64, 3) TQ_DEC_CASE(64, 4)
  TQ_DEC_CASE(128, 2) TQ_DEC_CASE(128, 3) TQ_DEC_CASE(128, 4)
  TQ_DEC_CASE(256, 2) TQ_DEC_CASE(256, 3) TQ_DEC_CASE(256, 4)
#undef TQ_DEC_CASE
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_launch_decode_os(const tq_ctx* ctx, const void* packed, const uint32_t* side, int64_t n, void* x,
                              void* stream) {
  if (n == 0) return TQ_OK;
  DecArgs a;
  memset(&a, 0, sizeof(a));
  a.packed = static_cast<const uint8_t*>(packed);
  a.norms = reinterpret_cast<const float*>(side);  // side words travel in the norms slot, bit for bit
  a.n = n;
  a.x = static_cast<__half*>(x);
  a.err = tq_error_word();
  if (!a.err) return TQ_ERR_CUDA;
  a.wait_limit = TQ_WAIT_LIMIT_CYCLES;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
#define TQ_DECOS_CASE(D_, B_) \
  if (ctx->d == D_ && ctx->bits == B_) e = launch_decode_t<D_, B_, true>(ctx->t, a, st);
  TQ_DECOS_CASE(64, 2) TQ_DECOS_CASE(64, 3) TQ_DECOS_CASE(64, 4)
  TQ_DECOS_CASE(128, 2) TQ_DECOS_CASE(128, 3) TQ_DECOS_CASE(128, 4)
  TQ_DECOS_CASE(256, 2) TQ_DECOS_CASE(256, 3) TQ_DECOS_CASE(256, 4)
#undef TQ_DECOS_CASE
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
