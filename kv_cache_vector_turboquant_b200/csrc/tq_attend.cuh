// Definitions shared by the two partial-attention kernels (tq_attend.cu: any
// bit widths; tq_attend_fast.cu: 4-bit keys with 2-bit values) and the split
// merge kernel: the launch arguments, the split-S geometry and small warp /
// tensor-core helpers.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "tq_common.cuh"

namespace tq {

constexpr int ATT_WARPS = 8;   // warps per CTA of the generic kernel: one per (kv head, group of 4 query heads)
constexpr int ATT_STAGES = 2;  // position tiles in flight (generic kernel)
constexpr int ATT_TILE = 32;   // positions per tile (two blocks of 16)
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
  // paged caches (block_tables non-null): K/V rows of position s of sequence
  // b are in block block_tables[b * max_blocks + s / 16], row s % 16, of a
  // cache of num_blocks blocks of 16 positions
  const int32_t* block_tables;
  int max_blocks;
  int64_t num_blocks;
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
  int nt;     // column tiles per kv head: 1 (<= 4 query heads per kv head) or 2
  int hw_max; // kv heads per CTA
  float q_scale;  // log2(e) / (d sqrt(d))
};

// Split count and chunk for `ctas` CTAs per kv-head group (one wave), chunks
// a multiple of the tile.
inline void attn_split_for(int64_t ctas, int B, int64_t s_max, int* n_split, int* chunk) {
  const int64_t tiles = (s_max + ATT_TILE - 1) / ATT_TILE;
  int64_t ns = ctas / (int64_t)B;
  ns = std::max<int64_t>(1, std::min<int64_t>(ns, tiles));
  const int64_t tiles_per = (tiles + ns - 1) / ns;
  *chunk = (int)(tiles_per * ATT_TILE);
  *n_split = (int)((tiles + tiles_per - 1) / tiles_per);
}

// Split geometry of the generic kernel. Depends only on (B, s_max), so the
// workspace size does too; it is the largest split count of either kernel.
inline void attn_split(int B, int64_t s_max, int* n_split, int* chunk) {
  attn_split_for(ATT_TARGET_CTAS, B, s_max, n_split, chunk);
}

inline size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

constexpr int ATT_BLOCK = 16;  // positions per block of a paged cache

// Cache row (position row, all kv heads) of position s of sequence b. A block
// number outside [0, num_blocks) is clamped and flagged.
TQ_DEV int64_t attn_pos_row(const AttnArgs& a, int b, int64_t s) {
  if (a.block_tables == nullptr) return (int64_t)b * a.s_max + s;
  int64_t blk = __ldg(a.block_tables + (int64_t)b * a.max_blocks + (s / ATT_BLOCK));
  if (blk < 0 || blk >= a.num_blocks) {
    record_error(a.err, TQ_DEVERR_BLOCK_RANGE);
    blk = blk < 0 ? 0 : a.num_blocks - 1;
  }
  return blk * ATT_BLOCK + (s % ATT_BLOCK);
}

TQ_DEV float warp_max8(float v) {  // max over the 8 lanes sharing lane & 3
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
}
TQ_DEV float warp_sum8(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  return v + __shfl_xor_sync(0xffffffffu, v, 16);
}

TQ_DEV uint32_t lds32(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}

// D += A * B on the tensor cores: m16n8k16, fp16 operands, f32 accumulate.
TQ_DEV void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

TQ_DEV uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace tq

// Launch of the split merge kernel (tq_attend.cu) for the arguments of either
// partial kernel.
cudaError_t tq_launch_attend_combine(const tq::AttnArgs& a, int d, cudaStream_t st);

// The fast partial kernel (tq_attend_fast.cu): returns cudaErrorNotSupported,
// launching nothing, when the shapes, widths or alignments are not ones it
// handles; otherwise launches the partial and merge kernels.
cudaError_t tq_launch_attend_fast(tq::AttnArgs& a, int d, int k_bits, int v_bits, int sm_count, cudaStream_t st);
