// Fused adapter switching for every layer in one pass (the merge path).
//
// "AdaFuse: Accelerating Dynamic Adapter Inference via Token-Level Pre-Gating
// and Fused Kernel Optimization", 方法详解, 关键设计 items 2 and 3: when the
// active adapters change between tokens, the previous ones are unmerged
// (negative weights) and the current ones merged (positive weights) as one
// update W <- W + DOWN·UP, DOWN = [-A_prev | A_cur], UP = [B_prev ; B_cur], and
// the updates of all layers are one launch, added in place into the backbone.
//
// Here the update runs on the fused GEMM kernel in its merge mode: DOWN is the
// A operand, written first by lora_switch_images_kernel as the same 128-row x
// 64-column swizzled bf16 images the forward's s·U uses (each term's c·A split
// into a hi and a lo bf16 part, so the weighted factor keeps ~16 bits), UP is
// the terms' B_pool rows, and the epilogue adds the accumulator to W in place.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace lora {

// img[tile][block][...] = the swizzled image of tile `tile` (layer l = tile /
// mt_per_layer, rows (tile % mt_per_layer) * 128 .. of that layer's d_in): column
// kofs + k of a term holds hi(c·A_l[pool_row + k][row]), column kofs + kc + k
// the remainder lo, zero for k >= rank and for rows past d_in. One thread per
// (tile, 8-column group, row): consecutive threads take consecutive rows, so the
// reads of A_pool's rows are coalesced.
__global__ void lora_switch_images_kernel(const uint16_t *__restrict__ A_pool, const SwitchTerm *__restrict__ terms,
                                          int n_terms, int64_t R, int64_t d_in, int mt_per_layer, int64_t n_tiles,
                                          int kaug, int64_t img_bytes, uint8_t *__restrict__ img) {
  const int groups = kaug / 8;
  const int64_t n = n_tiles * groups * kTileM;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(e % kTileM);
    const int64_t tg = e / kTileM;
    const int g = static_cast<int>(tg % groups);
    const int64_t tile = tg / groups;
    const int64_t l = tile / mt_per_layer;
    const int64_t i = (tile - l * mt_per_layer) * kTileM + row;  // row of the layer's weight
    const int k0 = g * 8;
    int j = 0;
    while (j + 1 < n_terms && k0 >= terms[j].kofs + 2 * terms[j].kc) ++j;
    const SwitchTerm t = terms[j];
    const bool lo = k0 >= t.kofs + t.kc;
    const int kk = k0 - t.kofs - (lo ? t.kc : 0);
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float a = 0.f;
      if (i < d_in && kk + q < t.rank)
        a = bf16_lo(A_pool[(l * R + t.pool_row + kk + q) * d_in + i]);
      v[q] = t.coef * a;
    }
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t hi = pack_bf16x2(v[2 * q], v[2 * q + 1]);
      w[q] = lo ? pack_bf16x2(v[2 * q] - bf16_lo(hi), v[2 * q + 1] - bf16_hi(hi)) : hi;
    }
    uint8_t *dst = img + tile * img_bytes + (k0 / kAugBlock) * kAugBlockBytes + sw128_offset(row, k0 % kAugBlock);
    *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace lora
