// Fused base + adapter GEMM on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
//   Y_tile = X_tile · W_tile + Ũ_tile · B_tile
//
// The adapter term is an augmented-K contraction [X | s·U]·[W ; B_a]: after the
// d_in-long base K loop, the same TMEM accumulator receives the tile's adapter
// K slices (one per adapter present in the tile, each r_a rounded up to 16),
// so the expand and the add happen in-tile and no intermediate Y goes back to
// HBM. This is the "split at the GEMM boundary, consume the intermediate in
// place" point of the kernel-layer section (Kernel 层：图分裂融合) of
// "LoRAFusion：消除冗余内存访问的多 LoRA 高效微调系统", applied to the
// multi-adapter batch of the batching section (批处理) of "S-LoRA：一个GPU运行
// 数千大模型成为可能" without padding adapters to a common rank.
//
// Structure: persistent CTAs (one per SM), 6 warps:
//   warp 0      TMA producer (one thread): X rows (tile load, or gather4 by the
//               plan's permutation), W tile, then the tile's s·U images (bulk
//               copy) and the matching rows of B_pool (tile loads)
//   warp 1      MMA issuer (one thread) + TMEM owner: 128x256 fp32 accumulator,
//               double-buffered in TMEM (512 columns) so the epilogue of tile i
//               overlaps the main loop of tile i+1
//   warps 2..5  epilogue: TMEM -> registers -> bf16 -> global rows in the
//               original token order; in backward mode also adds the dropout-
//               masked adapter term D ⊙ (dU·A^T)
// Every wait is bounded (mbar_wait); on a timeout the CTA flags the status
// word, stops issuing work and still frees its TMEM.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace lora {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kGemmStages = 4;
constexpr int kStageA = kBM * kBK * 2;            // 16 KB
constexpr int kStageB = kBN * kBK * 2;            // 32 KB
constexpr int kStageBytes = kStageA + kStageB;    // 48 KB
constexpr int kGemmThreads = 192;
constexpr int kGemmBarBytes = 256;
constexpr int kGemmSmem = 1024 + kGemmStages * kStageBytes + kGemmBarBytes + kBM * 4;

enum GemmEpi { kEpiStore = 0, kEpiBwdLora = 1 };

struct GemmParams {
  int32_t T;       // rows (tokens)
  int32_t K;       // contraction length (d_in forward, d_out backward)
  int32_t N;       // output columns (d_out forward, d_in backward)
  int32_t n_mt, n_nt;
  // plan (null: tiles are consecutive original rows and there is no adapter term)
  const TileDesc *tiles;
  const ChunkDesc *chunks;
  const int32_t *perm;
  const uint8_t *uimg;  // s·U images, one 16 KB block per 64 augmented columns
  __nv_bfloat16 *out;   // [T, N]
  // backward epilogue: out += keep(t, col) / (1 - p) * sum_k dU[t, k] * A[k, col]
  const float *dU;      // [T, r]
  const uint16_t *A;    // [r, N]
  int32_t r;
  uint64_t seed, thr;
  float inv_keep;
};

__device__ __forceinline__ TileDesc regular_tile(int mt, int T) {
  TileDesc td;
  td.row0 = mt * kBM;
  td.rows = min(kBM, T - mt * kBM);
  td.chunk0 = 0;
  td.nchunk = 0;
  td.kaug = 0;
  td.contig = td.row0;
  td.uofs = 0;
  return td;
}

// B_KMAJOR: the B operand tile is K-major (backward: W^T); otherwise MN-major (W).
template <bool B_KMAJOR, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    lora_gemm_kernel(const __grid_constant__ CUtensorMap mapA,    // rows of X/dY, box {64, 128}
                     const __grid_constant__ CUtensorMap mapAg,   // rows of X, box {64, 1} (gather4)
                     const __grid_constant__ CUtensorMap mapB,    // W
                     const __grid_constant__ CUtensorMap mapBl,   // B_pool rows, box {64, 16}
                     const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t stage0 = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kGemmStages * kStageBytes);
  const uint32_t full0 = smem_u32(bars);                    // [kGemmStages]
  const uint32_t empty0 = full0 + 8 * kGemmStages;          // [kGemmStages]
  const uint32_t accf0 = empty0 + 8 * kGemmStages;          // [2]
  const uint32_t acce0 = accf0 + 16;                        // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kGemmStages + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int32_t *rowcache = reinterpret_cast<int32_t *>(smem + kGemmStages * kStageBytes + kGemmBarBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_tiles = p.n_mt * p.n_nt;
  const int KB = (p.K + kBK - 1) / kBK;
  const bool has_plan = p.tiles != nullptr;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        const int mt = tile % p.n_mt;
        const int nt = tile / p.n_mt;
        const TileDesc td = has_plan ? p.tiles[mt] : regular_tile(mt, p.T);
        const int n0 = nt * kBN;
        if (td.contig < 0) {
          for (int i = 0; i < kBM; ++i) {
            const int rr = i < td.rows ? i : td.rows - 1;  // pad rows repeat a valid row
            rowcache[i] = p.perm[td.row0 + rr];
          }
        }
        const int nlb = (td.kaug + kAugBlock - 1) / kAugBlock;
        for (int blk = 0; blk < KB + nlb; ++blk) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { *abort_flag = 1; break; }
          const uint32_t a_dst = stage0 + stage * kStageBytes;
          const uint32_t b_dst = a_dst + kStageA;
          const uint32_t fb = full0 + 8 * stage;
          if (blk < KB) {
            const int k0 = blk * kBK;
            mbar_arrive_expect_tx(fb, kStageA + kStageB);
            if (td.contig >= 0) {
              tma_load_2d(a_dst, &mapA, fb, k0, td.contig);
            } else {
              for (int g = 0; g < kBM / 4; ++g)
                tma_gather4(a_dst + g * 512, &mapAg, fb, k0, rowcache[4 * g], rowcache[4 * g + 1],
                            rowcache[4 * g + 2], rowcache[4 * g + 3]);
            }
            if (B_KMAJOR) {
              tma_load_2d(b_dst, &mapB, fb, k0, n0);
            } else {
              for (int j = 0; j < kBN / 64; ++j) tma_load_2d(b_dst + j * 8192, &mapB, fb, n0 + j * 64, k0);
            }
          } else {
            // adapter K block: 64 augmented columns (up to 4 MMA K steps)
            const int lb = blk - KB;
            const int steps = min(4, (td.kaug - lb * kAugBlock) / 16);
            mbar_arrive_expect_tx(fb, kStageA + steps * (kBN / 64) * 2048);
            bulk_g2s(a_dst, p.uimg + td.uofs + static_cast<int64_t>(lb) * kAugBlockBytes, kAugBlockBytes,
                     fb);
            int c = td.chunk0;
            for (int q = 0; q < steps; ++q) {
              const int kq = lb * kAugBlock + q * 16;
              while (c + 1 < td.chunk0 + td.nchunk && kq >= p.chunks[c].kofs + p.chunks[c].kc) ++c;
              const int prow = p.chunks[c].pool_row + (kq - p.chunks[c].kofs);
              for (int j = 0; j < kBN / 64; ++j)
                tma_load_2d(b_dst + j * 8192 + q * 2048, &mapBl, fb, n0 + j * 64, prow);
            }
          }
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t kIdesc = idesc_bf16(kBM, kBN, false, !B_KMAJOR);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        const int mt = tile % p.n_mt;
        const int kaug = has_plan ? p.tiles[mt].kaug : 0;
        const int nlb = (kaug + kAugBlock - 1) / kAugBlock;
        if (!mbar_wait(acce0 + 8 * acc, aphase ^ 1)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        bool ok = true;
        for (int blk = 0; blk < KB + nlb; ++blk) {
          if (!mbar_wait(full0 + 8 * stage, phase)) { *abort_flag = 1; ok = false; break; }
          tc_fence_after();
          const uint32_t a_s = stage0 + stage * kStageBytes;
          const uint32_t b_s = a_s + kStageA;
          const int steps = blk < KB ? 4 : min(4, (kaug - (blk - KB) * kAugBlock) / 16);
          for (int q = 0; q < steps; ++q) {
            const uint64_t ad = sdesc_sw128(a_s + q * 32, 16, 1024);
            const uint64_t bd = B_KMAJOR ? sdesc_sw128(b_s + q * 32, 16, 1024)
                                         : sdesc_sw128(b_s + q * 2048, 8192, 1024);
            umma_bf16(d_tmem, ad, bd, kIdesc, (blk > 0 || q > 0) ? 1u : 0u);
          }
          umma_commit(empty0 + 8 * stage);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * acc);
        if (++acc == 2) { acc = 0; aphase ^= 1; }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t aphase = 0;
    for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
      const int mt = tile % p.n_mt;
      const int nt = tile / p.n_mt;
      const TileDesc td = has_plan ? p.tiles[mt] : regular_tile(mt, p.T);
      if (!mbar_wait(accf0 + 8 * acc, aphase)) { *abort_flag = 1; break; }
      tc_fence_after();
      const bool valid = row < td.rows;
      int64_t orig = 0;
      if (valid) orig = has_plan ? (td.contig >= 0 ? td.contig + row : p.perm[td.row0 + row]) : td.row0 + row;
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem_base + ((quarter * 32) << 16) + acc * kBN + c * 32, v);
        tmem_wait_ld();
        const int col0 = nt * kBN + c * 32;
        if (valid && col0 < p.N) {
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          if (EPI == kEpiBwdLora) {
            float l[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) l[i] = 0.f;
            for (int k = 0; k < p.r; ++k) {
              const float du = p.dU[orig * p.r + k];
              const uint4 *arow = reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(k) * p.N + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (col0 + 8 * j < p.N) {
                  const uint4 w = __ldg(arow + j);
                  l[8 * j + 0] += du * bf16_lo(w.x);
                  l[8 * j + 1] += du * bf16_hi(w.x);
                  l[8 * j + 2] += du * bf16_lo(w.y);
                  l[8 * j + 3] += du * bf16_hi(w.y);
                  l[8 * j + 4] += du * bf16_lo(w.z);
                  l[8 * j + 5] += du * bf16_hi(w.z);
                  l[8 * j + 6] += du * bf16_lo(w.w);
                  l[8 * j + 7] += du * bf16_hi(w.w);
                }
              }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const bool keep = keep_elem(p.seed, p.thr, orig, col0 + i, p.N);
              f[i] += keep ? p.inv_keep * l[i] : 0.f;
            }
          }
          uint4 *dst = reinterpret_cast<uint4 *>(p.out + orig * p.N + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (col0 + 8 * j < p.N) {
              uint4 o;
              o.x = pack_bf16x2(f[8 * j + 0], f[8 * j + 1]);
              o.y = pack_bf16x2(f[8 * j + 2], f[8 * j + 3]);
              o.z = pack_bf16x2(f[8 * j + 4], f[8 * j + 5]);
              o.w = pack_bf16x2(f[8 * j + 6], f[8 * j + 7]);
              dst[j] = o;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acce0 + 8 * acc);
      if (++acc == 2) { acc = 0; aphase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace lora
