// Fused base + adapter GEMM on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
//   Y_tile = X_tile · W_tile + Ũ_tile · B_tile
//
// The adapter term is an augmented-K contraction [X | s·U]·[W ; B_a]: the same
// TMEM accumulator receives the tile's adapter K slices (one per adapter present
// in the tile, each 2·r_a rounded up to 16: the hi and lo bf16 parts of s·U),
// issued before the d_in-long base K loop so that their scattered B_pool loads
// overlap it, so the expand and the add happen in-tile and no intermediate Y
// goes back to HBM. This is the "split at the GEMM boundary, consume the intermediate in
// place" point of the kernel-layer section (Kernel 层：图分裂融合) of
// "LoRAFusion：消除冗余内存访问的多 LoRA 高效微调系统", applied to the
// multi-adapter batch of the batching section (批处理) of "S-LoRA：一个GPU运行
// 数千大模型成为可能" without padding adapters to a common rank.
//
// Structure: persistent CTAs (one per SM), 8 warps:
//   warp 0      TMA producer (lane 0): a 128-row box of X (original rows when a
//               tile's tokens are consecutive, else the sorted copy of X the
//               shrink wrote while gathering), then the tile's s·U images (bulk
//               copy) and the matching B_pool rows
//   warp 6      TMA producer (lane 0) of the W tiles of the base K blocks. With
//               every SM loading, one thread's copies complete one after another
//               (a few hundred ns each, nearly independent of their size), so
//               two issuing threads double the rate at which stages fill
//   warp 7      fix-up (with a plan): releases each landed stage to the MMA
//               thread, after zeroing the B_pool rows of an adapter block that
//               belong to another adapter (rows past the adapter's rank)
//   warp 1      MMA issuer (one thread) + TMEM owner: 128x256 fp32 accumulator,
//               double-buffered in TMEM (512 columns) so the epilogue of tile i
//               overlaps the main loop of tile i+1
//   warps 2..5  epilogue: TMEM -> registers -> bf16 -> global rows in the
//               original token order; in backward mode also adds the dropout-
//               masked adapter term D ⊙ (dU·A^T); in merge mode adds the
//               accumulator to the weights in place
// Every wait is bounded (mbar_wait); on a timeout the CTA flags the status
// word, stops issuing work and still frees its TMEM.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "skinny.cuh"

namespace lora {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kGemmStages = 4;
constexpr int kStageA = kBM * kBK * 2;            // 16 KB
constexpr int kStageB = kBN * kBK * 2;            // 32 KB
constexpr int kStageBytes = kStageA + kStageB;    // 48 KB
// An adapter block's B operand: up to four 8 KB slots, each one 16-row slice of
// B_pool over the tile's 256 columns, stored [4 column blocks][16 rows][64 cols].
constexpr int kBSlot = 4 * 16 * 128;
constexpr int kGemmThreads = 256;
constexpr int kGemmWarpW = 6;  // the W-copy warp
constexpr int kGemmWarpFix = 7;  // the warp that clears B rows of other adapters
// merge mode: after its adapter blocks each tile's block sequence has two W
// blocks, the tile's current weights (128 rows x 128 columns each, in the B part
// of a stage), which the epilogue consumes and releases
constexpr int kMergeWBlocks = 2;
constexpr int kGemmBarBytes = 256;
constexpr int kGemmSmem = 1024 + kGemmStages * kStageBytes + kGemmBarBytes + kBM * 16;

// kEpiStore: out = accumulator. kEpiBwdLora: single-adapter backward, out =
// accumulator + D ⊙ (dU·A^T) on CUDA cores. kEpiMergeAdd: out += accumulator (in
// place). kEpiBwdMulti: multi-adapter backward with dropout, out = base
// accumulator + D ⊙ adapter accumulator (the adapter K blocks go to a second
// accumulator at TMEM columns 256..511; one accumulator pair, no double buffer).
enum GemmEpi { kEpiStore = 0, kEpiBwdLora = 1, kEpiMergeAdd = 2, kEpiBwdMulti = 3 };
constexpr int kEpiRankRegs = 16;  // dU values per row kept in registers by the backward epilogue
// backward epilogue: the tile's slice of A (ranks < kEpiRankRegs, 256 columns) as
// fp32 in shared memory, behind the adapter tables
constexpr int kEpiAsBytes = kEpiRankRegs * kBN * 4;  // 16 KB
constexpr int kGemmSmemBwd = kGemmSmem + kEpiAsBytes;

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
  int32_t a_sorted;     // 1: A rows are stored in the plan's sorted order (row td.row0 of the
                        // A tensor map), as written by the shrink; 0: tiles are consecutive originals
  __nv_bfloat16 *out;   // [T, N]
  // backward epilogue: out += keep(t, col) / (1 - p) * sum_k dU[t, k] * A[k, col]
  const float *dU;      // [T, du_stride] (ranks past r are zero)
  const uint16_t *A;    // [r, N]
  int32_t r;
  int32_t du_stride;
  uint64_t seed, thr;
  float inv_keep;
  const uint32_t *keep_bits;  // precomputed keep bits (null: hash), word t * wpr + col / 32
  int64_t wpr;
  const int32_t *mt_order;  // m-tile visiting order (heaviest adapter work first), or null
  const AugBlockDesc *augblocks;  // the plan's adapter K blocks (TileDesc::aug0 + block)
  int32_t group_m;          // m-tiles per group of the tile visiting order (>= 1)
  int32_t w3d;              // 1 (MN-major B only): mapB is the 3-D view {64, K, N/64} of W
                            // (N % 64 == 0), one copy per K block; 0: 2-D {64, 64}, four copies
  int32_t b3d;              // 1: mapBl is the 3-D view {64, rows, N/64} (N % 64 == 0) and one
                            // copy fills a B slot; 0: mapBl is 2-D {64, 16}, four copies per slot
  // K split: 1 = persistent CTAs over all tiles; S > 1 = one tile per cluster of
  // S CTAs, CTA q takes base K blocks [q*KB/S, (q+1)*KB/S) and adapter blocks
  // q, q+S, ...; partial accumulators are exchanged (through the L2 workspace
  // xws when given, else distributed shared memory) and CTA q sums and stores
  // output columns [q*256/S, (q+1)*256/S).
  int32_t ksplit;
  // persistent mode: CTA b runs tiles sched_tiles[sched_off[b] .. sched_off[b+1])
  // (indices in the visiting order); null: round robin
  const int32_t *sched_off;
  const int32_t *sched_tiles;
  // split-K exchange through L2: slot (tile, src, owner) at
  // xws + ((tile * S + src) * S + owner) * xslot_bytes(S); null: through
  // distributed shared memory
  uint8_t *xws;
  // merge mode (merge_kaug > 0, EPI kEpiMergeAdd, K = 0): a stack of layers'
  // weights, out = [layers * merge_rows, N], updated in place by the adapter
  // blocks alone. m-tile mt is row block mt % mt_per_layer of layer
  // mt / mt_per_layer; every tile has merge_kaug augmented columns whose images
  // sit merge_img_bytes apart in uimg, and the same adapter blocks (augblocks
  // 0..), whose B rows are offset by the layer's layer_brows rows.
  int32_t merge_kaug;
  int32_t mt_per_layer;
  int32_t merge_rows;
  int32_t layer_brows;
  int64_t merge_img_bytes;
  // fused forward (the FUSED instance): the same launch first copies X's rows
  // into the sorted copy (when a_sorted; then waits for every CTA's share),
  // then runs its shrink units, each counting itself done for its m-tile, then
  // the GEMM tiles with their adapter blocks last, each tile's first adapter
  // block waiting for the tile's count
  int32_t gemm_ctas;            // CTAs that run GEMM tiles (0: all); the fused launch's others only run units
  const int32_t *fz_unit_off;   // [grid + 1]: CTA b runs units fz_units[fz_unit_off[b] ..)
  const int32_t *fz_units;      // indices into fz_sp.units
  const int32_t *fz_tile_need;  // [n_mt]: units per m-tile
  int32_t *fz_tile_cnt;         // [n_mt]: units done per m-tile (zero at launch)
  int32_t *fz_grid_cnt;         // CTAs done with the row copy (zero at launch)
  const uint16_t *fz_X;         // X in the original token order
  uint16_t *fz_Xs;              // the plan's sorted copy of X
  ShrinkParams fz_sp;           // the shrink's parameters (one CTA per unit)
};

// Split-K exchange, inside the idle stage ring once every MMA of the cluster is
// done. Each CTA q owns output columns [q*w, (q+1)*w), w = 256/S. Partials move
// as 4 KB blocks (32 rows x 32 columns fp32, one epilogue warp's TMEM lanes),
// staged per owner and moved whole: by bulk shared-to-shared copies that
// complete on the owner's receive barrier, or through a global workspace (bulk
// store by the sender, bulk load by the owner into the same receive slot, with a
// cluster barrier between). Inside a block, row r's 16-byte column group j sits at group
// j ^ (r & 7), so both the row-per-thread writes and reads are conflict-free.
//   [0, (S-1)*w*512)  receive slots, one per other rank (rank order, own skipped),
//                     each [w/32 column blocks][4 warps][4 KB]
//   then              outgoing blocks: per warp (256-w)/32 blocks of 4 KB
constexpr int kXBlock = 32 * 32 * 4;
__host__ __device__ constexpr int xslot_bytes(int S) { return (kBN / S) * kBM * 4; }
__host__ __device__ constexpr int xstage_bytes(int S) { return 4 * ((kBN - kBN / S) / 32) * kXBlock; }
static_assert((2 - 1) * xslot_bytes(2) + xstage_bytes(2) <= kGemmStages * kStageBytes,
              "split-K exchange (S = 2) must fit the stage ring");
static_assert((4 - 1) * xslot_bytes(4) + xstage_bytes(4) <= kGemmStages * kStageBytes,
              "split-K exchange (S = 4) must fit the stage ring");
__host__ __device__ constexpr uint32_t xswz(int row, int j) { return static_cast<uint32_t>(row * 128 + ((j ^ (row & 7)) * 16)); }

// The K blocks one CTA contributes to one tile.
struct BlockRange {
  int kb_lo, nbase;  // base blocks kb_lo .. kb_lo + nbase - 1
  int q, S, nlb;     // adapter blocks q, q + S, ... < nlb
  bool alast;        // adapter blocks after the base blocks (fused forward)
  __device__ __forceinline__ int naug() const { return q < nlb ? (nlb - q + S - 1) / S : 0; }
  __device__ __forceinline__ int count() const { return nbase + naug(); }
  // index into the tile's block sequence: < KB base, >= KB adapter block (blk - KB).
  // Adapter blocks come first: their scattered B-row loads then overlap the base
  // K loop instead of draining the pipeline at the end of the tile. In the fused
  // forward they come last, when the shrink that writes their images is done.
  __device__ __forceinline__ int block(int i, int KB) const {
    if (alast) return i < nbase ? kb_lo + i : KB + q + (i - nbase) * S;
    const int na = naug();
    return i < na ? KB + q + i * S : kb_lo + (i - na);
  }
  // position of block i among the CTA's adapter blocks (i must be one)
  __device__ __forceinline__ int aug_index(int i) const { return alast ? i - nbase : i; }
};

__device__ __forceinline__ BlockRange block_range(int KB, int nlb, int q, int S, bool alast = false) {
  BlockRange br;
  br.kb_lo = KB * q / S;
  br.nbase = KB * (q + 1) / S - br.kb_lo;
  br.q = q;
  br.S = S;
  br.nlb = nlb;
  br.alast = alast;
  return br;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
  return ra;
}

// Output tile visiting order: tiles come in groups of group_m m-tiles; inside a
// group the m index runs fastest. The CTAs that run at the same time then share
// a few row blocks of A and a few column blocks of B through L2, and a group's A
// rows stay in L2 while its n-tiles are swept (A read from DRAM about once, B
// about n_mt / group_m times). The m-tile index goes through mt_order when the
// plan has one.
__host__ __device__ inline void tile_mn(int tile, int n_mt, int n_nt, int G, int &mi, int &nt) {
  const int per_group = G * n_nt;
  const int g = tile / per_group;
  const int r = tile - g * per_group;
  const int m0 = g * G;
  const int gm = G < n_mt - m0 ? G : n_mt - m0;
  mi = m0 + r % gm;
  nt = r / gm;
}
__device__ __forceinline__ void tile_coords(int tile, const GemmParams &p, int &mt, int &nt) {
  int mi;
  tile_mn(tile, p.n_mt, p.n_nt, p.group_m, mi, nt);
  mt = p.mt_order ? p.mt_order[mi] : mi;
}

// The k-th tile (in the visiting order above) of this CTA in persistent mode:
// the plan's schedule lists each CTA's tiles when it has one (tiles of unequal
// adapter work spread over the CTAs by estimated cost), else the CTA takes
// tiles blockIdx.x, blockIdx.x + gridDim.x, ...
__device__ __forceinline__ bool cta_tile(const GemmParams &p, int k, int tile0, int tile_step, int n_tiles,
                                         int &tile) {
  if (tile0 >= n_tiles) return false;  // a CTA without tiles
  if (p.sched_off) {
    const int i = p.sched_off[blockIdx.x] + k;
    if (i >= p.sched_off[blockIdx.x + 1]) return false;
    tile = p.sched_tiles[i];
    return true;
  }
  tile = tile0 + k * tile_step;
  return tile < n_tiles;
}

// Barrier 1 over the 4 epilogue warps (128 threads). The OR form returns, to every
// participant, whether any of them passed true: the warps then leave the tile
// loop together, so none is left waiting at the next barrier.
__device__ __forceinline__ bool epi_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// m-tile mt of the merge mode: rows of one layer, all tiles alike
__device__ __forceinline__ TileDesc merge_tile(const GemmParams &p, int mt) {
  const int l = mt / p.mt_per_layer;
  const int ml = mt - l * p.mt_per_layer;
  TileDesc td;
  td.row0 = l * p.merge_rows + ml * kBM;
  td.rows = min(kBM, p.merge_rows - ml * kBM);
  td.chunk0 = 0;
  td.nchunk = 0;
  td.kaug = p.merge_kaug;
  td.contig = td.row0;
  td.uofs = static_cast<int64_t>(mt) * p.merge_img_bytes;
  td.aug0 = 0;
  return td;
}

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
// FUSED: the fused forward (GemmParams fz_*; the shrink's maps in mapS*).
template <bool B_KMAJOR, int EPI, bool FUSED = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    lora_gemm_kernel(const __grid_constant__ CUtensorMap mapA,    // A rows (X, sorted X or dY), box {64, 128}
                     const __grid_constant__ CUtensorMap mapB,    // W (2-D or 3-D, see GemmParams::w3d)
                     const __grid_constant__ CUtensorMap mapBl,   // B_pool rows, box {64, 16(, 4)}
                     const __grid_constant__ CUtensorMap mapSIn,    // fused: the shrink's X rows, box {64, 16}
                     const __grid_constant__ CUtensorMap mapSF,     // fused: A_pool rows, box {64, 16}
                     const __grid_constant__ CUtensorMap mapSBits,  // fused: keep bits, box {4, 16}
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
  // per stage: the B slot each K step of an adapter block reads (2 bits per step)
  volatile uint32_t *bmap = tmem_slot + 2;
  const uint32_t recv_bar = full0 + 128;  // split-K: the other ranks' partials have landed
  // per stage: the adapter block's slot count and each slot's rows that belong to
  // its adapter (AugBlockDesc::valid | nslot << 20), for the fix-up warp
  volatile uint32_t *bvalid = reinterpret_cast<volatile uint32_t *>(bars) + 34;
  // per stage: released by the fix-up warp once the stage is ready for the MMAs
  const uint32_t fixed0 = full0 + 152;

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
    mbar_init(recv_bar, 1);
    for (int s = 0; s < kGemmStages; ++s) mbar_init(fixed0 + 8 * s, 1);
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
  // inputs written by the previous kernels of the forward (s·U images, the
  // sorted copy of X) and the output are touched only after they completed;
  // the W copies read only the weights and the plan's tables (written before
  // those kernels ran), so their warp starts streaming at once
  if (warp != kGemmWarpW) pdl_wait();

  if constexpr (FUSED) {
    // ---------------------------------------------------- fused forward, phase 0:
    // X's rows into the plan's sorted copy (every CTA a share), then every CTA
    // waits until all shares are written (the launch is cooperative: all CTAs
    // are resident, so the wait ends)
    if (p.a_sorted) {
      // one warp per row: the row's source index is read once, and each lane
      // has up to 8 16-byte loads in flight before its stores
      const int per_row = p.K / 8;
      const int nwarps = static_cast<int>(gridDim.x) * (kGemmThreads / 32);
      for (int i = static_cast<int>(blockIdx.x) * (kGemmThreads / 32) + warp; i < p.T; i += nwarps) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.fz_X + static_cast<int64_t>(__ldg(p.perm + i)) * p.K);
        uint4 *dst = reinterpret_cast<uint4 *>(p.fz_Xs + static_cast<int64_t>(i) * p.K);
        for (int c0 = 0; c0 < per_row; c0 += 8 * 32) {
          uint4 v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int c = c0 + u * 32 + lane;
            if (c < per_row) v[u] = __ldg(src + c);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int c = c0 + u * 32 + lane;
            if (c < per_row) dst[c] = v[u];
          }
        }
      }
      fence_proxy_async_global();  // other CTAs read the copy through TMA
      __syncthreads();
      if (threadIdx.x == 0) {
        signal_counter(p.fz_grid_cnt);
        if (!wait_counter(p.fz_grid_cnt, static_cast<int>(gridDim.x))) *abort_flag = 1;
      }
      __syncthreads();
      fence_proxy_async_global();  // the copies (async proxy) read what the stores wrote
    }
    // phase 1: this CTA's shrink units, by warps 2..5 (consumers) and 7
    // (producer) in the stage ring's memory; each unit then counts itself done
    // for its m-tile (release), which the tile's adapter blocks wait for
    const int lt = (warp >= 2 && warp <= 5) ? static_cast<int>(threadIdx.x) - 64 : (warp == kGemmWarpFix ? 128 + lane : -1);
    if (lt >= 0 && !*abort_flag) {
      // the unit's ring takes the whole stage ring of the GEMM (a deeper ring
      // than the standalone shrink's: the units run beside other CTAs' GEMM
      // tiles, whose HBM traffic lengthens every copy's round trip)
      constexpr int kPool = kGemmStages * kStageBytes - 4096;
      uint64_t *sbars = reinterpret_cast<uint64_t *>(smem + kPool);
      for (int j = p.fz_unit_off[blockIdx.x]; j < p.fz_unit_off[blockIdx.x + 1]; ++j) {
        const int u = p.fz_units[j];
        if (!shrink_unit<4, kPool>(smem, sbars, mapSIn, mapSF, mapSBits, p.fz_sp, u, 0u, ShrinkRole{lt, 2, false})) {
          if (lt == 0) *abort_flag = 1;  // a wait gave up (all 160 threads see it and leave together)
          break;
        }
        fence_proxy_async_global();  // the image is read by other CTAs' bulk copies
        shrink_bar_all(2);  // the unit's outputs are all written
        if (lt == 0) signal_counter(p.fz_tile_cnt + p.fz_sp.units[u].tile);
      }
    }
    fence_proxy_async_smem();  // the shrink's generic stores precede the ring's TMA writes
    __syncthreads();           // the stage ring is free again
  }

  const int n_tiles = p.n_mt * p.n_nt;
  const int KB = (p.K + kBK - 1) / kBK;
  const bool merge = p.merge_kaug > 0;
  const bool has_plan = p.tiles != nullptr || merge;
  // the tile table of the plan, the merge mode's layer geometry, or plain row blocks
  auto tile_desc = [&](int mt) -> TileDesc {
    return merge ? merge_tile(p, mt) : (p.tiles ? p.tiles[mt] : regular_tile(mt, p.T));
  };
  const bool split = p.ksplit > 1;
  const int S = split ? p.ksplit : 1;
  const int q = split ? static_cast<int>(cluster_rank()) : 0;
  // CTAs past gemm_ctas (the fused forward's unit-only CTAs) have no tiles
  const int gctas = p.gemm_ctas > 0 ? p.gemm_ctas : static_cast<int>(gridDim.x);
  const int tile0 = static_cast<int>(blockIdx.x) >= gctas ? n_tiles
                    : split                                ? static_cast<int>(blockIdx.x) / S
                                                           : static_cast<int>(blockIdx.x);
  const int tile_step = split ? n_tiles : gctas;
  // split-K tail inputs, set by the epilogue warps before their wait
  int split_rows = 0, split_nt = 0, split_kaug = 0;
  int64_t split_orig = 0;

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&mapA);
      if (has_plan) prefetch_tmap(&mapBl);
    }
    // The warp stages each tile's adapter table in shared memory (no dependent
    // global loads inside the K loop); lane 0 issues every TMA copy.
    int stage = 0;
    uint32_t phase = 0;
    int tile;
    for (int k = 0; !*abort_flag && cta_tile(p, k, tile0, tile_step, n_tiles, tile); ++k) {
      int mt, nt;
      tile_coords(tile, p, mt, nt);
      const TileDesc td = tile_desc(mt);
      const int n0 = nt * kBN;
      // merge mode: this tile's layer's rows of B_pool
      const int brow_ofs = merge ? (mt / p.mt_per_layer) * p.layer_brows : 0;
      // A rows: the sorted copy written by the shrink (rows in tile order), or the
      // original rows when the tile's tokens are consecutive originals
      const int arow = p.a_sorted ? td.row0 : td.contig;
      if (lane == 0) {
        if (arow < 0) { flag_status(LORA_DEV_BOUNDS); *abort_flag = 1; }
        const BlockRange br = block_range(KB, (td.kaug + kAugBlock - 1) / kAugBlock, q, S, FUSED);
        const int nmma = br.count();
        const int nblk = arow < 0 ? 0 : nmma + (merge ? kMergeWBlocks : 0);
        // adapter block descriptors, one load ahead of their use (the adapter
        // blocks come first: block i < naug is adapter block q + i * S)
        const int na = br.naug();
        int4 nprow = make_int4(0, 0, 0, 0);
        int ninfo = 0, nvalid = 0;
        if (na > 0) {
          nprow = __ldg(reinterpret_cast<const int4 *>(p.augblocks + td.aug0 + q));
          ninfo = __ldg(&p.augblocks[td.aug0 + q].info);
          nvalid = __ldg(&p.augblocks[td.aug0 + q].valid);
        }
        for (int i = 0; i < nblk; ++i) {
          const int blk = i < nmma ? br.block(i, KB) : -1;
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { *abort_flag = 1; break; }
          const uint32_t a_dst = stage0 + stage * kStageBytes;
          const uint32_t b_dst = a_dst + kStageA;
          const uint32_t fb = full0 + 8 * stage;
          if (blk < 0) {
            // merge mode: W block i - nmma, the tile's weights in columns
            // [n0 + 128h, n0 + 128h + 128) as two 64-column boxes of 128 rows
            const int h = i - nmma;
            mbar_arrive_expect_tx(fb, kStageB);
            tma_load_2d(b_dst, &mapA, fb, n0 + 128 * h, td.contig);
            tma_load_2d(b_dst + kStageB / 2, &mapA, fb, n0 + 128 * h + 64, td.contig);
          } else if (blk < KB) {
            // the W tile of this stage comes from warp kGemmWarpW's copy; the
            // expected bytes cover both (a copy may land before this arrive:
            // the phase cannot complete while the arrival is pending)
            mbar_arrive_expect_tx(fb, kStageA + kStageB);
            tma_load_2d(a_dst, &mapA, fb, blk * kBK, arow);
          } else {
            // adapter K block: 64 augmented columns (up to 4 MMA K steps). Each
            // chunk spans 2*kc columns: s*U rounded to bf16 (hi), then the
            // rounding remainder (lo); both multiply the same B rows, so each
            // distinct 16-row slice of B_pool is copied once, into its own slot
            // (the planner's descriptor lists the slices and each step's slot).
            const int lb = blk - KB;
            const int ai = br.aug_index(i);
            if (FUSED && ai == 0) {
              // the tile's shrink units are done (their images written) before
              // the first of its images is copied
              if (!wait_counter(p.fz_tile_cnt + mt, p.fz_tile_need[mt])) { *abort_flag = 1; break; }
              fence_proxy_async_global();
            }
            const int prow_s[4] = {nprow.x + brow_ofs, nprow.y + brow_ofs, nprow.z + brow_ofs, nprow.w + brow_ofs};
            const int nslot = ninfo & 15;
            const uint32_t map = static_cast<uint32_t>(ninfo >> 4) & 0xFFu;
            bvalid[stage] = static_cast<uint32_t>(nvalid) | (static_cast<uint32_t>(nslot) << 20);
            if (ai + 1 < na) {
              nprow = __ldg(reinterpret_cast<const int4 *>(p.augblocks + td.aug0 + lb + S));
              ninfo = __ldg(&p.augblocks[td.aug0 + lb + S].info);
              nvalid = __ldg(&p.augblocks[td.aug0 + lb + S].valid);
            }
            bmap[stage] = map;  // published to the MMA warp by the release arrive below
            mbar_arrive_expect_tx(fb, kStageA + nslot * kBSlot);
            bulk_g2s(a_dst, p.uimg + td.uofs + static_cast<int64_t>(lb) * kAugBlockBytes, kAugBlockBytes,
                     fb);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (u < nslot) {
                if (p.b3d) {
                  tma_load_3d(b_dst + u * kBSlot, &mapBl, fb, 0, prow_s[u], n0 / 64);
                } else {
                  for (int j = 0; j < kBN / 64; ++j)
                    tma_load_2d(b_dst + u * kBSlot + j * 2048, &mapBl, fb, n0 + j * 64, prow_s[u]);
                }
              }
            }
          }
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
      }
      __syncwarp();
    }
  } else if (warp == kGemmWarpW) {
    // ------------------------------------------------------------ W producer
    // Walks the same block sequence as warp 0 and fills the B half of each base
    // block's stage once the stage is free. It waits for every stage in turn,
    // adapter blocks' too: a parity wait is only exact while the waiter is at
    // most one phase ahead of the barrier.
    if (lane == 0) {
      prefetch_tmap(&mapB);
      int stage = 0;
      uint32_t phase = 0;
      int tile;
      for (int k = 0; !*abort_flag && cta_tile(p, k, tile0, tile_step, n_tiles, tile); ++k) {
        int mt, nt;
        tile_coords(tile, p, mt, nt);
        const TileDesc td = tile_desc(mt);
        const int n0 = nt * kBN;
        const int arow = p.a_sorted ? td.row0 : td.contig;
        const BlockRange br = block_range(KB, (td.kaug + kAugBlock - 1) / kAugBlock, q, S, FUSED);
        const int nmma = br.count();
        const int nblk = arow < 0 ? 0 : nmma + (merge ? kMergeWBlocks : 0);
        for (int i = 0; i < nblk; ++i) {
          const int blk = i < nmma ? br.block(i, KB) : KB;  // merge W blocks: nothing to copy here
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { *abort_flag = 1; break; }
          if (blk < KB) {
            const uint32_t b_dst = stage0 + stage * kStageBytes + kStageA;
            const uint32_t fb = full0 + 8 * stage;
            const int k0 = blk * kBK;
            if (B_KMAJOR) {
              tma_load_2d(b_dst, &mapB, fb, k0, n0);
            } else if (p.w3d) {
              tma_load_3d(b_dst, &mapB, fb, 0, k0, n0 / 64);  // the four 64-column blocks in one copy
            } else {
              for (int j = 0; j < kBN / 64; ++j) tma_load_2d(b_dst + j * 8192, &mapB, fb, n0 + j * 64, k0);
            }
          }
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (warp == kGemmWarpFix) {
    // ------------------------------------------------------------- fix-up warp
    // With a plan, every stage reaches the MMA thread through this warp: it waits
    // for the stage's copies and releases the stage's `fixed` barrier. For an
    // adapter block whose 16-row B slices run past the adapter's rank (the rows
    // after it are the next adapter's), it first zeroes those rows, so a token
    // never multiplies factor values of an adapter absent from its tile. Being a
    // warp of its own, the zeroing overlaps the MMAs of the blocks before; and
    // since the MMA thread waits on every stage's release, this warp is never more
    // than one phase behind a barrier, which keeps its parity waits exact.
    if (has_plan) {
      int stage = 0;
      uint32_t phase = 0;
      int tile;
      for (int k = 0;; ++k) {
        const bool go = !*abort_flag && cta_tile(p, k, tile0, tile_step, n_tiles, tile);
        if (!__shfl_sync(0xFFFFFFFFu, go ? 1 : 0, 0)) break;
        int mt, nt;
        tile_coords(tile, p, mt, nt);
        const TileDesc td = tile_desc(mt);
        const int arow = p.a_sorted ? td.row0 : td.contig;
        const BlockRange br = block_range(KB, (td.kaug + kAugBlock - 1) / kAugBlock, q, S, FUSED);
        const int nmma = br.count();
        const int nblk = arow < 0 ? 0 : nmma + (merge ? kMergeWBlocks : 0);
        bool ok = true;
        for (int i = 0; i < nblk; ++i) {
          const int blk = i < nmma ? br.block(i, KB) : -1;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(full0 + 8 * stage, phase))) {
            if (lane == 0) *abort_flag = 1;
            ok = false;
            break;
          }
          if (blk >= KB) {
            const uint32_t vw = bvalid[stage];
            const int nsl = static_cast<int>(vw >> 20);
            uint8_t *bsp = smem + stage * kStageBytes + kStageA;
            bool zeroed = false;
            for (int u = 0; u < nsl; ++u) {
              const int v = static_cast<int>((vw >> (5 * u)) & 31u);
              // rows v .. 15 of the slot in each of its 4 column blocks, as
              // 16-byte pieces (8 per 128-byte row)
              for (int e = lane; e < (16 - v) * 32; e += 32) {
                const int r = v + (e >> 5);
                const int j = (e >> 3) & 3;
                *reinterpret_cast<uint4 *>(bsp + u * kBSlot + j * 2048 + r * 128 + (e & 7) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
              }
              zeroed |= v < 16;
            }
            if (zeroed) fence_proxy_async_smem();  // the MMA reads through the async proxy
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(fixed0 + 8 * stage);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t kIdesc = idesc_bf16(kBM, kBN, false, !B_KMAJOR);
      constexpr uint32_t kIdescAug = idesc_bf16(kBM, kBN, false, true);  // adapter B slots are MN-major
      constexpr bool kDual = EPI == kEpiBwdMulti;
      // stage 0's descriptors: A K-major (SW128, 8-row groups 1 KB apart, a K16
      // step 32 bytes on); B K-major likewise, or MN-major with 64-column blocks
      // 8 KB apart and a K16 step 16 rows (2 KB) on
      const uint64_t adesc0 = sdesc_sw128(stage0, 16, 1024);
      const uint64_t bdesc0 = B_KMAJOR ? sdesc_sw128(stage0 + kStageA, 16, 1024)
                                       : sdesc_sw128(stage0 + kStageA, 8192, 1024);
      constexpr uint64_t kAStep = 32 >> 4;
      constexpr uint64_t kBStep = B_KMAJOR ? (32 >> 4) : (2048 >> 4);
      // with a plan a stage is ready once the fix-up warp has released it
      const uint32_t ready0 = has_plan ? fixed0 : full0;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      int tile;
      for (int k = 0; !*abort_flag && cta_tile(p, k, tile0, tile_step, n_tiles, tile); ++k) {
        int mt, nt;
        tile_coords(tile, p, mt, nt);
        const int kaug = merge ? p.merge_kaug : (p.tiles ? p.tiles[mt].kaug : 0);
        const BlockRange br = block_range(KB, (kaug + kAugBlock - 1) / kAugBlock, q, S, FUSED);
        const int nmma = br.count();
        const int nblk = nmma + (merge ? kMergeWBlocks : 0);
        if (!mbar_wait(acce0 + 8 * acc, aphase ^ 1)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        const uint32_t d_aug = kDual ? tmem_base + kBN : d_tmem;
        // the first base block starts the base accumulator (after the adapter
        // blocks when they have their own)
        const int first_base = kDual ? br.naug() : 0;
        bool ok = true;
        for (int i = 0; i < nblk; ++i) {
          if (i >= nmma) {
            // merge mode's W blocks: no MMA; the epilogue reads and releases them
            if (!mbar_wait(ready0 + 8 * stage, phase)) { *abort_flag = 1; ok = false; break; }
            if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
            continue;
          }
          const int blk = br.block(i, KB);
          if (!mbar_wait(ready0 + 8 * stage, phase)) { *abort_flag = 1; ok = false; break; }
          tc_fence_after();
          // One thread issues every MMA, so its instruction count per K block
          // bounds the tensor pipe: the descriptors of a stage are the stage's
          // base descriptors plus constants (address field in 16-byte units).
          const uint64_t ad = adesc0 + static_cast<uint64_t>(stage * (kStageBytes >> 4));
          const uint64_t bd = bdesc0 + static_cast<uint64_t>(stage * (kStageBytes >> 4));
          if (blk < KB) {
            umma_bf16(d_tmem, ad, bd, kIdesc, i > first_base ? 1u : 0u);
            umma_bf16_acc(d_tmem, ad + kAStep, bd + kBStep, kIdesc);
            umma_bf16_acc(d_tmem, ad + 2 * kAStep, bd + 2 * kBStep, kIdesc);
            umma_bf16_acc(d_tmem, ad + 3 * kAStep, bd + 3 * kBStep, kIdesc);
          } else {
            // adapter block (MN-major B slots [4 column blocks][16 rows][64 cols],
            // column-block stride 2 KB; the slot of each K step from bmap)
            const int steps = min(4, (kaug - (blk - KB) * kAugBlock) / 16);
            const uint32_t map = bmap[stage];
            const uint32_t b_s = stage0 + stage * kStageBytes + kStageA;
            for (int qq = 0; qq < steps; ++qq) {
              const uint64_t bq = sdesc_sw128(b_s + ((map >> (2 * qq)) & 3u) * kBSlot, 2048, 1024);
              umma_bf16(d_aug, ad + qq * kAStep, bq, kIdescAug, (i > 0 || qq > 0) ? 1u : 0u);
            }
          }
          umma_commit(empty0 + 8 * stage);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * acc);
        if (kDual) aphase ^= 1;  // one accumulator pair: buffer 0 every tile
        else if (++acc == 2) { acc = 0; aphase ^= 1; }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (warps 2..5)
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    float *as = reinterpret_cast<float *>(smem + kGemmStages * kStageBytes + kGemmBarBytes + kBM * 16);
    int acc = 0;
    uint32_t aphase = 0;
    int ep_stage = 0;  // merge mode: the epilogue's walk of the stage ring
    uint32_t ep_phase = 0;
    if (split) {
      // the split-K tail's table entry and output row, loaded while the K loop runs
      int mt = 0, nt = 0;
      tile_coords(tile0 < n_tiles ? tile0 : 0, p, mt, nt);
      const TileDesc td = tile_desc(mt);
      split_rows = td.rows;
      split_nt = nt;
      split_kaug = td.kaug;
      split_orig = row >= td.rows ? 0
                   : has_plan    ? (td.contig >= 0 ? td.contig + row : p.perm[td.row0 + row])
                                 : td.row0 + row;
    }
    // the backward's warps leave together (epi_bar_or), so its loop ignores the
    // flag here and tests it at the barrier
    int tile;
    for (int k = 0; (EPI == kEpiBwdLora || EPI == kEpiMergeAdd || !*abort_flag) &&
                    cta_tile(p, k, tile0, tile_step, n_tiles, tile);
         ++k) {
      int mt, nt;
      tile_coords(tile, p, mt, nt);
      const TileDesc td = tile_desc(mt);
      if constexpr (EPI == kEpiMergeAdd) {
        // W <- bf16(W + accumulator), in place. The tile's current weights come
        // through the stage ring as its two W blocks (after its adapter blocks):
        // walk the ring as the producer fills it, wait for each W block, add,
        // store, and release the stage.
        const int nmma = block_range(KB, (td.kaug + kAugBlock - 1) / kAugBlock, q, S, FUSED).count();
        for (int i = 0; i < nmma; ++i)
          if (++ep_stage == kGemmStages) { ep_stage = 0; ep_phase ^= 1; }
        const bool valid = row < td.rows;
        const int64_t orow = static_cast<int64_t>(td.contig) + row;
        // every wait is agreed by the four warps (bar.red.or), so that none
        // leaves while the others wait at the barrier below
        if (epi_bar_or(!mbar_wait(accf0 + 8 * acc, aphase) || *abort_flag)) { *abort_flag = 1; break; }
        tc_fence_after();
        bool ok = true;
        for (int h = 0; h < kMergeWBlocks; ++h) {
          if (epi_bar_or(!mbar_wait(full0 + 8 * ep_stage, ep_phase) || *abort_flag)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint8_t *wst = smem + ep_stage * kStageBytes + kStageA;  // [2 halves][128 rows][64 cols], SW128
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int c = 4 * h + cc;
            uint32_t v[32];
            tmem_ld32(tmem_base + ((quarter * 32) << 16) + acc * kBN + c * 32, v);
            tmem_wait_ld();
            const int col0 = nt * kBN + c * 32;
            if (valid && col0 < p.N) {
              const uint8_t *wrow = wst + (cc >> 1) * (kStageB / 2);
              uint4 *dst = reinterpret_cast<uint4 *>(p.out + orow * p.N + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (col0 + 8 * j < p.N) {
                  const uint4 w = *reinterpret_cast<const uint4 *>(wrow + sw128_offset(row, (cc & 1) * 32 + 8 * j));
                  const uint32_t *vv = v + 8 * j;
                  uint4 o;
                  o.x = pack_bf16x2(bf16_lo(w.x) + __uint_as_float(vv[0]), bf16_hi(w.x) + __uint_as_float(vv[1]));
                  o.y = pack_bf16x2(bf16_lo(w.y) + __uint_as_float(vv[2]), bf16_hi(w.y) + __uint_as_float(vv[3]));
                  o.z = pack_bf16x2(bf16_lo(w.z) + __uint_as_float(vv[4]), bf16_hi(w.z) + __uint_as_float(vv[5]));
                  o.w = pack_bf16x2(bf16_lo(w.w) + __uint_as_float(vv[6]), bf16_hi(w.w) + __uint_as_float(vv[7]));
                  dst[j] = o;
                }
              }
            }
          }
          epi_bar();  // every thread's reads of the W block are done
          if (threadIdx.x == 64) mbar_arrive(empty0 + 8 * ep_stage);
          if (++ep_stage == kGemmStages) { ep_stage = 0; ep_phase ^= 1; }
        }
        if (!ok) break;
        tc_fence_before();
        mbar_arrive(acce0 + 8 * acc);
        if (++acc == 2) { acc = 0; aphase ^= 1; }
        continue;
      }
      if constexpr (EPI == kEpiBwdMulti) {
        // dX = dY·W^T (TMEM columns of buffer 0) + keep / (1 - p) * sum over the
        // row's adapter of dU·A^T (columns 256..511)
        if (!mbar_wait(accf0, aphase)) { *abort_flag = 1; break; }
        tc_fence_after();
        const bool valid = row < td.rows;
        int64_t orig = 0;
        if (valid) orig = td.contig >= 0 ? td.contig + row : p.perm[td.row0 + row];
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32], w[32];
          tmem_ld32(tmem_base + ((quarter * 32) << 16) + c * 32, v);
          tmem_ld32(tmem_base + ((quarter * 32) << 16) + kBN + c * 32, w);
          tmem_wait_ld();
          const int col0 = nt * kBN + c * 32;
          if (valid && col0 < p.N) {
            const uint32_t keep = p.keep_bits ? __ldg(p.keep_bits + orig * p.wpr + (col0 >> 5))
                                              : keep_mask32(p.seed, p.thr, static_cast<uint64_t>(orig * p.N + col0));
            float f[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
              f[i] = __uint_as_float(v[i]) + (((keep >> i) & 1u) ? p.inv_keep * __uint_as_float(w[i]) : 0.f);
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
        mbar_arrive(acce0);
        aphase ^= 1;
        continue;
      }
      if (EPI == kEpiBwdLora) {
        // stage A[k][nt*256 .. +256) for k < min(r, 16) as fp32 (zero past r or N):
        // 8 threads per rank, 32 columns each
        const int et = static_cast<int>(threadIdx.x) - 64;
        const int k = et >> 3;
        const int cb = (et & 7) * 32;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = nt * kBN + cb + 8 * j;
          uint4 w = make_uint4(0, 0, 0, 0);
          if (k < p.r && col < p.N) w = __ldg(reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(k) * p.N + col));
          float4 *d4 = reinterpret_cast<float4 *>(as + k * kBN + cb + 8 * j);
          d4[0] = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
          d4[1] = make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
        }
        const bool waited = mbar_wait(accf0 + 8 * acc, aphase);
        if (epi_bar_or(!waited || *abort_flag)) { *abort_flag = 1; break; }
      } else {
        if (!mbar_wait(accf0 + 8 * acc, aphase)) { *abort_flag = 1; break; }
      }
      tc_fence_after();
      if (split) break;  // the cluster reduction below handles the single tile
      const bool valid = row < td.rows;
      int64_t orig = 0;
      if (valid) orig = has_plan ? (td.contig >= 0 ? td.contig + row : p.perm[td.row0 + row]) : td.row0 + row;
      float du[kEpiRankRegs];  // backward: this row's dU, loaded once per tile (ranks <= kEpiRankRegs)
      if (EPI == kEpiBwdLora) {
#pragma unroll
        for (int k = 0; k < kEpiRankRegs; ++k) du[k] = (valid && k < p.r) ? p.dU[orig * p.du_stride + k] : 0.f;
      }
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
            auto add_rank = [&](int k, float d) {
              const uint4 *arow = reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(k) * p.N + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (col0 + 8 * j < p.N) {
                  const uint4 w = __ldg(arow + j);  // same address across the warp: one broadcast
                  l[8 * j + 0] += d * bf16_lo(w.x);
                  l[8 * j + 1] += d * bf16_hi(w.x);
                  l[8 * j + 2] += d * bf16_lo(w.y);
                  l[8 * j + 3] += d * bf16_hi(w.y);
                  l[8 * j + 4] += d * bf16_lo(w.z);
                  l[8 * j + 5] += d * bf16_hi(w.z);
                  l[8 * j + 6] += d * bf16_lo(w.w);
                  l[8 * j + 7] += d * bf16_hi(w.w);
                }
              }
            };
#pragma unroll
            for (int k = 0; k < kEpiRankRegs; ++k) {
              if (k < p.r) {
                const float4 *ar = reinterpret_cast<const float4 *>(as + k * kBN + c * 32);  // broadcast reads
                const float d = du[k];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 a4 = ar[j];
                  l[4 * j + 0] += d * a4.x;
                  l[4 * j + 1] += d * a4.y;
                  l[4 * j + 2] += d * a4.z;
                  l[4 * j + 3] += d * a4.w;
                }
              }
            }
            for (int k = kEpiRankRegs; k < p.r; ++k) add_rank(k, p.dU[orig * p.du_stride + k]);
            const uint32_t keep = p.keep_bits ? __ldg(p.keep_bits + orig * p.wpr + (col0 >> 5))
                                              : keep_mask32(p.seed, p.thr, static_cast<uint64_t>(orig * p.N + col0));
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] += ((keep >> i) & 1u) ? p.inv_keep * l[i] : 0.f;
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
      if (EPI == kEpiBwdLora) epi_bar();  // every read of the A slice is done before it is replaced
    }
  }

  tc_fence_before();
  __syncthreads();
  if (split) {
    // --------------------------------------------------- split-K cluster reduction
    // The tile's table entry and the output rows are fetched before the barrier,
    // so their global latency overlaps the wait for the slowest peer.
    const int width = kBN / S;
    const uint32_t slot0 = smem_u32(smem);
    const uint32_t out0 = slot0 + (S - 1) * xslot_bytes(S);
    const int nt = split_nt;
    // a CTA with no K blocks for this tile contributes zeros (its TMEM was never written)
    const bool any = block_range(KB, (split_kaug + kAugBlock - 1) / kAugBlock, q, S).count() > 0;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool epi = warp >= 2 && warp < 6;
    const bool valid = epi && row < split_rows;
    const int64_t orig = valid ? split_orig : 0;
    // Two ways to move the partials. Through distributed shared memory: after a
    // cluster barrier (every CTA's MMAs are complete, so every stage ring is idle
    // and may receive; it also orders the receive barriers' initialisation before
    // any remote completion) each CTA copies its blocks into the owners' rings.
    // Through L2 (the plan's workspace): each CTA writes its blocks to global
    // memory, and after the cluster barrier each owner copies its blocks in; the
    // peers' rings are never written, and this measured faster.
    const bool via_l2 = p.xws != nullptr;
    if (!via_l2) {
      cluster_barrier();
      if (threadIdx.x == 64) mbar_arrive_expect_tx(recv_bar, (S - 1) * xslot_bytes(S));
    }
    bool go = false;
    if (epi) {
      go = tile0 < n_tiles && !*abort_flag;
      if (go) {
        // send, step 1: TMEM -> registers -> 4 KB blocks laid out per owner as the
        // owner's receive slot is ([column block][warp][32 rows x 32 fp32])
        tc_fence_after();
        for (int c = 0; c < kBN / 32; c += 2) {
          const int owner = (c * 32) / width;  // width >= 64: columns c, c + 1 share an owner
          if (owner == q) continue;
          const int oidx = owner < q ? owner : owner - 1;
          const int cc = (c * 32 - owner * width) / 32;
          uint32_t v0[32], v1[32];
          tmem_ld32(tmem_base + ((quarter * 32) << 16) + c * 32, v0);
          tmem_ld32(tmem_base + ((quarter * 32) << 16) + (c + 1) * 32, v1);
          tmem_wait_ld();
          uint8_t *b0 = smem + (out0 - slot0) + oidx * xslot_bytes(S) + (cc * 4 + quarter) * kXBlock;
          uint8_t *b1 = b0 + 4 * kXBlock;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            *reinterpret_cast<float4 *>(b0 + xswz(lane, j)) =
                any ? make_float4(__uint_as_float(v0[4 * j]), __uint_as_float(v0[4 * j + 1]),
                                  __uint_as_float(v0[4 * j + 2]), __uint_as_float(v0[4 * j + 3]))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(b1 + xswz(lane, j)) =
                any ? make_float4(__uint_as_float(v1[4 * j]), __uint_as_float(v1[4 * j + 1]),
                                  __uint_as_float(v1[4 * j + 2]), __uint_as_float(v1[4 * j + 3]))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        fence_proxy_async_smem();  // the bulk copies (async proxy) read what these stores wrote
      }
      // step 2: once all 4 warps have written, one thread sends each owner its
      // whole slot (width x 128 fp32) in one bulk copy; the reducing barrier
      // makes the warps agree on whether to go on
      go = !epi_bar_or(!go);
      if (go && threadIdx.x == 64) {
        for (int owner = 0; owner < S; ++owner) {
          if (owner == q) continue;
          const int oidx = owner < q ? owner : owner - 1;
          const uint32_t src = out0 + static_cast<uint32_t>(oidx * xslot_bytes(S));
          if (via_l2) {
            bulk_s2g(p.xws + (static_cast<int64_t>(tile0 * S + q) * S + owner) * xslot_bytes(S), src, xslot_bytes(S));
          } else {
            const int jq = q < owner ? q : q - 1;  // this rank's slot at the owner
            bulk_s2s_cluster(map_rank(slot0 + static_cast<uint32_t>(jq * xslot_bytes(S)), static_cast<uint32_t>(owner)),
                             src, xslot_bytes(S), map_rank(recv_bar, static_cast<uint32_t>(owner)));
          }
        }
        bulk_commit();
        if (via_l2) {
          bulk_wait_all();  // the partials are in global memory before the barrier releases them
          fence_proxy_async_global();
        }
      }
    }
    if (via_l2) {
      cluster_barrier();  // every rank's partials are written
      if (go && threadIdx.x == 64) {
        fence_proxy_async_global();
        mbar_arrive_expect_tx(recv_bar, (S - 1) * xslot_bytes(S));
        for (int src = 0; src < S; ++src) {
          if (src == q) continue;
          const int js = src < q ? src : src - 1;
          bulk_g2s(slot0 + static_cast<uint32_t>(js * xslot_bytes(S)),
                   p.xws + (static_cast<int64_t>(tile0 * S + src) * S + q) * xslot_bytes(S), xslot_bytes(S),
                   recv_bar);
        }
      }
    }
    if (epi) {
      // receive: own partial from TMEM + the other ranks' blocks in rank order
      // (a fixed order, so the result is deterministic)
      if (go) {
        if (!mbar_wait(recv_bar, 0)) {
          *abort_flag = 1;
        } else {
          for (int cc = 0; cc < width / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem_base + ((quarter * 32) << 16) + q * width + cc * 32, v);
            tmem_wait_ld();
            float s[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) s[e] = any ? __uint_as_float(v[e]) : 0.f;
            for (int src = 0; src < S; ++src) {
              if (src == q) continue;
              const int js = src < q ? src : src - 1;
              const uint8_t *bp = smem + js * xslot_bytes(S) + (cc * 4 + quarter) * kXBlock;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float4 t = *reinterpret_cast<const float4 *>(bp + xswz(lane, j));
                s[4 * j + 0] += t.x;
                s[4 * j + 1] += t.y;
                s[4 * j + 2] += t.z;
                s[4 * j + 3] += t.w;
              }
            }
            const int col = nt * kBN + q * width + cc * 32;
            if (valid) {
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                if (col + 8 * h < p.N) {
                  uint4 o;
                  o.x = pack_bf16x2(s[8 * h + 0], s[8 * h + 1]);
                  o.y = pack_bf16x2(s[8 * h + 2], s[8 * h + 3]);
                  o.z = pack_bf16x2(s[8 * h + 4], s[8 * h + 5]);
                  o.w = pack_bf16x2(s[8 * h + 6], s[8 * h + 7]);
                  *reinterpret_cast<uint4 *>(p.out + orig * p.N + col + 8 * h) = o;
                }
              }
            }
          }
        }
        if (threadIdx.x == 64) bulk_wait_read_all();  // the outgoing slots are read before this CTA can exit
      }
    }
    // every TMEM read is done before warp 1 frees it; every block bound for this
    // CTA has landed (the receive barrier) and every outgoing block has been read
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace lora
