// Skinny contractions around the fused GEMM, all memory-bound: the rank
// dimension r_a is 1..256 against d_in, d_out in the thousands.
//
//  * lora_shrink_kernel: U[t, k] = sum_i In[t, i] * F[k, i] over the rows of one
//    adapter run (forward: In = X with the dropout mask, F = A_pool rows of the
//    adapter; backward: In = dY, F = B rows). Each X tile is read once through
//    TMA into shared memory; warp-level MMA (mma.sync m16n8k16, bf16 -> fp32)
//    works on the skinny rank dimension. The d_in contraction is split across
//    the CTAs of a thread-block cluster and summed through distributed shared
//    memory, so a small adapter run still spreads its bytes over several SMs.
//    Tokens of one adapter are consecutive rows either of X or of the sorted
//    copy of X that lora_gather_rows_kernel writes first.
//    Forward output: the tile's s·U block, already in the 128-byte-swizzled
//    shared-memory image the fused GEMM's MMA reads, plus U for the backward.
//  * lora_tcontract_kernel: partial[q][k][n] = sum_{t in split q} G[t, k] * In[t, n]
//    (dB with G = U, In = dY; dA with G = dU, In = masked X), fixed token splits.
//    G stays fp32 and enters the MMA as three bf16 parts (hi, mid, lo: three
//    MMAs), about 24 mantissa bits, so each term carries fp32 precision: sums
//    whose terms cancel (per-token terms of +-1e3 summing to 1e-3 occur in the
//    fleet fine-tuning batch) keep an error at fp32-accumulation level.
//  * lora_reduce_splits_kernel: sums the splits in a fixed order (deterministic).
//  * lora_mask_kernel: the dropout mask itself (test hook).
//
// Where the LoRA shrink sits in the layer: the X·A product of the LoRA branch
// next to the frozen base GEMM, "LoRAFusion：消除冗余内存访问的多 LoRA 高效微调系统",
// 解决什么真问题, item 1; dropout of the branch input is one of the small ops
// listed there.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace lora {

constexpr int kSkConsumerWarps = 4;
constexpr int kSkThreads = (kSkConsumerWarps + 1) * 32;  // + 1 producer warp
constexpr int kSkBK = 64;                                 // columns per stage (one 128-byte swizzled row)
constexpr int kSkMaxStages = 16;
constexpr int kSkRedBytes = kSkConsumerWarps * 32 * kShrinkN * 4;  // per-warp partials, fp32
constexpr int kSkFinBytes = kTileM * kShrinkN * 4;        // CTA partial [128 x 64] fp32
// Two builds of the shrink: for pieces of up to 64 rank columns (four 16-column
// blocks), two CTAs per SM with a 108 KB stage ring; for pieces of at most 32
// (two blocks: fewer accumulator registers), three CTAs per SM with 72 KB, so
// runs of many small adapters fill the GPU in fewer waves.
__host__ __device__ constexpr int sk_ctas_per_sm(int max_nb16) { return max_nb16 <= 2 ? 3 : 2; }
__host__ __device__ constexpr int sk_pool(int max_nb16) { return max_nb16 <= 2 ? 72 * 1024 : 108 * 1024; }
__host__ __device__ constexpr int sk_smem(int max_nb16) { return 1024 + sk_pool(max_nb16) + 2 * kSkMaxStages * 8 + 64; }
// the partials and the CTA sum reuse the idle ring; the CTAs fit on an SM
static_assert(kSkRedBytes + kSkFinBytes <= sk_pool(2), "shrink reduction scratch exceeds the stage pool");
static_assert(2 * (sk_smem(4) + 1024) <= 228 * 1024, "two shrink CTAs must fit on an SM");
static_assert(3 * (sk_smem(2) + 1024) <= 228 * 1024, "three small-piece shrink CTAs must fit on an SM");

struct ShrinkParams {
  int32_t mode;     // 0: forward shrink over plan units; 1: backward dU over consecutive tiles
  int32_t T, K;     // tokens, contraction length
  int32_t ksplit;   // cluster size along the contraction
  int32_t kslice;   // contraction columns per cluster rank (multiple of kSkBK)
  int32_t x_sorted;   // 1: the In tensor map covers the plan's sorted copy of X (unit rows at g.row0)
  // forward
  const UnitDesc *units;
  const ChunkDesc *chunks;
  const TileDesc *tiles;
  const int32_t *perm;
  const float *scale;
  uint64_t seed, thr;
  float inv_keep;
  // precomputed keep bits (null: hash each element): word t * wpr + col / 32, bit col % 32
  const uint32_t *keep_bits;
  int64_t wpr;
  int32_t bits_tma;  // 1: units of consecutive tokens copy their bits with each stage (mapBits16)
  uint8_t *uimg;
  float *U_save;
  int32_t r_max;     // U_save's row length
  int32_t u_sorted;  // 1: U_save rows in the plan's sorted order, else the original token order
  // backward
  int32_t r;
  int32_t npieces;
  float scale1;
  float *dU;                 // [T, 16 * ceil(r / 16)] fp32, zero past r
};

struct UnitGeom {
  int32_t rows;      // valid rows (<= 128)
  int32_t row0;      // first sorted position (forward) or first token (backward)
  int32_t contig;    // original index of the first row if rows are consecutive originals, else -1
  int32_t frow;      // first F row of the piece
  int32_t nn;        // piece width (multiple of 16, <= 64)
  int32_t nvalid;    // columns of the piece that are real ranks (rest are zero)
  // forward only (lo: tile-local first row of the unit; clo, chi: the chunk's rows)
  int32_t tile, lo, kcol, kc, adapter, n0, last, clo, chi, zero_fill;
  int64_t uofs;  // the tile's image offset
};

__device__ __forceinline__ UnitGeom unit_geom(const ShrinkParams &p, int u) {
  UnitGeom g;
  if (p.mode == 0) {
    const UnitDesc ud = p.units[u];  // one 80-byte record
    g.rows = ud.r1 - ud.r0;
    g.row0 = ud.row0;
    g.contig = ud.contig;
    g.frow = ud.frow;
    g.nn = ud.nn;
    g.nvalid = ud.nvalid;
    g.tile = ud.tile;
    g.lo = ud.r0;
    g.clo = ud.clo;
    g.chi = ud.chi;
    g.zero_fill = ud.zero_fill;
    g.kcol = ud.kcol;
    g.kc = ud.kc;
    g.adapter = ud.adapter;
    g.n0 = ud.n0;
    g.last = ud.last;
    g.uofs = ud.uofs;
  } else {
    const int m = u / p.npieces;
    const int piece = u % p.npieces;
    g.rows = min(kTileM, p.T - m * kTileM);
    g.row0 = m * kTileM;
    g.contig = g.row0;
    g.n0 = piece * kShrinkN;
    g.nn = min(kShrinkN, ((p.r + 15) / 16) * 16 - g.n0);
    g.frow = g.n0;
    g.nvalid = max(0, min(g.nn, p.r - g.n0));
    g.tile = m;
    g.lo = 0;
    g.kcol = 0;
    g.kc = 0;
    g.adapter = 0;
    g.last = 0;
    g.clo = 0;
    g.chi = 0;
    g.zero_fill = 0;
    g.uofs = 0;
  }
  return g;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// zero the bf16 halves of a packed pair whose mask bit says "dropped"
__device__ __forceinline__ uint32_t mask_pair(uint32_t v, bool keep_lo, bool keep_hi) {
  return (keep_lo ? (v & 0xFFFFu) : 0u) | (keep_hi ? (v & 0xFFFF0000u) : 0u);
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// AND the A-fragment registers v01 (columns c, c + 1) and v89 (c + 8, c + 9)
// of one row with that row's keep bits x (bit 0 = column c): the two shifts put
// the bits on byte sign positions and prmt's sign-replicate selectors widen
// each to a 16-bit all-ones / all-zeros lane mask.
__device__ __forceinline__ void apply_keep(uint32_t &v01, uint32_t &v89, uint32_t x) {
  const uint32_t a = x << 7, b = x << 14;
  uint32_t m01, m89;
  asm("prmt.b32 %0, %1, %2, 0xDD88;" : "=r"(m01) : "r"(a), "r"(b));
  asm("prmt.b32 %0, %1, %2, 0xEE99;" : "=r"(m89) : "r"(a), "r"(b));
  v01 &= m01;
  v89 &= m89;
}

// What one consumer warp of the shrink needs to walk the stage ring.
struct ShrinkWarp {
  uint32_t pool, full0, empty0;
  int stage_bytes, nstage, nblk, kbeg, Rp, mb, MW, KW, mphase, kphase;
  int NB;  // 64-column blocks per ring stage (a multiple of KW)
  int mask;  // dropout on X: 0 none, 1 keep bits staged with the rows, 2 keep bits from HBM, 3 hash
};

constexpr int kSkConsumerBar = 1;  // named barrier of the 256 consumer threads

// One consumer warp: m16n8k16 MMAs of its m-blocks (mphase and, when the unit
// has more, mphase + MW) over the stages kphase, kphase + KW, ... against the
// NB16 16-column blocks of the F rows. The ldmatrix offsets inside a stage are
// the same for every stage (128-byte swizzle, 1024-byte aligned stage parts),
// so they are computed once. After the last stage the warp writes its partial
// sums to red[warp][slot * 16 + row][col] in the freed stage pool.
template <int NB16>
__device__ __forceinline__ void shrink_consume(const ShrinkWarp &w, const ShrinkParams &p, const UnitGeom &g,
                                               const int64_t (&orow)[2][2], const uint8_t *smem,
                                               volatile int *abort_flag, float *red, int warp, int lane) {
  float acc[2][2 * NB16][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2 * NB16; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  const int l7 = lane & 7, mi = lane >> 3;
  uint32_t aoff[4], boff[4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    // ldmatrix x4: lanes 8q .. 8q + 7 address the rows of matrix q; a row's
    // 16-byte chunk c sits at chunk c ^ (row & 7), and row & 7 == lane & 7
    aoff[ks] = ((mi & 1) * 8 + l7) * 128 + ((((2 * ks + (mi >> 1)) ^ l7) & 7) << 4);
    boff[ks] = ((mi >> 1) * 8 + l7) * 128 + ((((2 * ks + (mi & 1)) ^ l7) & 7) << 4);
  }
  const bool two = w.mphase + w.MW < w.mb;  // the warp has a second m-block
  const int q2 = 2 * (lane & 3);
  int rr[2][2];  // unit rows of the lane's fragments, clamped to the valid rows
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) rr[i][h] = min((w.mphase + i * w.MW) * 16 + (lane >> 2) + 8 * h, g.rows - 1);

  // the MMAs of 64-column block b, whose X rows start at xb
  auto consume = [&](int b, uint32_t xb) {
    const uint32_t fbuf = xb + w.Rp * 128;
    const int col = w.kbeg + b * kSkBK;  // first column of the stage, a multiple of 64
    // keep bits of the lane's rows for the stage's 64 columns: words
    // col / 32 and col / 32 + 1 of each row
    uint32_t kw[2][2][2];
    if (w.mask == 1) {
      // the stage holds words 4 * (col / 128) .. + 3 of every row; ours are
      // words (col / 32) & 3 (0 or 2) and the next
      const uint32_t *bs = reinterpret_cast<const uint32_t *>(smem + (fbuf - w.pool) + g.nn * 128);
      const int wd = (col >> 5) & 3;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (i == 1 && !two) break;
          const uint2 v = *reinterpret_cast<const uint2 *>(bs + rr[i][h] * 4 + wd);
          kw[i][h][0] = v.x;
          kw[i][h][1] = v.y;
        }
    } else if (w.mask == 2) {
      // columns past K are zero in the stage: their bits are not read
      const bool second = col + 32 < p.K;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (i == 1 && !two) break;
          const uint32_t *src = p.keep_bits + orow[i][h] * p.wpr + (col >> 5);
          kw[i][h][0] = __ldg(src);
          kw[i][h][1] = second ? __ldg(src + 1) : 0u;
        }
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t bf[NB16][4];
#pragma unroll
      for (int jj = 0; jj < NB16; ++jj)
        ldsm_x4(fbuf + boff[ks] + jj * 2048, bf[jj][0], bf[jj][1], bf[jj][2], bf[jj][3]);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (i == 1 && !two) break;
        const int mblk = w.mphase + i * w.MW;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(xb + aoff[ks] + mblk * 2048, a0, a1, a2, a3);
        if (w.mask == 1 || w.mask == 2) {
          const int s = (ks & 1) * 16 + q2;
          apply_keep(a0, a2, kw[i][0][ks >> 1] >> s);
          apply_keep(a1, a3, kw[i][1][ks >> 1] >> s);
        } else if (w.mask == 3) {
          const int c0 = col + ks * 16 + q2;
          a0 = mask_pair(a0, keep_elem(p.seed, p.thr, orow[i][0], c0, p.K), keep_elem(p.seed, p.thr, orow[i][0], c0 + 1, p.K));
          a1 = mask_pair(a1, keep_elem(p.seed, p.thr, orow[i][1], c0, p.K), keep_elem(p.seed, p.thr, orow[i][1], c0 + 1, p.K));
          a2 = mask_pair(a2, keep_elem(p.seed, p.thr, orow[i][0], c0 + 8, p.K), keep_elem(p.seed, p.thr, orow[i][0], c0 + 9, p.K));
          a3 = mask_pair(a3, keep_elem(p.seed, p.thr, orow[i][1], c0 + 8, p.K), keep_elem(p.seed, p.thr, orow[i][1], c0 + 9, p.K));
        }
#pragma unroll
        for (int jj = 0; jj < NB16; ++jj) {
          mma_bf16_16816(acc[i][2 * jj], a0, a1, a2, a3, bf[jj][0], bf[jj][1]);
          mma_bf16_16816(acc[i][2 * jj + 1], a0, a1, a2, a3, bf[jj][2], bf[jj][3]);
        }
      }
    }
  };

  // stage S of the ring holds blocks S*NB .. S*NB + NB - 1 (NB blocks of
  // stage_bytes each, NB a multiple of KW); warp group kphase takes blocks
  // kphase, kphase + KW, ... of it, and every consumer warp releases the stage
  const int nsuper = (w.nblk + w.NB - 1) / w.NB;
  for (int S = 0; S < nsuper; ++S) {
    const int stage = S % w.nstage;
    const uint32_t phase = static_cast<uint32_t>(S / w.nstage) & 1u;
    if (!mbar_wait(w.full0 + 8 * stage, phase)) { *abort_flag = 1; break; }
    for (int j = w.kphase; j < w.NB; j += w.KW) {
      const int b = S * w.NB + j;
      if (b < w.nblk) consume(b, w.pool + (stage * w.NB + j) * w.stage_bytes);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(w.empty0 + 8 * stage);
  }

  // every consumer warp is past its last stage: every TMA of the ring has
  // landed and been read, so the pool may be overwritten
  asm volatile("barrier.sync %0, %1;" ::"n"(kSkConsumerBar), "n"(kSkConsumerWarps * 32) : "memory");
  float *base = red + (warp * 32) * kShrinkN;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (i == 1 && !two) break;
#pragma unroll
    for (int j = 0; j < 2 * NB16; ++j) {
      const int r = i * 16 + (lane >> 2);
      const int c = j * 8 + q2;
      base[r * kShrinkN + c] = acc[i][j][0];
      base[r * kShrinkN + c + 1] = acc[i][j][1];
      base[(r + 8) * kShrinkN + c] = acc[i][j][2];
      base[(r + 8) * kShrinkN + c + 1] = acc[i][j][3];
    }
  }
}

// Where the 160 threads that run one shrink unit sit in their CTA: thread lt
// (0..159) is consumer warp lt / 32 (0..3) or, for lt >= 128, the producer warp.
// bar_id names the barrier over the 160 (0: they are the whole CTA, and
// __syncthreads serves); pdl: wait for the previous grid before touching X.
struct ShrinkRole {
  int lt;
  int bar_id;
  bool pdl;
};

// The producer warp reaches these barriers diverged (lane 0 may still be in its
// copy loop while lanes 1..31 arrive), so the named form is the non-aligned
// `barrier.sync`, which counts threads one by one; `bar.sync` is the aligned
// form, for warps that arrive converged (with a diverged warp it can complete
// before every thread has arrived). __syncthreads counts per thread as well.
__device__ __forceinline__ void shrink_bar_all(int bar_id) {
  if (bar_id == 0) __syncthreads();
  else asm volatile("barrier.sync %0, %1;" ::"r"(bar_id), "n"(kSkThreads) : "memory");
}

// One shrink unit (one CTA of its cluster): smem is the 1024-aligned stage pool
// (kPoolBytes, by default the standalone kernel's sk_pool(kMaxNB16)), bars room
// for 2 * kSkMaxStages mbarriers and a flag.
template <int kMaxNB16, int kPoolBytes = sk_pool(kMaxNB16)>
__device__ __forceinline__ bool shrink_unit(uint8_t *smem, uint64_t *bars, const CUtensorMap &mapIn16,
                                            const CUtensorMap &mapF16, const CUtensorMap &mapBits16,
                                            const ShrinkParams &p, int unit, uint32_t crank, const ShrinkRole role) {
  const uint32_t pool = smem_u32(smem);
  float *fin = reinterpret_cast<float *>(smem + kSkRedBytes);  // in the pool, after the partials
  constexpr int kSkPool = kPoolBytes;
  static_assert(kSkRedBytes + kSkFinBytes <= kPoolBytes, "the reduction scratch must fit the pool");
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kSkMaxStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 2 * kSkMaxStages);

  const int tid = role.lt;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (warp == kSkConsumerWarps && lane == 0) {
    prefetch_tmap(&mapIn16);
    prefetch_tmap(&mapF16);
    if (p.bits_tma) prefetch_tmap(&mapBits16);
  }
  const UnitGeom g = unit_geom(p, unit);  // plan tables: written before any kernel of the forward

  const int Rp = ((g.rows + 15) / 16) * 16;  // rows rounded to the MMA M step
  const int mb = Rp / 16;
  // a unit of consecutive tokens reads its keep bits from the stage: 4 words
  // (128 columns, the 16-byte-aligned span holding the stage's 64) per row
  const bool stage_bits = p.mode == 0 && p.thr != 0 && p.bits_tma && g.contig >= 0;
  // a stage: X rows, F rows (, bits); the next stage starts on a 1024-byte
  // boundary, as the 128-byte swizzle of its TMA boxes requires
  const int stage_tx = (Rp + g.nn) * 128 + (stage_bits ? Rp * 16 : 0);
  const int stage_bytes = (stage_tx + 1023) & ~1023;
  const int kbeg = static_cast<int>(crank) * p.kslice;
  const int kend = min(p.K, kbeg + p.kslice);
  const int nblk = kend > kbeg ? (kend - kbeg + kSkBK - 1) / kSkBK : 0;

  // warp work split: MW warps along rows (m-blocks), KW along the stages (warp
  // group kphase takes stages kphase, kphase + KW, ...), so the stages of a small
  // unit are consumed in parallel instead of one after another
  int MW = 1;
  while (MW * 2 <= mb && MW < kSkConsumerWarps) MW *= 2;
  const int KW = kSkConsumerWarps / MW;
  // a ring stage holds NB consecutive 64-column blocks: small units take eight
  // (at most 16 rows) or four (at most 32), shared out over the KW warp groups,
  // so their copies come in groups (a lone 16-row block pair per barrier round
  // trip kept too few bytes moving; eight measured 1.4 % faster than four on
  // fleet, the same on decode); larger units one
  const int NB = Rp <= 16 ? 8 : Rp <= 32 ? 4 : KW;
  const int nstage = min(kSkMaxStages, kSkPool / (NB * stage_bytes));

  if (tid == 0) {
    for (int s = 0; s < nstage; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kSkConsumerWarps);  // every consumer warp releases a stage
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the pool may hold what generic stores wrote before (a previous unit's sums,
  // or another role of the CTA): order them before the ring's TMA writes
  fence_proxy_async_smem();
  shrink_bar_all(role.bar_id);
  // X (or its sorted copy from the row gather) and everything else the launch
  // reads or writes come after the previous kernel on the stream has completed
  if (role.pdl) pdl_wait();

  if (warp == kSkConsumerWarps) {
    // -------------------------------------------------------------- producer
    // Lane 0 streams the unit's X rows (16-row TMA boxes: the rows are
    // consecutive either in X itself or in the plan's sorted copy of X) and
    // the adapter's F rows through the stage ring.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const int xrow = p.x_sorted ? g.row0 : g.contig;
      const int nsuper = (nblk + NB - 1) / NB;
      for (int S = 0; S < nsuper; ++S) {
        if (xrow < 0) { flag_status(LORA_DEV_BOUNDS); *abort_flag = 1; break; }
        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { *abort_flag = 1; break; }
        const uint32_t fb = full0 + 8 * stage;
        const int nb = min(NB, nblk - S * NB);  // blocks in this stage
        mbar_arrive_expect_tx(fb, nb * stage_tx);
        for (int j = 0; j < nb; ++j) {
          const uint32_t xb = pool + (stage * NB + j) * stage_bytes;
          const uint32_t fbuf = xb + Rp * 128;
          const int col = kbeg + (S * NB + j) * kSkBK;
          for (int r16 = 0; r16 < Rp; r16 += 16) tma_load_2d(xb + r16 * 128, &mapIn16, fb, col, xrow + r16);
          for (int n16 = 0; n16 < g.nn; n16 += 16) tma_load_2d(fbuf + n16 * 128, &mapF16, fb, col, g.frow + n16);
          if (stage_bits) {
            const uint32_t bb = fbuf + g.nn * 128;
            for (int r16 = 0; r16 < Rp; r16 += 16)
              tma_load_2d(bb + r16 * 16, &mapBits16, fb, (col >> 7) * 4, g.contig + r16);
          }
        }
        if (++stage == nstage) { stage = 0; phase ^= 1; }
      }
    }
  } else {
    // -------------------------------------------------------------- consumers
    ShrinkWarp w;
    w.pool = pool;
    w.full0 = full0;
    w.empty0 = empty0;
    w.stage_bytes = stage_bytes;
    w.nstage = nstage;
    w.nblk = nblk;
    w.kbeg = kbeg;
    w.Rp = Rp;
    w.mb = mb;
    w.MW = MW;
    w.KW = KW;
    w.NB = NB;
    w.mphase = warp % MW;
    w.kphase = warp / MW;
    w.mask = (p.mode != 0 || p.thr == 0) ? 0 : (stage_bits ? 1 : (p.keep_bits ? 2 : 3));
    // original token index of the two rows this lane's fragments touch, per m-block slot
    int64_t orow[2][2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = (w.mphase + i * MW) * 16 + (lane >> 2) + 8 * h;
        const int rc = min(r, g.rows - 1);
        orow[i][h] = g.contig >= 0 ? static_cast<int64_t>(g.contig + rc)
                                   : (p.mode == 0 ? static_cast<int64_t>(p.perm[g.row0 + rc]) : 0);
      }
    float *red = reinterpret_cast<float *>(smem);
    // the piece width nn is 16, 32, 48 or 64 (at most 16 * kMaxNB16: the host
    // launches the small build only for such pieces)
    if constexpr (kMaxNB16 <= 2) {
      if (g.nn <= 16) shrink_consume<1>(w, p, g, orow, smem, abort_flag, red, warp, lane);
      else shrink_consume<2>(w, p, g, orow, smem, abort_flag, red, warp, lane);
    } else {
      switch (g.nn >> 4) {
        case 1: shrink_consume<1>(w, p, g, orow, smem, abort_flag, red, warp, lane); break;
        case 2: shrink_consume<2>(w, p, g, orow, smem, abort_flag, red, warp, lane); break;
        case 3: shrink_consume<3>(w, p, g, orow, smem, abort_flag, red, warp, lane); break;
        default: shrink_consume<4>(w, p, g, orow, smem, abort_flag, red, warp, lane); break;
      }
    }
  }

  // ---------------------------------------------------------------- CTA reduction
  // the consumers left their partial sums in red[w][slot*16 + row][col] (fp32,
  // the idle stage pool); fin[row][col] = the sum over the KW warps of a row.
  // Threads work on float4 column groups: nq per row, rpp rows per pass.
  float *red = reinterpret_cast<float *>(smem);
  shrink_bar_all(role.bar_id);
  const int nq = g.nn >> 2;
  const int rpp = kSkThreads / nq;
  const int tq = tid % nq;
  const int tr = tid / nq;
  int lmw = 0;
  while ((1 << lmw) < MW) ++lmw;
  if (tr < rpp) {
    for (int r = tr; r < Rp; r += rpp) {
      const int mblk = r >> 4;
      const int row_in = ((mblk >> lmw) << 4) + (r & 15);  // slot * 16 + row in the m-block
      float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int kp = 0; kp < KW; ++kp) {
        const int w = kp * MW + (mblk & (MW - 1));
        const float4 v = *reinterpret_cast<const float4 *>(red + (w * 32 + row_in) * kShrinkN + tq * 4);
        s4.x += v.x;
        s4.y += v.y;
        s4.z += v.z;
        s4.w += v.w;
      }
      *reinterpret_cast<float4 *>(fin + r * kShrinkN + tq * 4) = s4;
    }
  }

  // ---------------------------------------------------------------- cluster reduction
  // rank q completes the tile rows [tr0, tr1): it sums those of the unit's rows
  // over the ranks (in rank order, so the result does not depend on which rank
  // sums) and writes their outputs; the ranks' shares run in parallel
  const int ksp = p.ksplit;
  const int tr0 = static_cast<int>(crank) * kTileM / ksp;
  const int tr1 = (static_cast<int>(crank) + 1) * kTileM / ksp;
  const int lr0 = max(0, tr0 - g.lo);
  const int lr1 = min(g.rows, tr1 - g.lo);
  if (ksp > 1) {
    cluster_sync_all();  // every rank's fin is final
    if (tr < rpp) {
      for (int lr = lr0 + tr; lr < lr1; lr += 4 * rpp) {
        // up to 4 rows per thread with their remote loads in flight together
        float4 part[4][4];  // [row][rank]
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rr = min(lr + u * rpp, lr1 - 1);
          const uint32_t la = smem_u32(fin + rr * kShrinkN + tq * 4);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q >= ksp) break;
            part[u][q] = q == static_cast<int>(crank) ? *reinterpret_cast<const float4 *>(fin + rr * kShrinkN + tq * 4)
                                                     : ld_dsmem_f32x4(map_to_rank(la, static_cast<uint32_t>(q)));
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rr = lr + u * rpp;
          if (rr >= lr1) break;
          float4 s4 = part[u][0];
#pragma unroll
          for (int q = 1; q < 4; ++q) {
            if (q >= ksp) break;
            s4.x += part[u][q].x;
            s4.y += part[u][q].y;
            s4.z += part[u][q].z;
            s4.w += part[u][q].w;
          }
          // only this rank reads these rows of fin from here on
          *reinterpret_cast<float4 *>(fin + rr * kShrinkN + tq * 4) = s4;
        }
      }
    }
    cluster_sync_all();  // the peers' fin was read: every rank may go on and exit
  } else {
    shrink_bar_all(role.bar_id);  // fin is complete before any thread reads a row of it
  }
  // every thread is past its last use of the ring's barriers: invalidate them, so
  // that the next unit of a fused launch can initialise them afresh (and the
  // GEMM's ring may overwrite their memory)
  // (not after a wait gave up: a copy may still be in flight to the ring)
  const bool unit_ok = !*abort_flag;
  if (tid == 0 && unit_ok)
    for (int s = 0; s < nstage; ++s) {
      mbar_inval(full0 + 8 * s);
      mbar_inval(empty0 + 8 * s);
    }

  if (p.mode == 0) {
    const float s_a = p.scale[g.adapter] * p.inv_keep;
    // s·U of the tile in columns [kcol, kcol + nn) (bf16 hi part) and
    // [kcol + kc, kcol + kc + nn) (bf16 lo part: the rounding remainder): the
    // unit's rows, and (one row piece per chunk) the zeros of the tile rows
    // outside the chunk; the chunk's other rows belong to its other pieces
    uint8_t *img = p.uimg + g.uofs;
    const int n8 = g.nn >> 3;
    const int rp8 = kSkThreads / n8;
    const int t8 = tid % n8;
    const int trow = tid / n8;
    if (trow < rp8) {
      const int c8 = t8 * 8;
      for (int row = tr0 + trow; row < tr1; row += rp8) {
        const int lr = row - g.lo;
        const bool mine = lr >= 0 && lr < g.rows;
        if (!mine && !(g.zero_fill && (row < g.clo || row >= g.chi))) continue;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
        if (mine) {
          const float4 x0 = *reinterpret_cast<const float4 *>(fin + lr * kShrinkN + c8);
          const float4 x1 = *reinterpret_cast<const float4 *>(fin + lr * kShrinkN + c8 + 4);
          const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = c8 + j < g.nvalid ? xs[j] * s_a : 0.f;
        }
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          hi[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
          lo[j] = pack_bf16x2(v[2 * j] - bf16_lo(hi[j]), v[2 * j + 1] - bf16_hi(hi[j]));
        }
        const int col = g.kcol + c8;
        uint8_t *dst = img + (col / kAugBlock) * kAugBlockBytes + sw128_offset(row, col % kAugBlock);
        *reinterpret_cast<uint4 *>(dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        const int col2 = col + g.kc;
        uint8_t *dst2 = img + (col2 / kAugBlock) * kAugBlockBytes + sw128_offset(row, col2 % kAugBlock);
        *reinterpret_cast<uint4 *>(dst2) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    if (p.U_save) {
      // one warp per row: columns n0 .. cend of the token's U_save row (zeros
      // past the adapter's rank up to r_max on the chunk's last piece)
      const int cend = g.last ? p.r_max : min(p.r_max, g.n0 + g.nn);
      const int ncol = max(0, cend - g.n0);
      const int nw = kSkThreads >> 5;
      for (int lr = lr0 + warp; lr < lr1; lr += nw) {
        const int64_t orig = p.u_sorted ? static_cast<int64_t>(g.row0 + lr)
                             : g.contig >= 0 ? static_cast<int64_t>(g.contig + lr) : p.perm[g.row0 + lr];
        float *dst = p.U_save + orig * p.r_max + g.n0;
        for (int c = lane; c < ncol; c += 32) dst[c] = c < g.nvalid ? fin[lr * kShrinkN + c] * p.inv_keep : 0.f;
      }
    }
  } else {
    // rows of dU are padded to a multiple of 16 ranks with zeros, so that the
    // token contraction reads whole 16-rank groups
    const int nw = kSkThreads >> 5;
    const int64_t stride = ((p.r + 15) / 16) * 16;
    for (int lr = lr0 + warp; lr < lr1; lr += nw) {
      float *dst = p.dU + static_cast<int64_t>(g.row0 + lr) * stride + g.n0;
      for (int c = lane; c < g.nn; c += 32) dst[c] = c < g.nvalid ? fin[lr * kShrinkN + c] * p.scale1 : 0.f;
    }
  }
  return unit_ok;
}

// Grid: n_units * ksplit CTAs, clusters of ksplit along x. Cluster c handles unit c;
// its rank q contracts columns [q*kslice, (q+1)*kslice).
template <int kMaxNB16>
__global__ void __launch_bounds__(kSkThreads, sk_ctas_per_sm(kMaxNB16))
    lora_shrink_kernel(const __grid_constant__ CUtensorMap mapIn16,  // In rows (X, sorted X or dY), box {64, 16}
                       const __grid_constant__ CUtensorMap mapF16,   // F rows, box {64, 16}
                       const __grid_constant__ CUtensorMap mapBits16,  // keep bits [T, wpr] u32, box {4, 16}
                       const ShrinkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  pdl_launch_dependents();  // the fused GEMM may set itself up meanwhile
  shrink_unit<kMaxNB16>(smem, reinterpret_cast<uint64_t *>(smem + sk_pool(kMaxNB16)), mapIn16, mapF16, mapBits16, p,
                        static_cast<int>(blockIdx.x) / p.ksplit, cluster_ctarank(),
                        ShrinkRole{static_cast<int>(threadIdx.x), 0, true});
}

// ------------------------------------------------------------------ token contraction
constexpr int kTcConsumerWarps = 4;
constexpr int kTcThreads = (kTcConsumerWarps + 1) * 32;  // + producer warp
constexpr int kTcMaxStages = 6;
constexpr int kTcTok = 64;        // tokens per stage
constexpr int kTcCols = 128;      // columns per CTA (32 per consumer warp)
constexpr int kTcMaxR = 64;
constexpr int kTcSmemBudget = 110 * 1024;  // stage ring per CTA: two CTAs share an SM
constexpr int kTcSmemBudgetWide = 216 * 1024;  // rank groups wider than 32: one CTA per SM
constexpr int kTcParts = 3;                 // bf16 parts of G (hi, mid, lo)
__host__ __device__ inline int tc_budget(int r) { return r <= 32 ? kTcSmemBudget : kTcSmemBudgetWide; }

// Bytes of one stage of the token contraction: In [64 tokens][128 columns] as two
// 64-column halves (128-byte swizzle), G [64 tokens][r] fp32 as copied, the
// stage's keep bits [64 tokens][4 words] when read, and G^T split into bf16
// parts (hi, mid, lo), [16 * mblocks ranks][64 tokens] each (128-byte rows,
// swizzled).
__host__ __device__ inline int tc_stage_bytes(int r, bool bits) {
  const int mblocks = (r + 15) / 16;
  return kTcTok * kTcCols * 2 + ((kTcTok * r * 4 + 1023) & ~1023) + (bits ? 1024 : 0) + kTcParts * mblocks * 2048;
}
__host__ __device__ inline int tc_stages(int r, bool bits) {
  const int n = tc_budget(r) / tc_stage_bytes(r, bits);
  return n < kTcMaxStages ? n : kTcMaxStages;
}
// dynamic shared memory of a launch whose rank groups are at most r wide
__host__ __device__ inline int tc_smem(int r) { return 1024 + tc_budget(r) + 2 * kTcMaxStages * 8; }

struct TcParams {
  int32_t T, N;
  int32_t r;               // ranks of this launch's group, a multiple of 16, <= kTcMaxR (G is
                           // zero past the real ranks)
  int32_t r_valid;         // real ranks of the group (<= r): rows written
  int32_t k0;              // first rank of the group
  int32_t r_total;         // ranks of the whole contraction (row count of a split's partial)
  int32_t splits, tsplit;  // token splits, tokens per split (multiple of 64)
  uint64_t seed, thr;      // mask on In (dA); thr = 0 for none
  const uint32_t *keep_bits;  // precomputed keep bits of In (null: hash), word t * wpr + col / 32
  int64_t wpr;
  float *partial;          // [splits][r_total][N]; piece mode: [partial rows][N]
  // piece mode (pieces != null, multi-adapter backward): CTA (x, y, z) takes
  // column block x of pieces range_off[y] .. range_off[y + 1] - 1, one after
  // another through one stage ring, ranks [64z, 64z + 64) of each piece's
  // adapter (rp: the ranks rounded up to 16 of the widest adapter; the group's
  // width selects the G map). A segment of one piece writes
  // out[(pool_row + k) * N + n] = scale[adapter] * factor * sum; the pieces of a
  // longer segment write partial rows (partial_row + k) for a later reduction.
  const PieceDesc *pieces;
  const int32_t *range_off;
  int32_t rp;
  const float *scale;
  float factor;
  float *out;
  const int32_t *perm;     // rows of In are sorted positions: the mask hash uses perm[row]
};

// split fp32 values into three bf16 parts, hi = rn(v), mid = rn(v - hi),
// lo = rn(v - hi - mid) (each remainder exact in fp32), packed in pairs
__device__ __forceinline__ void split3_pair(float v0, float v1, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
  hi = pack_bf16x2(v0, v1);
  const float r0 = v0 - bf16_lo(hi), r1 = v1 - bf16_hi(hi);
  mid = pack_bf16x2(r0, r1);
  lo = pack_bf16x2(r0 - bf16_lo(mid), r1 - bf16_hi(mid));
}

// Mask of a transposed B fragment register: its two bf16 halves are tokens t
// and t + 1 of one column, whose keep bits are bit 0 of xa and xb (sel 0xCC88)
// or bit 8 (the column 8 further on, sel 0xDD99).
template <uint32_t kSel>
__device__ __forceinline__ uint32_t keep_pair_t(uint32_t xa, uint32_t xb) {
  uint32_t m;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m) : "r"(xa << 7), "r"(xb << 7), "n"(kSel));
  return m;
}

// partial[q][k][n] = sum_{t in split q} G[t, k] * In[t, n] (In masked if thr != 0).
// Grid (N / 128, splits). Warp w < 4 owns columns [32w, 32w + 32) of the CTA's
// 128. The consumer warps first turn the stage's fp32 G into its transposed hi
// and lo bf16 images (once for all warps), then each k16 step takes two
// transposed In fragments and, per 16 ranks, two G^T fragments and eight MMAs.
// Barrier 1 over the consumer warps (kTcConsumerWarps * 32 threads): true for
// every participant when all of them passed true.
__device__ __forceinline__ bool tc_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kTcConsumerWarps * 32)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kTcThreads, 2)
    lora_tcontract_kernel(const __grid_constant__ CUtensorMap mapIn,  // In [T, N] bf16, box {64, 64}, swizzle 128B
                          const __grid_constant__ CUtensorMap mapG,   // G [T, >= k0 + r] fp32, box {r, 64}, no swizzle
                          const __grid_constant__ CUtensorMap mapBits,  // keep bits [T, wpr] u32, box {4, 64}
                          const __grid_constant__ CUtensorMap mapG16,  // piece mode: G maps of boxes {16, 64},
                          const __grid_constant__ CUtensorMap mapG32,  // {32, 64}, {48, 64} (mapG: {64, 64})
                          const __grid_constant__ CUtensorMap mapG48,
                          const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  // this CTA's ranks [k0, k0 + r) (r a multiple of 16) and its segments lo .. hi - 1:
  // one token split, or a range of pieces
  int r = p.r, k0 = p.k0, lo = 0, hi = 1;
  const CUtensorMap *gmap = &mapG;
  if (p.pieces) {
    k0 = static_cast<int>(blockIdx.z) * kTcMaxR;
    r = min(kTcMaxR, p.rp - k0);
    if (r <= 0) return;  // no barrier has been set up yet
    gmap = r == 16 ? &mapG16 : r == 32 ? &mapG32 : r == 48 ? &mapG48 : &mapG;
    lo = p.range_off[blockIdx.y];
    hi = p.range_off[blockIdx.y + 1];
  }
  // segment s: In (and keep-bit) rows [t0, t1), G rows from g0 (piece mode: the
  // piece's sorted positions); false when the segment's adapter has no rank in
  // this CTA's group
  auto segment = [&](int s, int &t0, int &t1, int &g0) -> bool {
    if (p.pieces) {
      const PieceDesc pc = p.pieces[s];
      if (pc.rank <= k0) return false;
      t0 = pc.in_row;
      t1 = pc.in_row + pc.len;
      g0 = pc.start;
    } else {
      t0 = blockIdx.y * p.tsplit;
      t1 = min(p.T, t0 + p.tsplit);
      g0 = t0;
    }
    return true;
  };
  const bool bits = p.keep_bits != nullptr;
  const int mblocks = (r + 15) / 16;
  const int in_bytes = kTcTok * kTcCols * 2;    // 16 KB (two 8 KB halves)
  const int g_bytes = kTcTok * r * 4;           // <= 16 KB
  const int g_pad = (g_bytes + 1023) & ~1023;
  const int bits_bytes = bits ? 1024 : 0;       // the stage's keep bits
  const int conv_off = in_bytes + g_pad + bits_bytes;  // G^T hi, mid, lo (mblocks * 2 KB each)
  const int stage_bytes = tc_stage_bytes(r, bits);
  const int nstage = tc_stages(r, bits);
  const uint32_t pool = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + nstage * stage_bytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kTcMaxStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTcCols;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kTcConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kTcConsumerWarps) {
    if (lane == 0) {
      prefetch_tmap(&mapIn);
      prefetch_tmap(gmap);
      if (bits) prefetch_tmap(&mapBits);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int sg = lo; sg < hi && ok; ++sg) {
        int t0, t1, g0;
        if (!segment(sg, t0, t1, g0)) continue;
        const int nblk = t1 > t0 ? (t1 - t0 + kTcTok - 1) / kTcTok : 0;
        for (int b = 0; b < nblk; ++b) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sb = pool + stage * stage_bytes;
          const int t = t0 + b * kTcTok;
          mbar_arrive_expect_tx(fb, in_bytes + g_bytes + bits_bytes);
          tma_load_2d(sb, &mapIn, fb, n0, t);
          tma_load_2d(sb + 8192, &mapIn, fb, n0 + 64, t);
          tma_load_2d(sb + in_bytes, gmap, fb, k0, t - t0 + g0);  // this CTA's group of ranks
          if (bits) tma_load_2d(sb + in_bytes + g_pad, &mapBits, fb, n0 / 32, t);
          if (++stage == nstage) { stage = 0; phase ^= 1; }
        }
      }
    }
    return;  // no block-wide barrier follows
  }

  // ------------------------------------------------------------------ consumers
  const int cw = warp * 32;     // the warp's first column of the CTA's 128
  const int half = cw / 64;     // which 64-column half of the stage
  const int cin = cw % 64;      // column offset inside the half (0 or 32)
  const int mi = lane >> 3;
  const int l7 = lane & 7;
  // transposed In fragments of column group g (16 columns) at k16 step ks:
  // lanes 8q .. 8q + 7 address tokens ks*16 + (q & 1)*8 + (lane & 7) of chunk
  // cin/8 + 2g + (q >> 1)
  uint32_t boff[4][2];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const int tr = ks * 16 + (mi & 1) * 8 + l7;
      const int chunk = (cin >> 3) + 2 * g + (mi >> 1);
      boff[ks][g] = half * 8192 + tr * 128 + (((chunk ^ (tr & 7)) & 7) << 4);
    }
  // G^T fragments (ranks x tokens, row-major) from the hi / mid / lo images:
  // rank rows (q & 1)*8 + (lane & 7) of the 16-rank block, token chunk ks*2 + (q >> 1)
  uint32_t aoff[4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int m = (mi & 1) * 8 + l7;
    aoff[ks] = m * 128 + ((((2 * ks + (mi >> 1)) ^ (m & 7)) & 7) << 4);
  }
  const int q2 = 2 * (lane & 3);
  const int tid = static_cast<int>(threadIdx.x);  // 0 .. 127

  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int sg = lo; sg < hi && ok; ++sg) {
    int t0, t1, g0;
    if (!segment(sg, t0, t1, g0)) continue;
    const int nblk = t1 > t0 ? (t1 - t0 + kTcTok - 1) / kTcTok : 0;
    float acc[4][2][2][4];  // [m-block][column group][n8][fragment]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[i][g][j][e] = 0.f;

    for (int b = 0; b < nblk; ++b) {
      // the stage's wait; the four warps agree on its outcome at the barrier
      // below, so that none is left waiting there for a warp that gave up
      const bool landed = mbar_wait(full0 + 8 * stage, phase);
      const uint32_t sb = pool + stage * stage_bytes;
      uint8_t *const sbp = smem + (sb - pool);
      // G^T images of this stage. Work item = (token pair tp, 4 consecutive ranks
      // from k4): G[2tp][k4 .. k4 + 3] and G[2tp + 1][k4 .. k4 + 3] as two 16-byte
      // reads (consecutive threads take consecutive ranks, so the reads do not
      // collide on banks), written as (hi, mid, lo) bf16 pairs at rank rows
      // k4 .. k4 + 3, tokens 2tp and 2tp + 1. Rank rows from r to 16 * mblocks
      // are zero, and so are the columns of tokens at or past t1 (in piece mode
      // the stage's last rows can be the next segment's tokens, which must not
      // enter the sums).
      // Only the stage's 16-token steps that hold tokens of the segment take
      // part (nk of them): a short piece (a few tokens of a small adapter)
      // converts and multiplies one step instead of four; the steps left out
      // would only add products of zero columns.
      const int nk = (min(kTcTok, t1 - (t0 + b * kTcTok)) + 15) / 16;
      {
        const int tb = t0 + b * kTcTok;
        const float *graw = reinterpret_cast<const float *>(sbp + in_bytes);
        uint8_t *ghi = sbp + conv_off;
        uint8_t *gmid = ghi + mblocks * 2048;
        uint8_t *glo = gmid + mblocks * 2048;
        const int q4 = mblocks * 4;  // 4-rank groups per token pair
        const int items = 8 * nk * q4;  // token pairs of the steps taken
        for (int item = landed ? tid : items; item < items; item += kTcConsumerWarps * 32) {
          const int tp = item / q4;
          const int k4 = (item - tp * q4) * 4;
          float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
          if (k4 < r) {  // r % 16 == 0: a group is all in or all out
            if (tb + 2 * tp < t1) v0 = *reinterpret_cast<const float4 *>(graw + (2 * tp) * r + k4);
            if (tb + 2 * tp + 1 < t1) v1 = *reinterpret_cast<const float4 *>(graw + (2 * tp + 1) * r + k4);
          }
          const float a0[4] = {v0.x, v0.y, v0.z, v0.w};
          const float a1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int k = k4 + u;
            uint32_t hi, mid, lo;
            split3_pair(a0[u], a1[u], hi, mid, lo);
            const uint32_t off = k * 128 + ((((tp >> 2) ^ (k & 7)) & 7) << 4) + (tp & 3) * 4;
            *reinterpret_cast<uint32_t *>(ghi + off) = hi;
            *reinterpret_cast<uint32_t *>(gmid + off) = mid;
            *reinterpret_cast<uint32_t *>(glo + off) = lo;
          }
        }
      }
      if (!tc_bar_and(landed)) { ok = false; break; }
      const uint32_t ghi_s = sb + conv_off;
      const uint32_t gmid_s = ghi_s + mblocks * 2048;
      const uint32_t glo_s = gmid_s + mblocks * 2048;
      const uint32_t *bs = reinterpret_cast<const uint32_t *>(sbp + in_bytes + g_pad);
      const int tbase = t0 + b * kTcTok;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks >= nk) break;  // uniform
        uint32_t bf[2][4];
#pragma unroll
        for (int g = 0; g < 2; ++g) ldsm_x4_t(sb + boff[ks][g], bf[g][0], bf[g][1], bf[g][2], bf[g][3]);
        if (p.thr != 0) {
          // bf[g][0]: tokens tl, tl + 1 of column c = n0 + cw + 16g + lane/4;
          // [1]: tokens + 8; [2], [3]: column + 8
          const int tl = ks * 16 + q2;
          if (bits) {
            // the stage's bits: [64 tokens][4 words] for its 128 columns; the
            // warp's 32 columns are word cw / 32, and c, c + 8 share it
            const int wd = cw >> 5;
            const uint32_t w0 = bs[tl * 4 + wd], w1 = bs[(tl + 1) * 4 + wd];
            const uint32_t w8 = bs[(tl + 8) * 4 + wd], w9 = bs[(tl + 9) * 4 + wd];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int sh = 16 * g + (lane >> 2);
              const uint32_t x0 = w0 >> sh, x1 = w1 >> sh, x8 = w8 >> sh, x9 = w9 >> sh;
              bf[g][0] &= keep_pair_t<0xCC88>(x0, x1);
              bf[g][1] &= keep_pair_t<0xCC88>(x8, x9);
              bf[g][2] &= keep_pair_t<0xDD99>(x0, x1);
              bf[g][3] &= keep_pair_t<0xDD99>(x8, x9);
            }
          } else {
            // the mask is indexed by original token: rows past the token range
            // meet zero G columns, their bits are never used
            const int tk = tbase + tl;
            int64_t o0 = tk, o1 = tk + 1, o8 = tk + 8, o9 = tk + 9;
            if (p.perm) {
              o0 = p.perm[min(tk, t1 - 1)];
              o1 = p.perm[min(tk + 1, t1 - 1)];
              o8 = p.perm[min(tk + 8, t1 - 1)];
              o9 = p.perm[min(tk + 9, t1 - 1)];
            }
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int c = n0 + cw + 16 * g + (lane >> 2);
              bf[g][0] = mask_pair(bf[g][0], keep_elem(p.seed, p.thr, o0, c, p.N), keep_elem(p.seed, p.thr, o1, c, p.N));
              bf[g][1] = mask_pair(bf[g][1], keep_elem(p.seed, p.thr, o8, c, p.N), keep_elem(p.seed, p.thr, o9, c, p.N));
              bf[g][2] = mask_pair(bf[g][2], keep_elem(p.seed, p.thr, o0, c + 8, p.N), keep_elem(p.seed, p.thr, o1, c + 8, p.N));
              bf[g][3] = mask_pair(bf[g][3], keep_elem(p.seed, p.thr, o8, c + 8, p.N), keep_elem(p.seed, p.thr, o9, c + 8, p.N));
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (i >= mblocks) break;
          uint32_t h0, h1, h2, h3, m0, m1, m2, m3, l0, l1, l2, l3;
          ldsm_x4(ghi_s + i * 2048 + aoff[ks], h0, h1, h2, h3);
          ldsm_x4(gmid_s + i * 2048 + aoff[ks], m0, m1, m2, m3);
          ldsm_x4(glo_s + i * 2048 + aoff[ks], l0, l1, l2, l3);
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            // smallest parts first, so the partial sums grow from the small end
            mma_bf16_16816(acc[i][g][0], l0, l1, l2, l3, bf[g][0], bf[g][1]);
            mma_bf16_16816(acc[i][g][1], l0, l1, l2, l3, bf[g][2], bf[g][3]);
            mma_bf16_16816(acc[i][g][0], m0, m1, m2, m3, bf[g][0], bf[g][1]);
            mma_bf16_16816(acc[i][g][1], m0, m1, m2, m3, bf[g][2], bf[g][3]);
            mma_bf16_16816(acc[i][g][0], h0, h1, h2, h3, bf[g][0], bf[g][1]);
            mma_bf16_16816(acc[i][g][1], h0, h1, h2, h3, bf[g][2], bf[g][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * stage);
      if (++stage == nstage) { stage = 0; phase ^= 1; }
    }
    if (!ok) break;
    // write partial[q][k0 + k][n] for the group's real ranks; piece mode: the
    // adapter's gradient rows (scaled) or the piece's partial rows. The stores
    // overlap the copies of the next segment's stages.
    float *out;
    float f = 1.f;
    int r_valid = p.r_valid;
    if (p.pieces) {
      const PieceDesc pc = p.pieces[sg];
      r_valid = min(r, pc.rank - k0);
      if (pc.seg_pieces == 1) {
        out = p.out + (static_cast<int64_t>(pc.pool_row) + k0) * p.N;
        f = p.scale[pc.adapter] * p.factor;
      } else {
        out = p.partial + (static_cast<int64_t>(pc.partial_row) + k0) * p.N;
      }
    } else {
      out = p.partial + (static_cast<int64_t>(blockIdx.y) * p.r_total + k0) * p.N;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i >= mblocks) break;
#pragma unroll
      for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int k = i * 16 + (lane >> 2);
          const int c = n0 + cw + 16 * g + j * 8 + q2;
          if (c < p.N) {
            if (k < r_valid) {
              out[static_cast<int64_t>(k) * p.N + c] = f * acc[i][g][j][0];
              out[static_cast<int64_t>(k) * p.N + c + 1] = f * acc[i][g][j][1];
            }
            if (k + 8 < r_valid) {
              out[static_cast<int64_t>(k + 8) * p.N + c] = f * acc[i][g][j][2];
              out[static_cast<int64_t>(k + 8) * p.N + c + 1] = f * acc[i][g][j][3];
            }
          }
        }
    }
  }
}

// Xs[i, :] = X[perm[i], :]: the plan's sorted copy of X, so every later load of a
// token tile (shrink and fused GEMM) is one TMA box instead of a row gather.
// Each thread copies 16-byte pieces; consecutive threads cover consecutive
// pieces of a row, so reads and writes are fully coalesced.
__global__ void lora_gather_rows_kernel(const uint16_t *__restrict__ X, const int32_t *__restrict__ perm,
                                        uint16_t *__restrict__ Xs, int64_t T, int64_t d) {
  pdl_launch_dependents();  // the shrink may set itself up meanwhile
  const int64_t per_row = d / 8;
  const int64_t n = T * per_row;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / per_row, c = e % per_row;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(perm[i]) * d) + c);
    reinterpret_cast<uint4 *>(Xs + i * d)[c] = v;
  }
}

// dst[t][k] = src[t][k] for k < r, 0 for r <= k < rp: a copy of an fp32 [T, r]
// matrix with rows padded to rp columns.
__global__ void lora_pad_cols_kernel(const float *__restrict__ src, int r, float *__restrict__ dst, int rp,
                                     int64_t T) {
  const int64_t n = T * rp;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = e / rp;
    const int k = static_cast<int>(e - t * rp);
    dst[e] = k < r ? src[t * r + k] : 0.f;
  }
}

// The multi-adapter backward's segments of several pieces: for each such
// segment (CTA row y = its first piece), row k < rank, column n:
// out[(pool_row + k) * N + n] = scale[adapter] * factor * sum over the
// segment's pieces, in piece order, of partial[(partial_row + k) * N + n].
__global__ void lora_reduce_pieces_kernel(const PieceDesc *__restrict__ pieces, const float *__restrict__ partial,
                                          int64_t N, const float *__restrict__ scale, float factor,
                                          float *__restrict__ out) {
  const PieceDesc pc = pieces[blockIdx.y];
  if (pc.seg_pieces == 1 || pc.first_piece != static_cast<int>(blockIdx.y)) return;
  const int64_t n = static_cast<int64_t>(pc.rank) * N;
  const float f = scale[pc.adapter] * factor;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t k = e / N, c = e - k * N;
    float s = 0.f;
    for (int q = 0; q < pc.seg_pieces; ++q) s += partial[(pieces[pc.first_piece + q].partial_row + k) * N + c];
    out[(pc.pool_row + k) * N + c] = f * s;
  }
}

// dst[i][k] = src[row(i)][k] for k < r, 0 for r <= k < rp, row(i) = perm[i] (or
// i without perm): rows of an fp32 [T, r] matrix in the plan's sorted order,
// padded to rp columns.
__global__ void lora_gather_pad_kernel(const float *__restrict__ src, int r, const int32_t *__restrict__ perm,
                                       float *__restrict__ dst, int rp, int64_t T) {
  const int64_t n = T * rp;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / rp;
    const int k = static_cast<int>(e - i * rp);
    const int64_t row = perm ? perm[i] : i;
    dst[e] = k < r ? src[row * r + k] : 0.f;
  }
}

// out[e] = factor * sum_q partial[q][e], q in order 0..splits-1.
__global__ void lora_reduce_splits_kernel(const float *__restrict__ partial, int splits, int64_t n,
                                          float factor, float *__restrict__ out) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int q = 0; q < splits; ++q) s += partial[static_cast<int64_t>(q) * n + e];
    out[e] = s * factor;
  }
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// will ever complete; the wait gives up after `limit_ns`, flags LORA_DEV_TIMEOUT
// and the kernel returns normally.
__global__ void lora_wait_selftest_kernel(uint64_t limit_ns, int *result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    *result = mbar_wait_for(smem_u32(&bar), 0, limit_ns) ? 1 : 0;
  }
}

// keep bits of the dropout mask: word t * wpr + w holds columns 32w .. 32w + 31 of
// token t (bit i set if column 32w + i is kept; bits past d_in are 0)
__global__ void lora_keep_bits_kernel(uint64_t seed, uint64_t thr, int64_t T, int64_t d_in, int64_t wpr,
                                      uint32_t *bits) {
  const int64_t n = T * wpr;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = e / wpr, w = e % wpr;
    const int64_t col0 = 32 * w;
    uint32_t m = keep_mask32(seed, thr, static_cast<uint64_t>(t * d_in + col0));
    if (d_in - col0 < 32) m &= (1u << (d_in - col0)) - 1u;
    bits[e] = m;
  }
}

__global__ void lora_mask_kernel(uint64_t seed, uint64_t thr, int64_t T, int64_t d_in, uint8_t *mask) {
  const int64_t n = T * d_in;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    mask[e] = keep_elem(seed, thr, e / d_in, e % d_in, d_in) ? 0 : 1;
}

}  // namespace lora
