// Batched tall-skinny QR (TSQR) for the factor construction of post-hoc LoRA
// compression: "LoRAForge：压缩与执行协同，让多LoRA服务更高效", FlashTSQR section
// (QR of many tall, skinny factor matrices at once, parallel across modules and
// across row blocks: a local QR of each row block, then the blocks' R factors
// merged). A matrix's rows are cut into leaf tiles of 128 (the last one takes
// the rest); each tile is factored by Householder reflections in fp32. Pairs of
// R factors are then stacked and factored again, level by level of a binary
// tree, until one R is left; its rows are made to have a non-negative diagonal
// (the unique QR of a full-rank matrix). Q, when wanted, goes back down the
// tree: the root's reflectors applied to [D; 0] (D the diagonal of the root's
// row signs), each node's to the block of its parent's result that belongs to
// it, the leaves' giving Q's rows. Each launch covers one level of every matrix
// of the batch.
//
// Two builds of the per-node work. For n <= 32 one warp owns a node: row
// i = 32·r + lane of the tile sits in register a[r][·] of that lane, so column
// norms and the dot products v^T·a_c are warp reductions (shuffles) and nothing
// waits on a block barrier. For 32 < n <= 64 one CTA owns a node, the tile in
// shared memory.
//
// Tree buffers are column-major: a stacked pair of node k is S[c][i] (c < n,
// i < 2n: rows of child 2k, then of child 2k + 1), a block of the way down
// C[c][i] (n x n), so that the lanes (rows) of a warp touch consecutive words.
#pragma once

#include "common.cuh"

namespace lora {

constexpr int kQrTile = 128;       // rows per leaf tile
constexpr int kQrMaxN = 64;        // columns
constexpr int kQrWarpMaxN = 32;    // the warp build's limit
constexpr int kQrWarpThreads = 128;  // 4 nodes per CTA in the warp build
constexpr int kQrThreads = 256;    // the CTA build
constexpr int kQrMaxRows = 128;    // rows of any node (a leaf, or two stacked R of n <= 64)

// shared memory of the CTA build's two kernels for n columns (rows padded to n + 1 floats)
__host__ __device__ constexpr int qr_factor_smem(int n) { return (kQrMaxRows * (n + 1) + 3 * kQrMaxN + 16) * 4; }
__host__ __device__ constexpr int qr_apply_smem(int n) { return (2 * kQrMaxRows * (n + 1) + 3 * kQrMaxN + 16) * 4; }

// One level of the tree. Level 0's nodes are the leaf tiles of the input;
// node k of level l >= 1 stacks the R factors of nodes 2k and 2k + 1 of level
// l - 1 (one R when 2k + 1 is past that level's last node).
struct QrLevel {
  int32_t nodes;   // nodes per matrix at this level
  int32_t below;   // nodes per matrix at level - 1 (level >= 1)
  int32_t up;      // nodes per matrix at level + 1 (0: this is the root level)
  float *S;        // level >= 1: stacked pairs [batch][nodes][n][2n] (reflectors after the QR)
  float *S_up;     // the next level's S
  float *hv;       // [batch][nodes][2][n]: v_0 and tau of each node's reflectors (Q wanted)
  float *C;        // down pass: [batch][nodes][n][n], each node's block of its parent's result
  float *C_down;   // the level below's C (level >= 1)
};

struct QrParams {
  int64_t batch, m;
  int32_t n, level;
  int64_t ld, bstride;  // input: element (i, j) of matrix b at F[b * bstride + j * ld + i]
  const uint16_t *F;    // bf16 factors, column-major (column j = an adapter pool's row)
  float *Q;             // [batch][n][m] fp32 column-major (NULL: R only); holds the leaves' reflectors in between
  float *R;             // [batch][n][n] row-major, upper triangular, diagonal >= 0
  float *sign;          // [batch][n]: the root's row signs (Q wanted)
  // way down only: the root's block, [batch][n][n] column-major (NULL: the sign
  // diagonal, giving Q); with it the leaves give Q·(that block's leading rows)
  const float *root_c;
  // way down only: the leaves write columns c < out_k[b] of their result as
  // bf16 rows out_row0[b] + c of out_rows (row length m) instead of Q
  uint16_t *out_rows;
  const int32_t *out_k;
  const int64_t *out_row0;
  QrLevel lv;
};

__host__ __device__ inline int qr_leaves(int64_t m) { return static_cast<int>((m + kQrTile - 1) / kQrTile); }
// rows of leaf tile t of an m-row matrix with `leaves` tiles
__host__ __device__ inline void qr_leaf_rows(int64_t m, int leaves, int t, int64_t &r0, int &rows) {
  r0 = static_cast<int64_t>(t) * kQrTile;
  rows = t + 1 < leaves ? kQrTile : static_cast<int>(m - r0);
}
// R factors stacked in node k of a level whose level below has `below` nodes
__host__ __device__ inline int qr_node_parts(int below, int k) { return min(2, below - 2 * k); }

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Householder step quantities of a column x (x_0 its diagonal entry, ||x||^2 =
// norm2): alpha = -sign(x_0)·||x||, v_0 = x_0 - alpha = x_0 + sign(x_0)·||x||,
// tau = 2 / (v^T v) with v^T v = 2·||x||·(||x|| + |x_0|) (no cancellation);
// tau = 0 for a zero column.
__device__ __forceinline__ void householder(float x0, float norm2, float &alpha, float &v0, float &tau) {
  const float norm = sqrtf(norm2);
  alpha = x0 >= 0.f ? -norm : norm;
  v0 = x0 - alpha;
  const float vtv = 2.f * norm * (norm + fabsf(x0));
  tau = vtv > 0.f ? 2.f / vtv : 0.f;
}

// ------------------------------------------------------------------ warp build (n <= 32)
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// x[c] <- sum over the warp's lanes of x[c], for every c (NV a power of two,
// 2 <= NV <= 32). Recursive halving: at the step with lane mask m each lane
// keeps half of its values, adds its partner's copy of that half and drops the
// other (NV - 1 shuffles in all); the lanes then finish their single value with
// the remaining masks, and every lane gathers the NV totals from the lanes
// that hold them (NV shuffles) - about 2·NV shuffles against 5·NV for one
// butterfly per value.
template <int NV>
__device__ __forceinline__ void warp_allreduce(float (&x)[NV]) {
  static_assert(NV >= 2 && NV <= 32 && (NV & (NV - 1)) == 0, "NV: a power of two in 2..32");
  constexpr int kSteps = NV == 2 ? 1 : NV == 4 ? 2 : NV == 8 ? 3 : NV == 16 ? 4 : 5;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < kSteps; ++t) {
    const int m = 16 >> t;
    const int half = NV >> (t + 1);  // values kept after this step
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? x[i] : x[i + half];
      const float keep = upper ? x[i + half] : x[i];
      x[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, m);
    }
  }
  float v = x[0];
#pragma unroll
  for (int m = 16 >> kSteps; m > 0; m >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, m);
  // lane L now holds the total of column L >> (5 - kSteps)
#pragma unroll
  for (int c = 0; c < NV; ++c) x[c] = __shfl_sync(0xFFFFFFFFu, v, c << (5 - kSteps));
}

// Householder QR of the warp's tile, in place: rows i = 32·r + lane (zero past
// the node's rows), columns c < n <= NC. On return a[·][c] holds R in the
// rows i <= c and the reflector's entries past its first in the rows i > c;
// v_0 and tau of column c (as in `householder`) go to hv[c] and hv[n + c] when
// hv is not null (stored by lane c at once, so they hold no registers).
template <int NC, int RPL>
__device__ __forceinline__ void warp_qr(float (&a)[RPL][NC], int n, float *hv) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    if (j >= n) continue;  // uniform
    if (j >= 32 * RPL) {   // a column past the node's rows: nothing to reflect
      if (hv && lane == j % 32) {
        hv[j] = 0.f;
        hv[n + j] = 0.f;
      }
      continue;
    }
    float part = 0.f;
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      const float x = 32 * r + lane >= j ? a[r][j] : 0.f;
      part += x * x;
    }
    const float norm2 = warp_sum(part);
    const float x0 = __shfl_sync(0xFFFFFFFFu, a[j / 32][j], j % 32);
    float alpha, v0, t;
    householder(x0, norm2, alpha, v0, t);
    if (hv && lane == j % 32) {
      hv[j] = v0;
      hv[n + j] = t;
    }
    if (t == 0.f) continue;  // uniform
    float v[RPL];
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      const int i = 32 * r + lane;
      v[r] = i > j ? a[r][j] : (i == j ? v0 : 0.f);
    }
    // w_c = v^T a_c for the columns after j (the others reduce zeros)
    float w[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float s = 0.f;
      if (c > j) {
#pragma unroll
        for (int r = 0; r < RPL; ++r) s += v[r] * a[r][c];
      }
      w[c] = s;
    }
    warp_allreduce<NC>(w);
#pragma unroll
    for (int c = j + 1; c < NC; ++c) {
#pragma unroll
      for (int r = 0; r < RPL; ++r) a[r][c] -= t * v[r] * w[c];
    }
    if (lane == j % 32) a[j / 32][j] = alpha;
  }
}

// After a node's tile is in registers: its QR, the reflectors and their v_0,
// tau for the way down (Q wanted), and its R (to the parent's stacked pair, or
// at the root with a non-negative diagonal).
template <int NC, int RPL>
__device__ __forceinline__ void warp_factor_node(const QrParams &p, float (&a)[RPL][NC], int64_t b, int k, int64_t r0,
                                                 int s) {
  const int lane = threadIdx.x & 31;
  const int nodes = p.lv.nodes;
  const int n = p.n;
  const bool want_q = p.Q != nullptr;
  warp_qr<NC, RPL>(a, n, want_q ? p.lv.hv + (b * nodes + k) * 2 * n : nullptr);
  if (want_q) {
    // the reflectors (entries below the diagonal) and their v_0, tau
    float *dst;
    int64_t cstride;
    if (p.level == 0) {
      dst = p.Q + b * n * p.m + r0;
      cstride = p.m;
    } else {
      dst = p.lv.S + (b * nodes + k) * 2 * n * n;
      cstride = 2 * n;
    }
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int i = 32 * r + lane;
        if (c < n && i < s) dst[c * cstride + i] = i > c ? a[r][c] : 0.f;
      }
  }
  // R: rows i < n <= 32 are rows of register group 0, row i in lane i
  if (lane < n) {
    float diag = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (c == lane) diag = a[0][c];
    if (p.lv.up == 0) {
      const float d = diag < 0.f ? -1.f : 1.f;
      float *rrow = p.R + b * n * n + lane * n;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (c < n) rrow[c] = c >= lane ? d * a[0][c] : 0.f;
      if (want_q) p.sign[b * n + lane] = d;
    } else {
      float *dst = p.lv.S_up + (b * p.lv.up + k / 2) * 2 * n * n + (k & 1) * n + lane;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (c < n) dst[c * 2 * n] = c >= lane ? a[0][c] : 0.f;
    }
  }
}

// Factor the nodes of one level, one warp per node (blockIdx.x · 4 + warp =
// matrix · nodes + node).
template <int NC, int RPL>
__global__ void __launch_bounds__(kQrWarpThreads, NC * RPL > 64 ? 2 : 4) lora_qr_factor_warp_kernel(const QrParams p) {
  const int lane = threadIdx.x & 31;
  const int nodes = p.lv.nodes;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * (kQrWarpThreads / 32) + (threadIdx.x >> 5);
  if (g >= p.batch * nodes) return;  // uniform per warp
  const int64_t b = g / nodes;
  const int k = static_cast<int>(g - b * nodes);
  const int n = p.n;
  float a[RPL][NC];
  int s;
  int64_t r0 = 0;
  if (p.level == 0) {
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const uint16_t *src = p.F + b * p.bstride + r0;
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int i = 32 * r + lane;
        a[r][c] = (c < n && i < s) ? bf16_to_f32(__ldg(src + c * p.ld + i)) : 0.f;
      }
  } else {
    s = qr_node_parts(p.lv.below, k) * n;
    const float *src = p.lv.S + (b * nodes + k) * 2 * n * n;
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int i = 32 * r + lane;
        a[r][c] = (c < n && i < s) ? src[c * 2 * n + i] : 0.f;
      }
  }
  warp_factor_node<NC, RPL>(p, a, b, k, r0, s);
}

// 16-byte copy global -> shared that does not wait (cp.async, L2 only), reading
// src_bytes (0 .. 16) and zero-filling the rest; a commit closes a group, and
// wait<N> returns once at most N of this thread's groups are in flight.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The leaf level, persistent: each warp takes leaves g, g + (all warps), ... and
// copies the next leaf's tile (bf16, [NC columns][128 rows], zero past the
// matrix's rows) into the other half of its shared-memory buffer while it
// factors the current one, so the tile loads no longer stall the warp.
// Needs 16-byte aligned rows: F, ld and bstride multiples of 8 elements.
template <int NC>
__host__ __device__ constexpr int qr_leaf_factor_smem() { return (kQrWarpThreads / 32) * 2 * NC * kQrTile * 2; }
template <int NC>
__global__ void __launch_bounds__(kQrWarpThreads, NC > 16 ? 2 : 4) lora_qr_factor_leaf_kernel(const QrParams p) {
  extern __shared__ __align__(16) uint8_t qlf[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint16_t *buf = reinterpret_cast<uint16_t *>(qlf) + wid * 2 * NC * kQrTile;
  const int nodes = p.lv.nodes, n = p.n;
  const int64_t total = p.batch * nodes;
  const int64_t step = static_cast<int64_t>(gridDim.x) * (kQrWarpThreads / 32);
  int64_t g = static_cast<int64_t>(blockIdx.x) * (kQrWarpThreads / 32) + wid;
  // chunk q of a tile: column q / 16, rows 8·(q % 16) .. + 7
  auto issue = [&](int64_t gg, int st) {
    const int64_t b = gg / nodes;
    const int k = static_cast<int>(gg - b * nodes);
    int64_t r0;
    int s;
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const uint16_t *src = p.F + b * p.bstride + r0;
    uint16_t *dst = buf + st * NC * kQrTile;
#pragma unroll
    for (int t = 0; t < NC / 2; ++t) {
      const int q = t * 32 + lane, c = q >> 4, r8 = (q & 15) * 8;
      const int valid = c < n ? max(0, min(8, s - r8)) : 0;
      cp_async16(dst + c * kQrTile + r8, valid > 0 ? static_cast<const void *>(src + c * p.ld + r8) : p.F,
                 valid * 2);
    }
    cp_async_commit();
  };
  if (g < total) issue(g, 0);
  for (int st = 0; g < total; g += step, st ^= 1) {
    if (g + step < total) issue(g + step, st ^ 1);
    else cp_async_commit();  // an empty group: the wait below still means "this tile is in"
    cp_async_wait<1>();
    __syncwarp();
    const int64_t b = g / nodes;
    const int k = static_cast<int>(g - b * nodes);
    int64_t r0;
    int s;
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const uint16_t *t = buf + st * NC * kQrTile;
    float a[4][NC];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) a[r][c] = c < n ? bf16_to_f32(t[c * kQrTile + 32 * r + lane]) : 0.f;
    __syncwarp();  // the buffer half is read: the next issue may refill it
    warp_factor_node<NC, 4>(p, a, b, k, r0, s);
  }
  cp_async_wait<0>();
}

// The way down's start for one node: y = [C; 0] with C the node's block of its
// parent's result (at the root: the root block when given, else the sign
// diagonal), rows i = 32·r + lane.
template <int NC, int RPL>
__device__ __forceinline__ void warp_apply_init(const QrParams &p, float (&y)[RPL][NC], int64_t b, int k) {
  const int lane = threadIdx.x & 31;
  const int n = p.n, nodes = p.lv.nodes;
#pragma unroll
  for (int r = 0; r < RPL; ++r)
#pragma unroll
    for (int c = 0; c < NC; ++c) y[r][c] = 0.f;
  if (lane < n) {
    if (p.lv.up == 0 && p.root_c) {
      const float *cb = p.root_c + b * n * n + lane;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (c < n) y[0][c] = cb[c * n];
    } else if (p.lv.up == 0) {
      const float d = p.sign[b * n + lane];
#pragma unroll
      for (int c = 0; c < NC; ++c) y[0][c] = c == lane ? d : 0.f;
    } else {
      const float *cb = p.lv.C + (b * nodes + k) * n * n + lane;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (c < n) y[0][c] = cb[c * n];
    }
  }
}

// The way down's end for one node: a leaf writes its rows of Q (or the export's
// bf16 rows), an inner node its row blocks into the children's C.
template <int NC, int RPL>
__device__ __forceinline__ void warp_apply_store(const QrParams &p, const float (&y)[RPL][NC], int64_t b, int k,
                                                 int64_t r0, int s) {
  const int lane = threadIdx.x & 31;
  const int n = p.n;
  if (p.level == 0 && p.out_rows) {
    const int kb = min(p.out_k[b], n);
    uint16_t *o = p.out_rows + p.out_row0[b] * p.m + r0;
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int i = 32 * r + lane;
        if (c < kb && i < s) o[c * p.m + i] = f32_to_bf16_rn(y[r][c]);
      }
  } else if (p.level == 0) {
    float *q = p.Q + b * n * p.m + r0;
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int i = 32 * r + lane;
        if (c < n && i < s) q[c * p.m + i] = y[r][c];
      }
  } else {
    // row i of y is row i % n of child 2k + i / n's block
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      const int i = 32 * r + lane;
      if (i >= s) continue;
      const int child = 2 * k + i / n, ri = i % n;
      float *cb = p.lv.C_down + (b * p.lv.below + child) * n * n + ri;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (c < n) cb[c * n] = y[r][c];
    }
  }
}

// Going down, one warp per node: y = H_0·...·H_{n-1}·[C; 0] (C the node's block
// of its parent's result, the sign diagonal at the root), the reflectors read
// column by column from where the factor pass stored them. The row blocks of y
// go to the children's C or, at a leaf, to Q.
template <int NC, int RPL>
__global__ void __launch_bounds__(kQrWarpThreads, NC * RPL > 64 ? 2 : 4) lora_qr_apply_warp_kernel(const QrParams p) {
  const int lane = threadIdx.x & 31;
  const int nodes = p.lv.nodes;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * (kQrWarpThreads / 32) + (threadIdx.x >> 5);
  if (g >= p.batch * nodes) return;
  const int64_t b = g / nodes;
  const int k = static_cast<int>(g - b * nodes);
  const int n = p.n;
  int s;
  int64_t r0 = 0;
  const float *vsrc;
  int64_t cstride;
  if (p.level == 0) {
    qr_leaf_rows(p.m, nodes, k, r0, s);
    vsrc = p.Q + b * n * p.m + r0;
    cstride = p.m;
  } else {
    s = qr_node_parts(p.lv.below, k) * n;
    vsrc = p.lv.S + (b * nodes + k) * 2 * n * n;
    cstride = 2 * n;
  }
  const float *hv = p.lv.hv + (b * nodes + k) * 2 * n;
  float y[RPL][NC];
  warp_apply_init<NC, RPL>(p, y, b, k);
#pragma unroll
  for (int j = NC - 1; j >= 0; --j) {
    if (j >= n) continue;  // uniform
    const float t = hv[n + j];
    if (t == 0.f) continue;  // uniform
    const float v0 = hv[j];
    float v[RPL];
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      const int i = 32 * r + lane;
      v[r] = (i > j && i < s) ? vsrc[j * cstride + i] : (i == j ? v0 : 0.f);
    }
    float w[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < RPL; ++r) sum += v[r] * y[r][c];
      w[c] = sum;
    }
    warp_allreduce<NC>(w);
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
      for (int r = 0; r < RPL; ++r) y[r][c] -= t * v[r] * w[c];
  }
  warp_apply_store<NC, RPL>(p, y, b, k, r0, s);
}

// The way down's leaf level, persistent: each warp takes leaves g, g + (all
// warps), ... and copies the next leaf's reflectors (fp32, [NC columns][128
// rows] of Q's buffer, zero past the matrix's rows) into the other half of its
// shared-memory buffer while it applies the current ones; the leaf's v_0 and tau
// are read once per leaf, lane c holding column c's, and passed out by shuffle.
// Needs m a multiple of 4 (16-byte rows of Q's buffer).
template <int NC>
__host__ __device__ constexpr int qr_leaf_apply_smem() { return (kQrWarpThreads / 32) * 2 * NC * kQrTile * 4; }
template <int NC>
__global__ void __launch_bounds__(kQrWarpThreads, 3) lora_qr_apply_leaf_kernel(const QrParams p) {
  extern __shared__ __align__(16) uint8_t qla[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float *buf = reinterpret_cast<float *>(qla) + wid * 2 * NC * kQrTile;
  const int nodes = p.lv.nodes, n = p.n;
  const int64_t total = p.batch * nodes;
  const int64_t step = static_cast<int64_t>(gridDim.x) * (kQrWarpThreads / 32);
  int64_t g = static_cast<int64_t>(blockIdx.x) * (kQrWarpThreads / 32) + wid;
  // chunk q of a tile: column q / 32, rows 4·(q % 32) .. + 3
  auto issue = [&](int64_t gg, int st) {
    const int64_t b = gg / nodes;
    const int k = static_cast<int>(gg - b * nodes);
    int64_t r0;
    int s;
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const float *src = p.Q + b * n * p.m + r0;
    float *dst = buf + st * NC * kQrTile;
#pragma unroll
    for (int t = 0; t < NC; ++t) {
      const int q = t * 32 + lane, c = q >> 5, r4 = (q & 31) * 4;
      const int valid = c < n ? max(0, min(4, s - r4)) : 0;
      cp_async16(dst + c * kQrTile + r4, valid > 0 ? static_cast<const void *>(src + c * p.m + r4) : p.Q, valid * 4);
    }
    cp_async_commit();
  };
  if (g < total) issue(g, 0);
  for (int st = 0; g < total; g += step, st ^= 1) {
    if (g + step < total) issue(g + step, st ^ 1);
    else cp_async_commit();  // an empty group: the wait below still means "this tile is in"
    const int64_t b = g / nodes;
    const int k = static_cast<int>(g - b * nodes);
    int64_t r0;
    int s;
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const float *hv = p.lv.hv + (b * nodes + k) * 2 * n;
    const float my_v0 = lane < n ? hv[lane] : 0.f, my_tau = lane < n ? hv[n + lane] : 0.f;
    float y[4][NC];
    warp_apply_init<NC, 4>(p, y, b, k);
    cp_async_wait<1>();
    __syncwarp();
    const float *t = buf + st * NC * kQrTile;
#pragma unroll
    for (int j = NC - 1; j >= 0; --j) {
      if (j >= n) continue;  // uniform
      const float tj = __shfl_sync(0xFFFFFFFFu, my_tau, j);
      if (tj == 0.f) continue;  // uniform
      const float v0 = __shfl_sync(0xFFFFFFFFu, my_v0, j);
      float v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = 32 * r + lane;
        v[r] = i > j ? t[j * kQrTile + i] : (i == j ? v0 : 0.f);
      }
      float w[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) sum += v[r] * y[r][c];
        w[c] = sum;
      }
      warp_allreduce<NC>(w);
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int r = 0; r < 4; ++r) y[r][c] -= tj * v[r] * w[c];
    }
    __syncwarp();  // the buffer half is read: the next issue may refill it
    warp_apply_store<NC, 4>(p, y, b, k, r0, s);
  }
  cp_async_wait<0>();
}

// ------------------------------------------------------------------ CTA build (32 < n <= 64)
// Sum of v over the CTA's 256 threads, returned to every thread (red: 8 floats).
__device__ __forceinline__ float qr_block_sum(float v, float *red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red is free (its previous readers are done)
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kQrThreads / 32; ++w) s += red[w];
  return s;
}

// Householder QR of a[rows][ld] (rows >= n, zero past the node's own rows), in
// place, with the same output convention as warp_qr. Warps take rows, lanes
// columns in the updates (no index division); one warp per column in the dot
// products.
__device__ void qr_tile(float *a, int ld, int rows, int n, float *vh, float *tau, float *w, float *red) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int j = 0; j < n; ++j) {
    float part = 0.f;
    for (int i = j + tid; i < rows; i += kQrThreads) part += a[i * ld + j] * a[i * ld + j];
    const float norm2 = qr_block_sum(part, red);
    const float x0 = a[j * ld + j];
    float alpha, v0, tj;
    householder(x0, norm2, alpha, v0, tj);
    if (tid == 0) {
      vh[j] = v0;
      tau[j] = tj;
    }
    if (tj != 0.f) {  // uniform
      // w_c = v^T a[j:, c], one warp per column (lanes over rows)
      for (int c = j + 1 + warp; c < n; c += kQrThreads / 32) {
        float sum = 0.f;
        for (int i = j + lane; i < rows; i += 32) sum += (i == j ? v0 : a[i * ld + j]) * a[i * ld + c];
        sum = warp_sum(sum);
        if (lane == 0) w[c] = sum;
      }
      __syncthreads();
      for (int i = j + warp; i < rows; i += kQrThreads / 32) {
        const float vi = i == j ? v0 : a[i * ld + j];
        for (int c = j + 1 + lane; c < n; c += 32) a[i * ld + c] -= tj * vi * w[c];
      }
      __syncthreads();
      if (tid == 0) a[j * ld + j] = alpha;
    }
    __syncthreads();
  }
}

// y[rows][ld] <- H_0·H_1·...·H_{n-1}·y for qr_tile's reflectors (entries below
// the diagonal of v[rows][ld]), applied last one first.
__device__ void qr_apply(float *y, const float *v, int ld, int rows, int n, const float *vh, const float *tau,
                         float *w) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int j = n - 1; j >= 0; --j) {
    const float tj = tau[j], v0 = vh[j];
    if (tj == 0.f) continue;  // uniform: every thread reads the same tau
    for (int c = warp; c < n; c += kQrThreads / 32) {
      float sum = 0.f;
      for (int i = j + lane; i < rows; i += 32) sum += (i == j ? v0 : v[i * ld + j]) * y[i * ld + c];
      sum = warp_sum(sum);
      if (lane == 0) w[c] = sum;
    }
    __syncthreads();
    for (int i = j + warp; i < rows; i += kQrThreads / 32) {
      const float vi = i == j ? v0 : v[i * ld + j];
      for (int c = lane; c < n; c += 32) y[i * ld + c] -= tj * vi * w[c];
    }
    __syncthreads();
  }
}

// Factor one node per CTA (blockIdx.x = matrix · nodes + node).
__global__ void __launch_bounds__(kQrThreads) lora_qr_factor_kernel(const QrParams p) {
  extern __shared__ float qsm[];
  const int n = p.n, ld = n + 1;
  const int nodes = p.lv.nodes;
  const int k = static_cast<int>(blockIdx.x % nodes);
  const int64_t b = blockIdx.x / nodes;
  float *a = qsm;                       // [kQrMaxRows][ld]
  float *vh = a + kQrMaxRows * ld;      // [n]
  float *tau = vh + kQrMaxN;            // [n]
  float *w = tau + kQrMaxN;             // [n]
  float *red = w + kQrMaxN + 4;         // [8]
  const bool want_q = p.Q != nullptr;
  int s;
  int64_t r0 = 0;
  if (p.level == 0) qr_leaf_rows(p.m, nodes, k, r0, s);
  else s = qr_node_parts(p.lv.below, k) * n;
  const int rows = max(s, n);  // a short last leaf is padded with zero rows
  if (p.level == 0) {
    const uint16_t *src = p.F + b * p.bstride + r0;
    for (int c = 0; c < n; ++c)
      for (int i = threadIdx.x; i < rows; i += kQrThreads)
        a[i * ld + c] = i < s ? bf16_to_f32(__ldg(src + c * p.ld + i)) : 0.f;
  } else {
    const float *src = p.lv.S + (b * nodes + k) * 2 * n * n;
    for (int c = 0; c < n; ++c)
      for (int i = threadIdx.x; i < rows; i += kQrThreads) a[i * ld + c] = src[c * 2 * n + i];
  }
  __syncthreads();
  qr_tile(a, ld, rows, n, vh, tau, w, red);
  if (want_q) {
    float *dst;
    int64_t cstride;
    if (p.level == 0) {
      dst = p.Q + b * n * p.m + r0;
      cstride = p.m;
    } else {
      dst = p.lv.S + (b * nodes + k) * 2 * n * n;
      cstride = 2 * n;
    }
    for (int c = 0; c < n; ++c)
      for (int i = threadIdx.x; i < s; i += kQrThreads) dst[c * cstride + i] = i > c ? a[i * ld + c] : 0.f;
    float *hv = p.lv.hv + (b * nodes + k) * 2 * n;
    for (int c = threadIdx.x; c < n; c += kQrThreads) {
      hv[c] = vh[c];
      hv[n + c] = tau[c];
    }
  }
  if (p.lv.up == 0) {
    float *rdst = p.R + b * n * n;
    for (int i = 0; i < n; ++i) {
      const float d = a[i * ld + i] < 0.f ? -1.f : 1.f;
      for (int c = threadIdx.x; c < n; c += kQrThreads) rdst[i * n + c] = c >= i ? d * a[i * ld + c] : 0.f;
    }
    if (want_q)
      for (int i = threadIdx.x; i < n; i += kQrThreads) p.sign[b * n + i] = a[i * ld + i] < 0.f ? -1.f : 1.f;
  } else {
    float *dst = p.lv.S_up + (b * p.lv.up + k / 2) * 2 * n * n + (k & 1) * n;
    for (int c = 0; c < n; ++c)
      for (int i = threadIdx.x; i < n; i += kQrThreads) dst[c * 2 * n + i] = c >= i ? a[i * ld + c] : 0.f;
  }
}

// Going down, one node per CTA.
__global__ void __launch_bounds__(kQrThreads) lora_qr_apply_kernel(const QrParams p) {
  extern __shared__ float qsm[];
  const int n = p.n, ld = n + 1;
  const int nodes = p.lv.nodes;
  const int k = static_cast<int>(blockIdx.x % nodes);
  const int64_t b = blockIdx.x / nodes;
  float *y = qsm;                         // [kQrMaxRows][ld]
  float *v = y + kQrMaxRows * ld;         // [kQrMaxRows][ld]
  float *vh = v + kQrMaxRows * ld;        // [n]
  float *tau = vh + kQrMaxN;              // [n]
  float *w = tau + kQrMaxN;               // [n]
  int s;
  int64_t r0 = 0;
  const float *vsrc;
  int64_t cstride;
  if (p.level == 0) {
    qr_leaf_rows(p.m, nodes, k, r0, s);
    vsrc = p.Q + b * n * p.m + r0;
    cstride = p.m;
  } else {
    s = qr_node_parts(p.lv.below, k) * n;
    vsrc = p.lv.S + (b * nodes + k) * 2 * n * n;
    cstride = 2 * n;
  }
  const int rows = max(s, n);
  for (int c = 0; c < n; ++c)
    for (int i = threadIdx.x; i < rows; i += kQrThreads) v[i * ld + c] = i < s ? vsrc[c * cstride + i] : 0.f;
  const float *hv = p.lv.hv + (b * nodes + k) * 2 * n;
  for (int c = threadIdx.x; c < n; c += kQrThreads) {
    vh[c] = hv[c];
    tau[c] = hv[n + c];
  }
  const bool root = p.lv.up == 0;
  const float *cblk = root ? nullptr : p.lv.C + (b * nodes + k) * n * n;
  for (int c = 0; c < n; ++c)
    for (int i = threadIdx.x; i < rows; i += kQrThreads) {
      float val = 0.f;
      if (i < n)
        val = !root ? cblk[c * n + i] : p.root_c ? p.root_c[b * n * n + c * n + i] : (i == c ? p.sign[b * n + i] : 0.f);
      y[i * ld + c] = val;
    }
  __syncthreads();
  qr_apply(y, v, ld, rows, n, vh, tau, w);
  if (p.level == 0 && p.out_rows) {
    uint16_t *o = p.out_rows + p.out_row0[b] * p.m + r0;
    for (int c = 0; c < min(p.out_k[b], n); ++c)
      for (int i = threadIdx.x; i < s; i += kQrThreads) o[c * p.m + i] = f32_to_bf16_rn(y[i * ld + c]);
  } else if (p.level == 0) {
    float *q = p.Q + b * n * p.m + r0;
    for (int c = 0; c < n; ++c)
      for (int i = threadIdx.x; i < s; i += kQrThreads) q[c * p.m + i] = y[i * ld + c];
  } else {
    for (int c = 0; c < n; ++c)
      for (int i = threadIdx.x; i < s; i += kQrThreads)
        p.lv.C_down[(b * p.lv.below + 2 * k + i / n) * n * n + c * n + i % n] = y[i * ld + c];
  }
}

}  // namespace lora
