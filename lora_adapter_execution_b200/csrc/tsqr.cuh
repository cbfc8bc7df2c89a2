// Batched tall-skinny QR (TSQR) for the factor construction of post-hoc LoRA
// compression: "LoRAForge：压缩与执行协同，让多LoRA服务更高效", FlashTSQR section
// (QR of many tall, skinny factor matrices at once, parallel across modules and
// across row blocks: a local QR of each row block, then the blocks' R factors
// merged). A matrix's rows are cut into leaf tiles of 128 (the last tile takes
// the remainder, up to 255 rows); one CTA factors one tile by Householder
// reflections in shared memory (fp32). Pairs of R factors are then stacked and
// factored again, level by level of a binary tree, until one R is left; its rows
// are made to have a non-negative diagonal (the unique QR of a full-rank matrix).
// Q, when wanted, goes back down the tree: the root's reflectors applied to
// [D; 0] (D the diagonal of the root's row signs), each node's to the block of
// its parent's result that belongs to it, the leaves' giving Q's rows. Each
// launch covers one level of every matrix of the batch (blockIdx.x = matrix *
// nodes + node).
#pragma once

#include "common.cuh"

namespace lora {

constexpr int kQrThreads = 256;
constexpr int kQrTile = 128;                  // rows per leaf tile
constexpr int kQrMaxN = 64;                   // columns
constexpr int kQrMaxRows = 2 * kQrTile - 1;   // the last leaf tile of a matrix

// shared memory of the two kernels for n columns (rows padded to n + 1 floats)
__host__ __device__ constexpr int qr_factor_smem(int n) { return (kQrMaxRows * (n + 1) + 3 * kQrMaxN + 16) * 4; }
__host__ __device__ constexpr int qr_apply_smem(int n) { return (2 * kQrMaxRows * (n + 1) + 3 * kQrMaxN + 16) * 4; }

// Sum of v over the CTA's 256 threads, returned to every thread (red: 8 floats).
__device__ __forceinline__ float qr_block_sum(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red is free (its previous readers are done)
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kQrThreads / 32; ++w) s += red[w];
  return s;
}

// Householder QR of a[s][ld] (s rows, n columns, s >= n), in place. Column j:
// x = a[j:, j], alpha = -sign(x_0)·||x||, v = x - alpha·e_0, tau = 2 / (v^T v);
// a[j:, c] -= tau·v·(v^T a[j:, c]) for c > j; then a[j][j] = alpha. On return the
// upper triangle holds R, column j below the diagonal holds v's entries past
// its first, vh[j] = v_0, tau[j] (0 when the column was already zero).
__device__ void qr_tile(float *a, int ld, int s, int n, float *vh, float *tau, float *w, float *red) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int j = 0; j < n; ++j) {
    float part = 0.f;
    for (int i = j + tid; i < s; i += kQrThreads) part += a[i * ld + j] * a[i * ld + j];
    const float norm2 = qr_block_sum(part, red);
    if (tid == 0) {
      const float x0 = a[j * ld + j];
      const float norm = sqrtf(norm2);
      const float alpha = x0 >= 0.f ? -norm : norm;
      const float v0 = x0 - alpha;  // x_0 + sign(x_0)·||x||: no cancellation
      const float vtv = 2.f * norm * (norm + fabsf(x0));  // v^T v, in the same form
      vh[j] = v0;
      tau[j] = vtv > 0.f ? 2.f / vtv : 0.f;
      w[kQrMaxN] = alpha;
    }
    __syncthreads();
    const float tj = tau[j], v0 = vh[j];
    // w_c = v^T a[j:, c], one warp per column (lanes over rows)
    for (int c = j + 1 + warp; c < n; c += kQrThreads / 32) {
      float sum = 0.f;
      for (int i = j + lane; i < s; i += 32) sum += (i == j ? v0 : a[i * ld + j]) * a[i * ld + c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      if (lane == 0) w[c] = sum;
    }
    __syncthreads();
    const int nc = n - j - 1;
    if (nc > 0 && tj != 0.f) {
      for (int e = tid; e < (s - j) * nc; e += kQrThreads) {
        const int i = j + e / nc, c = j + 1 + e % nc;
        a[i * ld + c] -= tj * (i == j ? v0 : a[i * ld + j]) * w[c];
      }
    }
    __syncthreads();
    if (tid == 0 && tj != 0.f) a[j * ld + j] = w[kQrMaxN];
  }
  __syncthreads();
}

// y[s][ld] <- H_0·H_1·...·H_{n-1}·y for the reflectors of qr_tile (their entries
// past the first in v[s][ld] below the diagonal), applied last one first. Only
// the first n rows of y are non-zero on entry, so H_j touches rows j .. s - 1.
__device__ void qr_apply(float *y, const float *v, int ld, int s, int n, const float *vh, const float *tau, float *w) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int j = n - 1; j >= 0; --j) {
    const float tj = tau[j], v0 = vh[j];
    if (tj == 0.f) continue;  // uniform: every thread reads the same tau
    for (int c = warp; c < n; c += kQrThreads / 32) {
      float sum = 0.f;
      for (int i = j + lane; i < s; i += 32) sum += (i == j ? v0 : v[i * ld + j]) * y[i * ld + c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      if (lane == 0) w[c] = sum;
    }
    __syncthreads();
    for (int e = tid; e < (s - j) * n; e += kQrThreads) {
      const int i = j + e / n, c = e % n;
      y[i * ld + c] -= tj * (i == j ? v0 : v[i * ld + j]) * w[c];
    }
    __syncthreads();
  }
}

// One level of the tree. Level 0's nodes are the leaf tiles of the input;
// node k of level l >= 1 stacks the R factors of nodes 2k and 2k + 1 of level
// l - 1 (one R when 2k + 1 is past that level's last node).
struct QrLevel {
  int32_t nodes;   // nodes per matrix at this level
  int32_t below;   // nodes per matrix at level - 1 (level >= 1)
  int32_t up;      // nodes per matrix at level + 1 (0: this is the root level)
  float *S;        // level >= 1: stacked pairs [batch][nodes][2n][n], row-major (reflectors after the QR)
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
  QrLevel lv;
};

// rows of leaf tile t of an m-row matrix with `leaves` tiles
__host__ __device__ inline void qr_leaf_rows(int64_t m, int leaves, int t, int64_t &r0, int &rows) {
  r0 = static_cast<int64_t>(t) * kQrTile;
  rows = t + 1 < leaves ? kQrTile : static_cast<int>(m - r0);
}
__host__ __device__ inline int qr_leaves(int64_t m) { return m < 2 * kQrTile ? 1 : static_cast<int>(m / kQrTile); }
// R factors stacked in node k of a level whose level below has `below` nodes
__host__ __device__ inline int qr_node_parts(int below, int k) { return min(2, below - 2 * k); }

// Factor one tile (leaf) or stacked pair (node). The R goes to the parent's
// stacked buffer (slot k % 2) or, at the root, to R with its rows' signs made
// non-negative on the diagonal.
__global__ void __launch_bounds__(kQrThreads) lora_qr_factor_kernel(const QrParams p) {
  extern __shared__ float qsm[];
  const int n = p.n, ld = n + 1;
  const int nodes = p.lv.nodes;
  const int k = static_cast<int>(blockIdx.x % nodes);
  const int64_t b = blockIdx.x / nodes;
  float *a = qsm;                       // [kQrMaxRows][ld]
  float *vh = a + kQrMaxRows * ld;      // [n]
  float *tau = vh + kQrMaxN;            // [n]
  float *w = tau + kQrMaxN;             // [n + 1]
  float *red = w + kQrMaxN + 4;         // [8]
  const bool want_q = p.Q != nullptr;
  int s;
  int64_t r0 = 0;
  if (p.level == 0) {
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const uint16_t *src = p.F + b * p.bstride + r0;
    for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
      const int j = e / s, i = e - j * s;
      a[i * ld + j] = __uint_as_float(static_cast<uint32_t>(__ldg(src + j * p.ld + i)) << 16);
    }
  } else {
    s = qr_node_parts(p.lv.below, k) * n;
    const float *src = p.lv.S + (b * nodes + k) * 2 * n * n;
    for (int e = threadIdx.x; e < s * n; e += kQrThreads) a[(e / n) * ld + e % n] = src[e];
  }
  __syncthreads();
  qr_tile(a, ld, s, n, vh, tau, w, red);
  if (want_q) {
    // the reflectors and their v_0, tau, for the way down
    if (p.level == 0) {
      float *dst = p.Q + b * n * p.m + r0;
      for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
        const int j = e / s, i = e - j * s;
        dst[j * p.m + i] = i > j ? a[i * ld + j] : 0.f;
      }
    } else {
      float *dst = p.lv.S + (b * nodes + k) * 2 * n * n;
      for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
        const int i = e / n, c = e % n;
        dst[e] = i > c ? a[i * ld + c] : 0.f;
      }
    }
    float *hv = p.lv.hv + (b * nodes + k) * 2 * n;
    for (int c = threadIdx.x; c < n; c += kQrThreads) {
      hv[c] = vh[c];
      hv[n + c] = tau[c];
    }
  }
  if (p.lv.up == 0) {
    // the root: R with row i negated where its diagonal is negative
    float *rdst = p.R + b * n * n;
    for (int e = threadIdx.x; e < n * n; e += kQrThreads) {
      const int i = e / n, c = e % n;
      const float d = a[i * ld + i] < 0.f ? -1.f : 1.f;
      rdst[e] = c >= i ? d * a[i * ld + c] : 0.f;
    }
    if (want_q)
      for (int i = threadIdx.x; i < n; i += kQrThreads) p.sign[b * n + i] = a[i * ld + i] < 0.f ? -1.f : 1.f;
  } else {
    float *rdst = p.lv.S_up + ((b * p.lv.up + k / 2) * 2 + (k & 1)) * n * n;
    for (int e = threadIdx.x; e < n * n; e += kQrThreads) {
      const int i = e / n, c = e % n;
      rdst[e] = c >= i ? a[i * ld + c] : 0.f;
    }
  }
}

// Going down: y = H·[C; 0] for one node (C its block of the parent's result;
// the sign diagonal at the root). Its row blocks go to the children's C or, at
// a leaf, to Q.
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
  float *w = tau + kQrMaxN;               // [n + 1]
  int s;
  int64_t r0 = 0;
  if (p.level == 0) {
    qr_leaf_rows(p.m, nodes, k, r0, s);
    const float *src = p.Q + b * n * p.m + r0;
    for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
      const int j = e / s, i = e - j * s;
      v[i * ld + j] = src[j * p.m + i];
    }
  } else {
    s = qr_node_parts(p.lv.below, k) * n;
    const float *src = p.lv.S + (b * nodes + k) * 2 * n * n;
    for (int e = threadIdx.x; e < s * n; e += kQrThreads) v[(e / n) * ld + e % n] = src[e];
  }
  const float *hv = p.lv.hv + (b * nodes + k) * 2 * n;
  for (int c = threadIdx.x; c < n; c += kQrThreads) {
    vh[c] = hv[c];
    tau[c] = hv[n + c];
  }
  const bool root = p.lv.up == 0;
  const float *cblk = root ? nullptr : p.lv.C + (b * nodes + k) * n * n;
  for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
    const int i = e / n, c = e % n;
    float val = 0.f;
    if (i < n) val = root ? (i == c ? p.sign[b * n + i] : 0.f) : cblk[i * n + c];
    y[i * ld + c] = val;
  }
  __syncthreads();
  qr_apply(y, v, ld, s, n, vh, tau, w);
  if (p.level == 0) {
    float *q = p.Q + b * n * p.m + r0;
    for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
      const int j = e / s, i = e - j * s;
      q[j * p.m + i] = y[i * ld + j];
    }
  } else {
    // row block j of the result is child 2k + j's block
    for (int e = threadIdx.x; e < s * n; e += kQrThreads) {
      const int i = e / n, c = e % n;
      p.lv.C_down[((b * p.lv.below + 2 * k + i / n) * n + i % n) * n + c] = y[i * ld + c];
    }
  }
}

}  // namespace lora
