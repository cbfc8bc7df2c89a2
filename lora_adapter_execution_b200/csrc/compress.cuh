// Post-hoc compression of adapter modules: "LoRAForge：压缩与执行协同，让多LoRA服务更高效",
// sections 核心设计 (the explicit retained-rank representation; LoRAForge-U, one
// retention ratio for every module; LoRAForge-S, a rank budget spent by each
// module's cumulative spectral energy) and FlashTSQR (the factor construction),
// with the note on spectral energy (the squared singular values).
//
// A module's update A·B (A: d_in x r, B: r x d_out) is, after the QRs
// A = Q_A·R_A and B^T = Q_B·R_B, Q_A·(R_A·R_B^T)·Q_B^T with orthonormal Q_A,
// Q_B: its singular values are those of the r x r core M = R_A·R_B^T, and its
// best rank-k approximation is A'·B' with A' = Q_A·U_k·Σ_k^½ and
// B' = Σ_k^½·V_k^T·Q_B^T (M = U·Σ·V^T). The kernels here: the core and its SVD
// per module; the rank allocation over all modules; the way-down blocks that
// make the tall-skinny QR's way down write A' and B' directly.
#pragma once

#include "common.cuh"

namespace lora {

constexpr int kSvdThreads = 256;
constexpr int kSvdMaxN = 64;
constexpr int kSvdMaxSweeps = 30;
constexpr float kSvdTol = 4e-7f;  // |w_p·w_q| / (||w_p||·||w_q||) below this: a pair is orthogonal

// shared memory: W and V [n][n + 1] each, the column norms and the sweep's largest cosine
__host__ __device__ constexpr int svd_smem(int n) { return (2 * (n + 1) * (n + 1) + 2 * kSvdMaxN + 16) * 4; }

// One module per CTA: M = R_A·R_B^T (R row-major, upper triangular), then a
// one-sided Jacobi SVD (Hestenes): column pairs (p, q) of W (starting at M)
// are rotated until orthogonal, V accumulates the rotations, so M = W·V^T at
// every step; at the end sigma_j = ||w_j||, U's column j = w_j / sigma_j. The
// pairs of a sweep follow the round-robin tournament (n - 1 rounds of n / 2
// disjoint pairs, n rounded up to even with a zero column), one warp per pair,
// the same order in every run. Outputs sorted by sigma, largest first:
// sigma [b][n], U and V [b][n][n] column-major (U[b][c][i] = row i of column c).
__global__ void __launch_bounds__(kSvdThreads) lora_core_svd_kernel(const float *__restrict__ RA,
                                                                    const float *__restrict__ RB, int n,
                                                                    float *__restrict__ sigma, float *__restrict__ U,
                                                                    float *__restrict__ V) {
  extern __shared__ float sv[];
  const int ld = n + 1;
  const int N = n + (n & 1);  // even
  float *W = sv;                  // [N][ld] (row i, column j at W[i * ld + j]); column n is the padding
  float *Vs = W + N * ld;         // [N][ld]
  float *nrm = Vs + N * ld;       // [kSvdMaxN + 1]
  float *red = nrm + kSvdMaxN + 1;  // [8]
  const int64_t b = blockIdx.x;
  const float *ra = RA + b * n * n, *rb = RB + b * n * n;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < N * N; e += kSvdThreads) {
    const int i = e / N, j = e - i * N;
    float m = 0.f;
    if (i < n && j < n)
      for (int l = max(i, j); l < n; ++l) m += ra[i * n + l] * rb[j * n + l];
    W[i * ld + j] = m;
    Vs[i * ld + j] = i == j && i < n ? 1.f : 0.f;
  }
  __syncthreads();
  for (int sweep = 0; sweep < kSvdMaxSweeps; ++sweep) {
    float worst = 0.f;
    for (int round = 0; round < N - 1; ++round) {
      for (int k = warp; k < N / 2; k += kSvdThreads / 32) {
        // tournament positions k and N - 1 - k; position 0 stays, the others rotate
        auto at = [&](int pos) { return pos == 0 ? 0 : (pos - 1 + round) % (N - 1) + 1; };
        const int pc = at(k), qc = at(N - 1 - k);
        float al = 0.f, be = 0.f, ga = 0.f;
        for (int i = lane; i < N; i += 32) {
          const float wp = W[i * ld + pc], wq = W[i * ld + qc];
          al += wp * wp;
          be += wq * wq;
          ga += wp * wq;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          al += __shfl_xor_sync(0xFFFFFFFFu, al, o);
          be += __shfl_xor_sync(0xFFFFFFFFu, be, o);
          ga += __shfl_xor_sync(0xFFFFFFFFu, ga, o);
        }
        const float den = sqrtf(al) * sqrtf(be);
        if (ga != 0.f && den > 0.f && fabsf(ga) > kSvdTol * den) {
          worst = fmaxf(worst, fabsf(ga) / den);
          const float zeta = (be - al) / (2.f * ga);
          const float t = (zeta >= 0.f ? 1.f : -1.f) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
          const float c = 1.f / sqrtf(1.f + t * t), s = c * t;
          for (int i = lane; i < N; i += 32) {
            const float wp = W[i * ld + pc], wq = W[i * ld + qc];
            W[i * ld + pc] = c * wp - s * wq;
            W[i * ld + qc] = s * wp + c * wq;
            const float vp = Vs[i * ld + pc], vq = Vs[i * ld + qc];
            Vs[i * ld + pc] = c * vp - s * vq;
            Vs[i * ld + qc] = s * vp + c * vq;
          }
        }
      }
      __syncthreads();
    }
    // the sweep's largest cosine over all warps decides (every thread the same)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xFFFFFFFFu, worst, o));
    if (lane == 0) red[warp] = worst;
    __syncthreads();
    float w = 0.f;
#pragma unroll
    for (int q = 0; q < kSvdThreads / 32; ++q) w = fmaxf(w, red[q]);
    __syncthreads();
    if (w <= kSvdTol) break;
  }
  // column norms, then each column's place in the descending order (ties by index)
  for (int j = warp; j < n; j += kSvdThreads / 32) {
    float s2 = 0.f;
    for (int i = lane; i < n; i += 32) s2 += W[i * ld + j] * W[i * ld + j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
    if (lane == 0) nrm[j] = sqrtf(s2);
  }
  __syncthreads();
  for (int j = warp; j < n; j += kSvdThreads / 32) {
    const float sj = nrm[j];
    int rank = 0;
    for (int l = 0; l < n; ++l) rank += (nrm[l] > sj || (nrm[l] == sj && l < j)) ? 1 : 0;
    if (lane == 0) sigma[b * n + rank] = sj;
    const float inv = sj > 0.f ? 1.f / sj : 0.f;
    for (int i = lane; i < n; i += 32) {
      U[(b * n + rank) * n + i] = W[i * ld + j] * inv;
      V[(b * n + rank) * n + i] = Vs[i * ld + j];
    }
  }
}

// The way-down root blocks of module b: C[b][c][i] = d[i]·X[b][c][i]·sqrt(sigma[b][c])
// for c < k[b], 0 past it (X = U for A', V for B'; d the root's row signs of
// that factor's QR, which make Q = H·[D; 0]). One thread per element.
__global__ void lora_export_roots_kernel(const float *__restrict__ X, const float *__restrict__ sigma,
                                         const float *__restrict__ sign, const int32_t *__restrict__ k,
                                         int64_t batch, int n, float *__restrict__ C) {
  const int64_t total = batch * n * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / (n * n);
    const int cw = static_cast<int>(e - b * n * n);
    const int c = cw / n, i = cw - c * n;
    C[e] = c < k[b] ? sign[b * n + i] * X[e] * sqrtf(sigma[b * n + c]) : 0.f;
  }
}

constexpr int kAllocThreads = 1024;

// Block-wide sum of an int64 over kAllocThreads threads (red: 32 slots).
__device__ __forceinline__ int64_t alloc_sum(int64_t v, int64_t *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  int64_t s = 0;
  for (int w = 0; w < kAllocThreads / 32; ++w) s += red[w];
  return s;
}

// Retained ranks of n modules, one CTA. Policy 0 (LoRAForge-U):
// k_b = clamp(ceil(keep·r_b), floor_b, r_b), floor_b = min(k_floor, r_b).
// Policy 1 (LoRAForge-S): the budget P = floor(keep·Σ r_b·c_b) parameters, c_b
// the parameters of one rank of module b; floors first; then each further rank
// i of module b scores g = (sigma_bi² / E_b) / c_b (E_b = Σ_j sigma_bj², summed
// in j order, all in float32 with no fused multiply-add, g = 0 when E_b = 0),
// and the ranks are taken largest g first (equal g: lower module, then lower
// i) while their costs fit in P - Σ floor_b·c_b, up to the first that does
// not. That order is the order of the 64-bit keys (bits of g, then the
// complement of b·r_max + i), all distinct, so the taken ranks are those with
// key >= K*, K* the smallest key whose ranks at or above it cost at most the
// rest of the budget: a radix select over the keys. Offsets: the exclusive
// prefix sum of k.
__global__ void __launch_bounds__(kAllocThreads) lora_compress_alloc_kernel(
    const float *__restrict__ sigma, const int32_t *__restrict__ ranks, const int64_t *__restrict__ costs,
    int64_t n, int r_max, int policy, double keep, int k_floor, uint64_t *__restrict__ keys,
    int32_t *__restrict__ k, int64_t *__restrict__ offsets) {
  __shared__ int64_t red[32];
  __shared__ int64_t chunk_tot[kAllocThreads];
  __shared__ int64_t whist[8 * 256];  // byte histograms of the radix select, one per 4 warps
  __shared__ int64_t hist[256];
  __shared__ int sel[1];
  __shared__ int64_t sel_above[1];
  const int tid = threadIdx.x;
  if (policy == 0) {
    for (int64_t b = tid; b < n; b += kAllocThreads) {
      const int r = ranks[b];
      const int fl = min(k_floor, r);
      k[b] = min(r, max(fl, static_cast<int>(ceil(keep * static_cast<double>(r)))));
    }
  } else {
    int64_t tot = 0, flc = 0;
    for (int64_t b = tid; b < n; b += kAllocThreads) {
      tot += static_cast<int64_t>(ranks[b]) * costs[b];
      flc += static_cast<int64_t>(min(k_floor, ranks[b])) * costs[b];
    }
    tot = alloc_sum(tot, red);
    flc = alloc_sum(flc, red);
    const int64_t budget = static_cast<int64_t>(floor(keep * static_cast<double>(tot)));
    const int64_t left = budget - flc;
    // keys of every rank past the floors (0: no such rank)
    for (int64_t b = tid; b < n; b += kAllocThreads) {
      const int r = ranks[b], fl = min(k_floor, r);
      const float *sb = sigma + b * r_max;
      float e = 0.f;
      for (int j = 0; j < r; ++j) e = __fadd_rn(e, __fmul_rn(sb[j], sb[j]));
      const float c = static_cast<float>(costs[b]);
      for (int i = 0; i < r_max; ++i) {
        uint64_t key = 0;
        if (i >= fl && i < r) {
          const float g = e > 0.f ? __fdiv_rn(__fdiv_rn(__fmul_rn(sb[i], sb[i]), e), c) : 0.f;
          key = (static_cast<uint64_t>(__float_as_uint(g)) << 32) |
                static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(b * r_max + i));
        }
        keys[b * r_max + i] = key;
      }
    }
    __syncthreads();
    // K*: the smallest key whose ranks at or above it cost at most `left`
    // (keys are never 0 for real ranks: the complement term is at least 1 while
    // b·r_max + i < 2^32 - 1). Radix select, 8 bits a pass from the top: the
    // candidates are the keys with the prefix fixed so far; a pass histograms
    // their next byte weighted by cost (a copy per 4 warps, then summed) and walks
    // the bytes from the top while the cost of the keys above still fits; the
    // byte where it stops joins the prefix. Keys are distinct, so after 8 passes
    // the prefix is the first key that does not fit, k0, and K* = k0 + 1.
    bool none = left <= 0;
    uint64_t kstar = ~0ull;
    if (!none) {
      int64_t all = 0;
      for (int64_t e = tid; e < n * r_max; e += kAllocThreads)
        if (keys[e]) all += costs[e / r_max];
      all = alloc_sum(all, red);
      if (all <= left) {
        kstar = 1;  // every rank fits
      } else {
        uint64_t prefix = 0;
        int64_t above = 0;  // cost of the keys above the current prefix's range
        for (int pass = 0; pass < 8; ++pass) {
          const int shift = 56 - 8 * pass;
          for (int e = tid; e < 8 * 256; e += kAllocThreads) whist[e] = 0;
          __syncthreads();
          unsigned long long *wh = reinterpret_cast<unsigned long long *>(whist) + (tid >> 7) * 256;
          for (int64_t e = tid; e < n * r_max; e += kAllocThreads) {
            const uint64_t key = keys[e];
            if (!key) continue;
            // the fixed bytes match (pass 0: everything)
            if (pass > 0 && (key >> (shift + 8)) != prefix) continue;
            atomicAdd(wh + ((key >> shift) & 0xFF), static_cast<unsigned long long>(costs[e / r_max]));
          }
          __syncthreads();
          if (tid < 256) {
            int64_t s = 0;
            for (int w = 0; w < 8; ++w) s += whist[w * 256 + tid];
            hist[tid] = s;
          }
          __syncthreads();
          if (tid == 0) {
            int64_t acc = above;
            int d = 255;
            for (; d > 0; --d) {
              if (acc + hist[d] > left) break;
              acc += hist[d];
            }
            sel[0] = d;
            sel_above[0] = acc;
          }
          __syncthreads();
          prefix = (prefix << 8) | static_cast<uint64_t>(sel[0]);
          above = sel_above[0];
          __syncthreads();
        }
        kstar = prefix + 1;
      }
    }
    for (int64_t b = tid; b < n; b += kAllocThreads) {
      const int r = ranks[b];
      int kb = min(k_floor, r);
      if (!none)
        for (int i = 0; i < r_max; ++i) {
          const uint64_t key = keys[b * r_max + i];
          if (key && key >= kstar) ++kb;
        }
      k[b] = kb;
    }
  }
  __syncthreads();
  // offsets: each thread sums a contiguous chunk, thread 0 scans the chunk totals
  const int64_t per = (n + kAllocThreads - 1) / kAllocThreads;
  const int64_t b0 = tid * per, b1 = min(n, b0 + per);
  int64_t s = 0;
  for (int64_t b = b0; b < b1; ++b) s += k[b];
  chunk_tot[tid] = s;
  __syncthreads();
  if (tid == 0) {
    int64_t run = 0;
    for (int t = 0; t < kAllocThreads; ++t) {
      const int64_t v = chunk_tot[t];
      chunk_tot[t] = run;
      run += v;
    }
    offsets[n] = run;
  }
  __syncthreads();
  s = chunk_tot[tid];
  for (int64_t b = b0; b < b1; ++b) {
    offsets[b] = s;
    s += k[b];
  }
}

}  // namespace lora
