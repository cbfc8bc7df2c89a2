/*
 * CPU oracle for the heterogeneous multi-adapter LoRA linear layer.
 *
 * TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg load this file's library; the product path never does.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Everything is plain loops in fp64 over bf16 inputs widened exactly, in the
 * order the definitions below state, with no blocking or fusion. OpenMP only
 * splits independent outputs (rows or columns) across threads; every single
 * output is summed in the same sequential order regardless of thread count.
 *
 * Definitions followed (page titles as published):
 *  - LoRA reparameterisation, Y = X·W + X·(A·B), A in R^{d x r}, B in R^{r x k},
 *    W frozen: "LoRAFusion：消除冗余内存访问的多 LoRA 高效微调系统",
 *    section 解决什么真问题 (what problem it solves), item 1.
 *  - Per-request unmerged xAB computed on the fly for a batch of different
 *    adapters, no padding: "S-LoRA：一个GPU运行数千大模型成为可能",
 *    section 批处理 (batching), the paragraphs on formula 1 and formula 2.
 *  - Dropout on the LoRA branch input is one of the small ops between the
 *    GEMMs: LoRAFusion explainer, same section. Its mask is a SplitMix64
 *    counter hash (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *    generators", OOPSLA 2014), with the kept elements scaled by 1/(1-p)
 *    (inverted dropout; the pages are silent on the scaling).
 *  - The per-adapter scale s_a multiplies the LoRA term; the pages never
 *    write it and it is taken as stated for the workloads.
 *  - Rank-exact factor pool: adapter a owns rows [off_a, off_a + r_a) of
 *    A_pool (length d_in, i.e. columns of A_a) and of B_pool (length d_out),
 *    off_a = sum of ranks of adapters 0..a-1 (S-LoRA article, section
 *    Unified Paging: a rank-R weight takes R vectors).
 *  - Backward: plain chain rule of the forward with W frozen.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf(uint16_t h) {
    union { uint32_t u; float f; } v;
    v.u = ((uint32_t)h) << 16;
    return (double)v.f;
}

/* ---------------------------------------------------------------- SplitMix64
 * The generator keeps a 64-bit state that advances by the golden-ratio
 * increment 0x9E3779B97F4A7C15 before each output; the output is the state
 * passed through the finaliser (xor-shift 30, multiply, xor-shift 27,
 * multiply, xor-shift 31). The n-th output (0-based) of a generator seeded
 * with `seed` therefore mixes seed + (n+1)*increment. */
uint64_t oracle_splitmix64_next(uint64_t *state) {
    *state += 0x9E3779B97F4A7C15ULL;
    uint64_t z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t oracle_splitmix64_at(uint64_t seed, uint64_t n) {
    uint64_t state = seed + n * 0x9E3779B97F4A7C15ULL;
    return oracle_splitmix64_next(&state);
}

/* Drop threshold: an element is dropped iff its hash h < floor(p * 2^64),
 * which happens with probability p. p = 0 drops nothing. */
uint64_t oracle_drop_threshold(double p) {
    if (!(p > 0.0)) return 0;
    if (p >= 1.0) return UINT64_MAX;
    return (uint64_t)ldexp(p, 64);
}

/* mask element for input row t (original token index), column col. */
static int dropped(uint64_t seed, uint64_t thr, int64_t t, int64_t col, int64_t d_in) {
    if (thr == 0) return 0;
    return oracle_splitmix64_at(seed, (uint64_t)(t * d_in + col)) < thr;
}

void oracle_mask(uint64_t seed, double p, int64_t T, int64_t d_in, uint8_t *mask) {
    uint64_t thr = oracle_drop_threshold(p);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t i = 0; i < d_in; ++i)
            mask[t * d_in + i] = (uint8_t)dropped(seed, thr, t, i, d_in);
}

/* Multiplier applied to X[t,i] on the LoRA branch: 0 if dropped, else 1/(1-p). */
static double keep_factor(uint64_t seed, uint64_t thr, double p, int64_t t, int64_t i, int64_t d_in) {
    if (thr == 0) return 1.0;
    return dropped(seed, thr, t, i, d_in) ? 0.0 : 1.0 / (1.0 - p);
}

/* ---------------------------------------------------------------- plan
 * Stable grouping of tokens by adapter id: sorted position -> original token,
 * ties kept in original order; then run lengths per adapter (ascending id,
 * adapters without tokens get no segment). */
typedef struct { int32_t id; int32_t t; } pair_t;

static int cmp_pair(const void *a, const void *b) {
    const pair_t *x = (const pair_t *)a, *y = (const pair_t *)b;
    if (x->id != y->id) return x->id < y->id ? -1 : 1;
    return x->t < y->t ? -1 : (x->t > y->t);
}

/* Returns 0, or -1 if an id is outside [0, n_adapters). seg is n_seg x 3
 * (adapter, start, length); it must hold min(T, n_adapters) rows. */
int oracle_plan(const int32_t *ids, int64_t T, int32_t n_adapters,
                int32_t *perm, int32_t *seg, int32_t *n_seg) {
    for (int64_t t = 0; t < T; ++t)
        if (ids[t] < 0 || ids[t] >= n_adapters) return -1;
    pair_t *p = (pair_t *)malloc(sizeof(pair_t) * (size_t)(T > 0 ? T : 1));
    for (int64_t t = 0; t < T; ++t) { p[t].id = ids[t]; p[t].t = (int32_t)t; }
    qsort(p, (size_t)T, sizeof(pair_t), cmp_pair);
    int32_t ns = 0;
    for (int64_t i = 0; i < T; ++i) {
        perm[i] = p[i].t;
        if (i == 0 || p[i].id != p[i - 1].id) {
            seg[3 * ns + 0] = p[i].id;
            seg[3 * ns + 1] = (int32_t)i;
            seg[3 * ns + 2] = 0;
            ++ns;
        }
        seg[3 * (ns - 1) + 2] += 1;
    }
    *n_seg = ns;
    free(p);
    return 0;
}

static void offsets_of(const int32_t *ranks, int32_t n, int64_t *off) {
    off[0] = 0;
    for (int32_t a = 0; a < n; ++a) off[a + 1] = off[a] + ranks[a];
}

/* ---------------------------------------------------------------- forward
 * For each requested original token t (rows[0..n_rows)), a = ids[t]:
 *   Xd[i]  = X[t,i] * keep(t,i)
 *   U[k]   = sum_i Xd[i] * A_a[i,k]                       k < r_a
 *   Y[j]   = sum_i X[t,i] * W[i,j] + s_a * sum_k U[k] * B_a[k,j]
 * A_a[i,k] is A_pool[off_a + k][i]; B_a[k,j] is B_pool[off_a + k][j].
 * Y is n_rows x d_out; U (may be NULL) is n_rows x u_stride with entries
 * k >= r_a set to 0. */
void oracle_fwd(int64_t T, int64_t d_in, int64_t d_out, int32_t n_adapters,
                const int32_t *ids, const int32_t *ranks, const float *scale,
                const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                const uint16_t *B_pool, double p, uint64_t seed,
                const int64_t *rows, int64_t n_rows,
                double *Y, double *U, int64_t u_stride) {
    (void)T;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_adapters + 1));
    offsets_of(ranks, n_adapters, off);
    uint64_t thr = oracle_drop_threshold(p);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < n_rows; ++q) {
        int64_t t = rows[q];
        int32_t a = ids[t];
        int32_t r = ranks[a];
        double s = (double)scale[a];
        double *y = Y + q * d_out;
        double *u = (double *)calloc((size_t)(r > 0 ? r : 1), sizeof(double));
        /* base term X[t,:] * W */
        for (int64_t j = 0; j < d_out; ++j) y[j] = 0.0;
        for (int64_t i = 0; i < d_in; ++i) {
            double x = bf(X[t * d_in + i]);
            const uint16_t *wrow = W + i * d_out;
            for (int64_t j = 0; j < d_out; ++j) y[j] += x * bf(wrow[j]);
        }
        /* shrink: U = Xd * A_a, Xd[i] = X[t,i] * keep(t,i) */
        double *xd = (double *)malloc(sizeof(double) * (size_t)d_in);
        for (int64_t i = 0; i < d_in; ++i)
            xd[i] = bf(X[t * d_in + i]) * keep_factor(seed, thr, p, t, i, d_in);
        for (int32_t k = 0; k < r; ++k) {
            const uint16_t *arow = A_pool + (off[a] + k) * d_in;
            double acc = 0.0;
            for (int64_t i = 0; i < d_in; ++i) acc += xd[i] * bf(arow[i]);
            u[k] = acc;
        }
        free(xd);
        /* expand: Y += s * U * B_a */
        for (int64_t j = 0; j < d_out; ++j) {
            double acc = 0.0;
            for (int32_t k = 0; k < r; ++k)
                acc += u[k] * bf(B_pool[(off[a] + k) * d_out + j]);
            y[j] += s * acc;
        }
        if (U) {
            for (int64_t k = 0; k < u_stride; ++k) U[q * u_stride + k] = k < r ? u[k] : 0.0;
        }
        free(u);
    }
    free(off);
}

/* ---------------------------------------------------------------- backward
 * Chain rule of the forward with W frozen, for every token t (a = ids[t]):
 *   dU[t,k]   = s_a * sum_j dY[t,j] * B_a[k,j]
 *   dB_a[k,j] = s_a * sum_{t in a} U[t,k] * dY[t,j]
 *   dA_a[i,k] = sum_{t in a} Xd[t,i] * dU[t,k]
 *   dX[t,i]   = sum_j dY[t,j] * W[i,j] + keep(t,i) * sum_k dU[t,k] * A_a[i,k]
 * dA_pool has the pool's layout (row off_a + k holds dA_a[:,k], length d_in),
 * dB_pool likewise (row off_a + k holds dB_a[k,:]). dX is computed for the
 * requested rows only (n_rows x d_in); dA_pool / dB_pool (NULL to skip) sum
 * over all T tokens. */
void oracle_bwd(int64_t T, int64_t d_in, int64_t d_out, int32_t n_adapters,
                const int32_t *ids, const int32_t *ranks, const float *scale,
                const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                const uint16_t *B_pool, double p, uint64_t seed, const uint16_t *dY,
                const int64_t *rows, int64_t n_rows, double *dX,
                double *dA_pool, double *dB_pool) {
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_adapters + 1));
    offsets_of(ranks, n_adapters, off);
    int32_t rmax = 1;
    for (int32_t a = 0; a < n_adapters; ++a) if (ranks[a] > rmax) rmax = ranks[a];
    uint64_t thr = oracle_drop_threshold(p);
    int need_all = (dA_pool != NULL) || (dB_pool != NULL);
    double *U = NULL, *dU = NULL;
    if (need_all) {
        U = (double *)calloc((size_t)T * (size_t)rmax, sizeof(double));
        dU = (double *)calloc((size_t)T * (size_t)rmax, sizeof(double));
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            int32_t a = ids[t];
            double s = (double)scale[a];
            double *xd = (double *)malloc(sizeof(double) * (size_t)d_in);
            for (int64_t i = 0; i < d_in; ++i)
                xd[i] = bf(X[t * d_in + i]) * keep_factor(seed, thr, p, t, i, d_in);
            for (int32_t k = 0; k < ranks[a]; ++k) {
                const uint16_t *arow = A_pool + (off[a] + k) * d_in;
                const uint16_t *brow = B_pool + (off[a] + k) * d_out;
                double acc = 0.0;
                for (int64_t i = 0; i < d_in; ++i) acc += xd[i] * bf(arow[i]);
                U[t * rmax + k] = acc;
                double g = 0.0;
                for (int64_t j = 0; j < d_out; ++j) g += bf(dY[t * d_out + j]) * bf(brow[j]);
                dU[t * rmax + k] = s * g;
            }
            free(xd);
        }
    }
    if (dB_pool) {
        int64_t R = off[n_adapters];
        for (int64_t q = 0; q < R * d_out; ++q) dB_pool[q] = 0.0;
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < d_out; ++j) {
            for (int64_t t = 0; t < T; ++t) {
                int32_t a = ids[t];
                double s = (double)scale[a];
                double g = bf(dY[t * d_out + j]);
                for (int32_t k = 0; k < ranks[a]; ++k)
                    dB_pool[(off[a] + k) * d_out + j] += s * U[t * rmax + k] * g;
            }
        }
    }
    if (dA_pool) {
        int64_t R = off[n_adapters];
        for (int64_t q = 0; q < R * d_in; ++q) dA_pool[q] = 0.0;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < d_in; ++i) {
            for (int64_t t = 0; t < T; ++t) {
                int32_t a = ids[t];
                double xd = bf(X[t * d_in + i]) * keep_factor(seed, thr, p, t, i, d_in);
                for (int32_t k = 0; k < ranks[a]; ++k)
                    dA_pool[(off[a] + k) * d_in + i] += xd * dU[t * rmax + k];
            }
        }
    }
    if (dX && n_rows > 0) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t q = 0; q < n_rows; ++q) {
            int64_t t = rows[q];
            int32_t a = ids[t];
            int32_t r = ranks[a];
            double s = (double)scale[a];
            double *du = (double *)calloc((size_t)(r > 0 ? r : 1), sizeof(double));
            for (int32_t k = 0; k < r; ++k) {
                const uint16_t *brow = B_pool + (off[a] + k) * d_out;
                double g = 0.0;
                for (int64_t j = 0; j < d_out; ++j) g += bf(dY[t * d_out + j]) * bf(brow[j]);
                du[k] = s * g;
            }
            for (int64_t i = 0; i < d_in; ++i) {
                const uint16_t *wrow = W + i * d_out;
                double acc = 0.0;
                for (int64_t j = 0; j < d_out; ++j) acc += bf(dY[t * d_out + j]) * bf(wrow[j]);
                double lora = 0.0;
                for (int32_t k = 0; k < r; ++k) lora += du[k] * bf(A_pool[(off[a] + k) * d_in + i]);
                dX[q * d_in + i] = acc + keep_factor(seed, thr, p, t, i, d_in) * lora;
            }
            free(du);
        }
    }
    free(U);
    free(dU);
    free(off);
}

/* ---------------------------------------------------------------- adapter switch (merge path)
 * Fused adapter switching of "AdaFuse: Accelerating Dynamic Adapter Inference
 * via Token-Level Pre-Gating and Fused Kernel Optimization" (方法详解, 关键设计
 * item 2): the previous token's active adapters are unmerged (negative
 * weights) and the current token's merged (positive weights) in one update of
 * every layer's weight, W_l <- W_l + DOWN·UP with DOWN the concatenation of the
 * weighted A factors and UP the stacked B factors. Term j names adapter
 * term_adapter[j] and its coefficient term_coef[j] (the caller's signed gate
 * times the adapter's scale). For every layer l, row i, column j:
 *   Wx[l,i,j] = W[l,i,j] + sum_terms c * sum_{k < r_a} A_pool_l[off_a + k][i] * B_pool_l[off_a + k][j]
 * in fp64, exact inputs; Wx is the unrounded result (the caller rounds to the
 * weight's precision). Layer l's pools are A_pool + l*R*d_in, B_pool + l*R*d_out
 * (R = sum of all ranks), with the same adapter offsets in every layer. */
void oracle_switch(int64_t L, int64_t d_in, int64_t d_out, int32_t n_adapters, const int32_t *ranks,
                   const uint16_t *W, const uint16_t *A_pool, const uint16_t *B_pool,
                   int32_t n_terms, const int32_t *term_adapter, const double *term_coef, double *Wx) {
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_adapters + 1));
    offsets_of(ranks, n_adapters, off);
    int64_t R = off[n_adapters];
#pragma omp parallel for schedule(static)
    for (int64_t li = 0; li < L * d_in; ++li) {
        int64_t l = li / d_in, i = li % d_in;
        const uint16_t *Al = A_pool + l * R * d_in;
        const uint16_t *Bl = B_pool + l * R * d_out;
        for (int64_t j = 0; j < d_out; ++j) {
            double acc = bf(W[(l * d_in + i) * d_out + j]);
            for (int32_t q = 0; q < n_terms; ++q) {
                int32_t a = term_adapter[q];
                double dot = 0.0;
                for (int32_t k = 0; k < ranks[a]; ++k)
                    dot += bf(Al[(off[a] + k) * d_in + i]) * bf(Bl[(off[a] + k) * d_out + j]);
                acc += term_coef[q] * dot;
            }
            Wx[(l * d_in + i) * d_out + j] = acc;
        }
    }
    free(off);
}

/* ---------------------------------------------------------------- tall-skinny QR (FlashTSQR)
 * "LoRAForge：压缩与执行协同，让多LoRA服务更高效", FlashTSQR section: the
 * factor construction of post-hoc compression runs a QR of many tall, skinny
 * factor matrices (rows far more than columns), parallel across modules and
 * across row blocks. The oracle is the QR itself, by Householder reflections
 * on the whole matrix in fp64 (the textbook algorithm, column by column):
 * for column j, x = A[j:, j], alpha = -sign(x_0)·||x||, v = x - alpha·e_0,
 * A[j:, j:] -= 2·v·(v^T·A[j:, j:]) / (v^T·v). R is the upper n x n triangle of
 * the result; Q (m x n) = H_0·H_1·...·H_{n-1} applied to the first n columns
 * of the identity. For each of `batch` matrices A [m x n] (row-major), outputs
 * R [n x n] (zeros below the diagonal) and Q [m x n] (NULL to skip). */
void oracle_qr(int64_t batch, int64_t m, int64_t n, const double *A, double *R, double *Q) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < batch; ++b) {
        double *a = (double *)malloc(sizeof(double) * (size_t)(m * n));
        double *V = (double *)calloc((size_t)(m * n), sizeof(double)); /* reflector j in column j */
        double *vv = (double *)calloc((size_t)n, sizeof(double));      /* v_j^T v_j */
        memcpy(a, A + b * m * n, sizeof(double) * (size_t)(m * n));
        for (int64_t j = 0; j < n; ++j) {
            double norm2 = 0.0;
            for (int64_t i = j; i < m; ++i) norm2 += a[i * n + j] * a[i * n + j];
            double norm = sqrt(norm2);
            double x0 = a[j * n + j];
            double alpha = x0 >= 0.0 ? -norm : norm;
            for (int64_t i = j; i < m; ++i) V[i * n + j] = a[i * n + j];
            V[j * n + j] = x0 - alpha;
            double vtv = 0.0;
            for (int64_t i = j; i < m; ++i) vtv += V[i * n + j] * V[i * n + j];
            vv[j] = vtv;
            if (vtv == 0.0) continue; /* the column is already zero below the diagonal */
            for (int64_t c = j; c < n; ++c) {
                double w = 0.0;
                for (int64_t i = j; i < m; ++i) w += V[i * n + j] * a[i * n + c];
                double f = 2.0 * w / vtv;
                for (int64_t i = j; i < m; ++i) a[i * n + c] -= f * V[i * n + j];
            }
        }
        for (int64_t i = 0; i < n; ++i)
            for (int64_t c = 0; c < n; ++c) R[(b * n + i) * n + c] = c >= i ? a[i * n + c] : 0.0;
        if (Q) {
            double *q = Q + b * m * n;
            for (int64_t i = 0; i < m; ++i)
                for (int64_t c = 0; c < n; ++c) q[i * n + c] = i == c ? 1.0 : 0.0;
            for (int64_t j = n - 1; j >= 0; --j) { /* Q = H_0 (H_1 (... (H_{n-1} E))) */
                if (vv[j] == 0.0) continue;
                for (int64_t c = 0; c < n; ++c) {
                    double w = 0.0;
                    for (int64_t i = j; i < m; ++i) w += V[i * n + j] * q[i * n + c];
                    double f = 2.0 * w / vv[j];
                    for (int64_t i = j; i < m; ++i) q[i * n + c] -= f * V[i * n + j];
                }
            }
        }
        free(a);
        free(V);
        free(vv);
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
