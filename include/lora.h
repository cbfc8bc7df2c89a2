/*
 * lora.h — C ABI of the B200 (sm_100a) heterogeneous multi-adapter LoRA linear layer.
 *
 * The layer computes, for every token t carrying adapter id a = ids[t],
 *
 *     Y[t] = X[t]·W + s_a·((D ⊙ X)[t]·A_a)·B_a
 *
 * with W frozen and each adapter keeping its own rank r_a (no padding to a
 * common rank), D an optional dropout mask on the LoRA-branch input.
 *  - The LoRA reparameterisation Y = X·W + X·(A·B) with A in R^{d x r},
 *    B in R^{r x k}, W frozen: "LoRAFusion：消除冗余内存访问的多 LoRA 高效微调系统",
 *    section 解决什么真问题 (what problem it solves), item 1.
 *  - Computing xAB on the fly for a batch mixing many adapters, base part
 *    batched, without padding: "S-LoRA：一个GPU运行数千大模型成为可能",
 *    section 批处理 (batching).
 *  - Rank-exact factor storage (a rank-R weight occupies R vectors of the
 *    hidden size): same S-LoRA article, section Unified Paging.
 *  - Keeping each adapter at its retained rank instead of padding or
 *    re-expanding: "LoRAForge：压缩与执行协同，让多LoRA服务更高效",
 *    section 核心设计 (core design).
 *  - Dropout is one of the small memory-bound ops between the GEMMs of a LoRA
 *    forward: LoRAFusion explainer, section 解决什么真问题, item 1.
 *
 * Conventions for every entry point:
 *  - bf16 tensors are passed as `uint16_t*` holding bf16 bit patterns, row-major,
 *    contiguous, in DEVICE memory, 16-byte aligned. Sizes are element counts.
 *  - The caller owns every tensor buffer. A plan owns its own small device and
 *    host arrays (and its forward scratch) until lora_plan_destroy.
 *  - Every call that launches work is asynchronous and ordered on `stream`
 *    (a cudaStream_t; NULL is the legacy default stream). Nothing synchronises
 *    the host except lora_plan_build (which copies the plan to the device) and
 *    lora_device_status.
 *  - Return value: LORA_OK (0) or a negative LORA_ERR_* code. Arguments are
 *    validated on the host before any launch; on an error nothing is launched.
 *    No exception crosses the ABI.
 *  - Kernels never trap: a device-side bounds violation or a wait that runs
 *    out of time sets a per-device status word (see lora_device_status) and the
 *    kernel returns early.
 */
#ifndef LORA_B200_H
#define LORA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *lora_stream_t; /* identical to cudaStream_t */
typedef struct lora_plan *lora_plan_t;

enum lora_status {
    LORA_OK = 0,
    LORA_ERR_ARG = -1,         /* null pointer, non-positive size, size not a multiple of 8, misaligned pointer */
    LORA_ERR_ID = -2,          /* an adapter id outside [0, n_adapters) */
    LORA_ERR_RANK = -3,        /* a rank outside [1, LORA_MAX_RANK] */
    LORA_ERR_CUDA = -4,        /* a CUDA runtime or driver call failed */
    LORA_ERR_DEVICE = -5,      /* the device status word was set (bounds or wait timeout) */
    LORA_ERR_UNSUPPORTED = -6, /* the current device is not sm_100 */
    LORA_ERR_NOMEM = -7,       /* a plan allocation failed */
    LORA_ERR_WORKSPACE = -8    /* workspace pointer null or smaller than required */
};

#define LORA_MAX_RANK 256
#define LORA_TILE_M 128 /* tokens per output tile of the fused GEMM */

/* Device status word bits (lora_device_status). */
#define LORA_DEV_TIMEOUT 0x1u /* a bounded wait inside a kernel ran out of time */
#define LORA_DEV_BOUNDS 0x2u  /* a kernel saw an index outside its buffers and skipped it */

/* ------------------------------------------------------------------------
 * lora_plan_build — group a batch's tokens by adapter (once per batch).
 *
 * Sorts the T tokens by adapter id (stable: ties keep their original order)
 * into segments of consecutive tokens sharing one adapter, cuts the sorted
 * order into 128-token output tiles, and lists for each tile the adapters it
 * touches with their ranks and factor-pool offsets (off_a = sum of ranks of
 * adapters 0..a-1). A plan depends only on (ids, ranks, d_in, d_out) and can be
 * reused by every LoRA linear layer of one batch that shares them; deciding the
 * routing once per batch and reusing it across layers follows the token-level
 * pre-gating idea of "AdaFuse: Accelerating Dynamic Adapter Inference via
 * Token-Level Pre-Gating and Fused Kernel Optimization", 方法详解 (method),
 * 整体框架 (framework).
 *
 *   ids_host    int32[T] host: adapter id of each token, in [0, n_adapters)
 *   T           number of tokens, >= 1
 *   ranks_host  int32[n_adapters] host: r_a in [1, LORA_MAX_RANK]
 *   n_adapters  >= 1
 *   d_in, d_out input / output width, multiples of 8, >= 8
 *   stream      stream for the plan's host-to-device copy; the call
 *               synchronises it, so the plan is on the device on return (and
 *               the host arrays may be freed)
 *   out         receives the plan; unchanged on error
 * The plan belongs to the device current at this call: lora_plan_rebuild,
 * lora_linear_shrink, lora_fused_gemm and lora_linear_fwd return LORA_ERR_ARG
 * when another device is current.
 * Errors: LORA_ERR_ARG, LORA_ERR_ID, LORA_ERR_RANK, LORA_ERR_NOMEM, LORA_ERR_CUDA.
 * ------------------------------------------------------------------------ */
int lora_plan_build(const int32_t *ids_host, int64_t T, const int32_t *ranks_host,
                    int32_t n_adapters, int64_t d_in, int64_t d_out, lora_stream_t stream,
                    lora_plan_t *out);

/* Refill an existing device plan with a new batch (arguments as in
 * lora_plan_build). The plan's device tables and scratch are reused when they
 * are large enough and reallocated otherwise, so a serving loop that builds one
 * plan per batch does not allocate device memory per batch; its host tables are
 * kept in two sets (the new batch is planned into the spare set, which becomes
 * the plan's on success), so once they have grown a rebuild allocates no host
 * memory either. The tables are
 * copied to the device on `stream` from one of two pinned host staging buffers
 * the plan owns (used in turn; a buffer is refilled only after its previous copy
 * has completed), and the call returns without waiting for that copy: work that
 * uses the rebuilt plan must run on `stream` or after it, and work on other
 * streams that uses the plan's previous contents must be finished before the
 * call or ordered before `stream` by the caller (work earlier on `stream` is
 * ordered by the stream). The host arrays may be freed on return. When the
 * plan's device buffers must grow they are reallocated, which waits for the
 * device. On LORA_ERR_ARG / LORA_ERR_ID / LORA_ERR_RANK the plan is unchanged;
 * after LORA_ERR_NOMEM or LORA_ERR_CUDA it holds no device memory and is only
 * good for lora_plan_destroy. No counterpart in the pages (the plan's device
 * lifetime is this library's design). */
int lora_plan_rebuild(lora_plan_t plan, const int32_t *ids_host, int64_t T, const int32_t *ranks_host,
                      int32_t n_adapters, int64_t d_in, int64_t d_out, lora_stream_t stream);

/* Host-only variant of lora_plan_build: the same grouping and tile layout,
 * but no device buffers (no CUDA call at all). Such a plan can be inspected
 * with lora_plan_get / lora_plan_info and destroyed; lora_linear_fwd rejects
 * it with LORA_ERR_ARG. Errors: LORA_ERR_ARG, LORA_ERR_ID, LORA_ERR_RANK,
 * LORA_ERR_NOMEM. */
int lora_plan_build_host(const int32_t *ids_host, int64_t T, const int32_t *ranks_host,
                         int32_t n_adapters, int64_t d_in, int64_t d_out, lora_plan_t *out);

/* Copy the plan's grouping to host memory.
 *   perm_host   int32[T] or NULL: perm[i] = original index of the token at sorted position i
 *   seg_host    int32[n_seg*3] or NULL: (adapter, start, length) per segment, ascending
 *               adapter id, start = first sorted position; adapters without tokens have none
 *   n_seg       int32* or NULL: number of segments
 * No counterpart in the pages (inspection of this library's plan).
 * Errors: LORA_ERR_ARG (null plan). */
int lora_plan_get(lora_plan_t plan, int32_t *perm_host, int32_t *seg_host, int32_t *n_seg);

typedef struct lora_plan_info {
    int64_t T, d_in, d_out;
    int32_t n_adapters;
    int32_t n_segments;
    int32_t n_tiles;        /* ceil(T / LORA_TILE_M) */
    int32_t r_max;          /* largest rank among adapters that own tokens */
    int64_t sum_r_used;     /* sum of ranks of adapters that own tokens */
    int64_t sum_r_tokens;   /* sum over tokens of their adapter's rank */
    int64_t aug_k_total;    /* sum over tiles of the tile's augmented K (multiples of 16) */
    int64_t scratch_bytes;  /* device scratch owned by the plan */
    int32_t gathers_x;      /* 1 if the forward first writes the adapter-sorted copy of X
                               into the scratch (some tile is not a run of consecutive
                               tokens): one more kernel launch per forward */
} lora_plan_info_t;

/* The plan's sizes. No counterpart in the pages (inspection of this library's
 * plan). Errors: LORA_ERR_ARG. */
int lora_plan_info(lora_plan_t plan, lora_plan_info_t *info);

/* Free the plan (waits for nothing; the caller must not free a plan that queued
 * work still uses). NULL is ignored. No counterpart in the pages (the plan's
 * lifetime is this library's design). */
void lora_plan_destroy(lora_plan_t plan);

/* ------------------------------------------------------------------------
 * lora_linear_fwd — Y = X·W + s_a·((D ⊙ X)·A_a)·B_a for every token.
 * Source: the LoRA reparameterisation of the LoRAFusion explainer (section
 * 解决什么真问题, item 1), applied per token with that token's adapter, the
 * base part batched and no padding (S-LoRA article, section 批处理).
 *
 *   X       bf16 [T, d_in]     tokens in their original order
 *   W       bf16 [d_in, d_out] frozen base weight
 *   A_pool  bf16 [R, d_in]     R = sum of all ranks; row off_a + k is column k of A_a
 *   B_pool  bf16 [R, d_out]    row off_a + k is row k of B_a
 *   scale   f32  [n_adapters]  DEVICE array of s_a
 *   p_drop  dropout probability on the LoRA-branch input, in [0, 1); 0 disables.
 *           Element (t, i) of X (t = original token index) is dropped iff
 *           h < floor(p_drop * 2^64), where h is output number t*d_in + i
 *           (0-based) of the SplitMix64 generator seeded with `seed`; kept
 *           elements are scaled by 1/(1 - p_drop). The base term X·W never sees
 *           dropout.
 *   seed    dropout seed
 *   Y       bf16 [T, d_out]    output, original token order (fp32 accumulation,
 *           rounded once to bf16)
 *   U_save  f32 [T, r_max] or NULL: U[t,k] = ((D ⊙ X)[t]·A_a)[k] for k < r_a,
 *           zero for k >= r_a (r_max from lora_plan_info); the backward's input.
 *           Kept in fp32: the backward reduces it over all tokens, where a bf16
 *           rounding of every term would dominate the error of small sums.
 *   keep_bits  u32 [T, ceil(d_in/32)] DEVICE array or NULL: the dropout mask as
 *           written by lora_dropout_keep_bits(seed, p_drop, T, d_in) (4-byte
 *           aligned). Read instead of re-deriving each bit from the generator;
 *           ignored when p_drop is 0. The caller guarantees it matches seed and
 *           p_drop. One mask array serves a forward and its backward.
 *   stream  launch stream
 * The plan's scratch holds s_a·U rounded to bf16 between the two kernels, so
 * two forwards with one plan must not run concurrently.
 * Adapter isolation: a token's output reads only its own adapter's factor rows
 * and the factor rows of adapters whose tokens share its 128-token tile of the
 * sorted order (the tile's adapter K slices form one block-diagonal
 * contraction, where other adapters' rows meet zeros). Factor rows of adapters
 * with no token in that tile never enter it, even where a rank is not a
 * multiple of 16 (the rows past it are zeroed on chip). Non-finite values in
 * an adapter's B rows therefore reach, as NaN, only tokens of tiles that adapter
 * shares.
 * Errors: LORA_ERR_ARG, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA.
 * ------------------------------------------------------------------------ */
int lora_linear_fwd(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                    const uint16_t *B_pool, const float *scale, double p_drop, uint64_t seed,
                    uint16_t *Y, float *U_save, const uint32_t *keep_bits, lora_stream_t stream);

/* The forward's two phases, for callers that schedule or time them apart
 * (lora_linear_fwd is exactly lora_linear_shrink followed by lora_fused_gemm
 * on one stream).
 *
 * Source: the shrink (X·A) and expand (·B) halves of the same
 * reparameterisation; the pages keep them as separate small kernels next to
 * the base GEMM, here the expand is folded into the GEMM.
 *
 * lora_linear_shrink: U = (D ⊙ X)·A_a for every token, written as s_a·U in
 * bf16 into the plan's scratch (in the layout the fused GEMM reads) and, if
 * U_save is not NULL, as U into U_save. When the plan's tiles are not runs of
 * consecutive tokens, it first copies X's rows in sorted order into the plan's
 * scratch (a sorted copy both kernels read). Arguments as in lora_linear_fwd.
 *
 * lora_fused_gemm: Y = X·W + (s_a·U)·B_a from the plan's scratch, which must
 * hold the output of a lora_linear_shrink with the same plan that is ordered
 * before this call on the stream.
 * Errors: LORA_ERR_ARG, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA. */
int lora_linear_shrink(lora_plan_t plan, const uint16_t *X, const uint16_t *A_pool, const float *scale,
                       double p_drop, uint64_t seed, float *U_save, const uint32_t *keep_bits,
                       lora_stream_t stream);
int lora_fused_gemm(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *B_pool,
                    uint16_t *Y, lora_stream_t stream);

/* lora_linear_fwd_host — one serving step from host memory: the batch's plan
 * from its host ids (lora_plan_rebuild of `plan` with the plan's d_in, d_out),
 * the copy of X from host to device, lora_linear_fwd, and the copy of Y from
 * device to host, queued on `stream` in that order. The call returns once the
 * work is queued: Y_host holds the step's result when `stream` has passed it
 * (synchronise the stream or wait on an event recorded after the call). With
 * pinned host buffers both copies run asynchronously, so steps queued on two
 * streams with two plans and two sets of buffers overlap one step's copies with
 * the other's kernels. No counterpart in the pages (the per-batch host-to-device
 * path of a serving loop around the layer).
 *
 *   plan        a device plan (lora_plan_build); rebuilt for this batch, so work on
 *               other streams that still uses its previous batch must be ordered first
 *   ids_host, T, ranks_host, n_adapters   the batch, as in lora_plan_build
 *   X_host      bf16 [T, d_in] host
 *   X_dev       bf16 [T, d_in] device buffer the step copies X into (16-byte aligned)
 *   W, A_pool, B_pool, scale, p_drop, seed, U_save, keep_bits   as in lora_linear_fwd
 *   Y_dev       bf16 [T, d_out] device output of the forward (16-byte aligned)
 *   Y_host      bf16 [T, d_out] host destination of the copy out
 * The caller owns every buffer; the call allocates nothing (beyond what a plan
 * rebuild does when the batch outgrows the plan's buffers).
 * Errors: as lora_plan_rebuild (the plan is unchanged on LORA_ERR_ARG, _ID or
 * _RANK from it) and lora_linear_fwd; LORA_ERR_ARG for a null or misaligned
 * buffer before anything is queued; LORA_ERR_CUDA when a copy cannot be queued. */
int lora_linear_fwd_host(lora_plan_t plan, const int32_t *ids_host, int64_t T, const int32_t *ranks_host,
                         int32_t n_adapters, const uint16_t *X_host, uint16_t *X_dev, const uint16_t *W,
                         const uint16_t *A_pool, const uint16_t *B_pool, const float *scale, double p_drop,
                         uint64_t seed, uint16_t *Y_dev, uint16_t *Y_host, float *U_save,
                         const uint32_t *keep_bits, lora_stream_t stream);

/* lora_linear_fwd_fused — lora_linear_fwd in one launch (arguments and results
 * as lora_linear_fwd). Source: the kernel-layer fusion of the LoRAFusion
 * explainer (Kernel 层: split the graph only at real GEMM boundaries and keep
 * the small ops' work next to the big GEMM), applied to the shrink and the row
 * gather, which otherwise run as kernels of their own before the fused GEMM.
 * The launch's CTAs first copy X's rows into the plan's sorted copy (when the
 * plan gathers) and wait for every CTA's share, then run the plan's shrink units
 * (one CTA per unit), each counting itself done for its 128-token tile, then the
 * fused GEMM's tiles with the adapter K blocks last, a tile's first adapter
 * block waiting (bounded) for its tile's count. The launch is cooperative, so
 * every CTA is resident and every wait ends; the plan holds the lists of units
 * per CTA for the launch's grid, and its counters are zeroed on `stream` before
 * the launch (two fused forwards with one plan must not overlap). Results agree
 * with lora_linear_fwd within rounding (each unit's contraction is summed by one
 * CTA instead of a cluster, and the adapter blocks enter the accumulator after
 * the base blocks instead of before).
 * Errors: LORA_ERR_ARG, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA (also when the device
 * refuses the cooperative launch). */
int lora_linear_fwd_fused(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                          const uint16_t *B_pool, const float *scale, double p_drop, uint64_t seed, uint16_t *Y,
                          float *U_save, const uint32_t *keep_bits, lora_stream_t stream);

/* Y = X·W only (no adapter term), through the same tcgen05 GEMM kernel: the
 * base-only reference the adapter overhead is measured against (the frozen
 * base term of the LoRAFusion explainer's reparameterisation).
 * Errors: LORA_ERR_ARG, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA. */
int lora_base_gemm(const uint16_t *X, const uint16_t *W, uint16_t *Y, int64_t T, int64_t d_in,
                   int64_t d_out, lora_stream_t stream);

/* ------------------------------------------------------------------------
 * lora_linear_bwd — backward of the forward for one adapter (fine-tuning;
 * every token uses it), W frozen so no dW. The pages fix the forward and that
 * W is frozen (LoRAFusion explainer, section 解决什么真问题, item 1); the
 * backward is its plain chain rule:
 *   dU = s·dY·B^T                       [T, r]
 *   dB = s·U^T·dY                       [r, d_out]
 *   dA = ((D ⊙ X)^T·dU)^T, stored [r, d_in] (row k = column k of dA)
 *   dX = dY·W^T + D ⊙ (dU·A^T)          [T, d_in], D = keep mask / (1 - p)
 *
 *   X, W, A (bf16 [r, d_in], rows = columns of A), B (bf16 [r, d_out]),
 *   scale, p_drop, seed    as in the forward (same mask)
 *   r       the adapter's rank, 1 .. LORA_MAX_RANK
 *   U_save  f32 [T, r]     the forward's U_save (16-byte aligned when r % 16 == 0,
 *                          else 4-byte aligned)
 *   dY      bf16 [T, d_out]
 *   dX      bf16 [T, d_in]  output
 *   dA      f32 [r, d_in]   output (4-byte aligned)
 *   dB      f32 [r, d_out]  output (4-byte aligned)
 *   workspace, workspace_bytes  device scratch of at least
 *           lora_linear_bwd_workspace_size(T, d_in, d_out, r) bytes, 256-byte
 *           aligned, owned by the caller; contents on entry are ignored.
 *   keep_bits  NULL or the mask as in lora_linear_fwd (the forward's own array)
 * Reductions over tokens use a fixed split and a fixed summation order, so
 * results are deterministic run to run.
 * Errors: LORA_ERR_ARG, LORA_ERR_RANK, LORA_ERR_WORKSPACE, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA.
 * ------------------------------------------------------------------------ */
size_t lora_linear_bwd_workspace_size(int64_t T, int64_t d_in, int64_t d_out, int32_t r);

int lora_linear_bwd(const uint16_t *X, const uint16_t *W, const uint16_t *A, const uint16_t *B,
                    float scale, double p_drop, uint64_t seed, const float *U_save,
                    const uint16_t *dY, uint16_t *dX, float *dA, float *dB, int64_t T,
                    int64_t d_in, int64_t d_out, int32_t r, void *workspace,
                    size_t workspace_bytes, const uint32_t *keep_bits, lora_stream_t stream);

/* ------------------------------------------------------------------------
 * lora_linear_bwd_multi — the backward of lora_linear_fwd for a batch that
 * mixes adapters (multi-adapter fine-tuning: several jobs' adapters trained on
 * one frozen base in one batch), W frozen. Source: the LoRAFusion explainer,
 * section 解决什么真问题 (several LoRA jobs sharing one base model) and item 1
 * (the reparameterisation whose chain rule this is); per token t with adapter a:
 *   dU[t]  = s_a·dY[t]·B_a^T
 *   dX[t]  = dY[t]·W^T + D[t] ⊙ (dU[t]·A_a^T)         D = keep mask / (1 - p)
 *   dA_a   = sum over the tokens of a of (D ⊙ X)[t]^T·dU[t]   (pool layout, as A_pool)
 *   dB_a   = s_a · sum over the tokens of a of U[t]^T·dY[t]  (pool layout, as B_pool)
 *
 *   plan, X, W, A_pool, B_pool, scale, p_drop, seed, keep_bits
 *           as in lora_linear_fwd (the same plan and mask as the forward)
 *   U_save  f32 [T, r_max]  the forward's U_save (4-byte aligned)
 *   dY      bf16 [T, d_out]
 *   dX      bf16 [T, d_in]   output, original token order
 *   dA_pool f32 [R, d_in]    output: rows off_a .. off_a + r_a - 1 of every
 *                            adapter with tokens in the batch (4-byte aligned);
 *                            rows of adapters without tokens are not written
 *   dB_pool f32 [R, d_out]   output, likewise
 *   workspace, workspace_bytes  device scratch of at least
 *           lora_linear_bwd_multi_workspace_size(plan) bytes, 256-byte aligned,
 *           caller-owned; contents on entry are ignored
 * Each adapter's gradient is summed over its tokens in pieces of at most 1024
 * sorted tokens, in a fixed order: results are deterministic run to run. The
 * call reads the plan's tables but not its scratch. A segment's last piece may
 * share a 64-token stage with the next segment's tokens, which enter as zeros:
 * inputs are assumed finite.
 * Errors: LORA_ERR_ARG, LORA_ERR_WORKSPACE, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA.
 * ------------------------------------------------------------------------ */
size_t lora_linear_bwd_multi_workspace_size(lora_plan_t plan);

int lora_linear_bwd_multi(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                          const uint16_t *B_pool, const float *scale, double p_drop, uint64_t seed,
                          const float *U_save, const uint16_t *dY, uint16_t *dX, float *dA_pool, float *dB_pool,
                          void *workspace, size_t workspace_bytes, const uint32_t *keep_bits, lora_stream_t stream);

/* ------------------------------------------------------------------------
 * lora_linear_bwd_static — lora_linear_bwd without a caller workspace.
 *
 * No counterpart on the pages: this is an integration aid. Some callers cannot
 * allocate device memory at the point where they run the backward: a process
 * whose whole device memory is owned by another allocator (a framework's
 * caching allocator, or an arena a serving process reserves at start-up), where
 * an extra cudaMalloc fails or fragments that pool; plugins hosted by a program
 * that gives them no allocator; and code that must not allocate once it is
 * running (fixed-memory or real-time deployments). This entry point takes the
 * same arguments as lora_linear_bwd except the workspace and allocates nothing:
 * its scratch is a file-scope device array of LORA_BWD_STATIC_SCRATCH_BYTES
 * bytes inside the library, which every GPU that loads the library holds until
 * the process exits.
 *
 *  - Requests whose workspace need (lora_linear_bwd_workspace_size) exceeds
 *    LORA_BWD_STATIC_SCRATCH_BYTES are rejected with LORA_ERR_WORKSPACE before
 *    anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture on the device.
 *  - Every call shares the one array, and the array keeps what the last call
 *    left in it. Nothing in it needs to start at zero: each call writes every
 *    scratch byte it later reads. Calls that overlap on the GPU (different
 *    streams, or different host threads, without ordering between them) race
 *    on the array and give wrong results; order them.
 * Errors: as lora_linear_bwd.
 * ------------------------------------------------------------------------ */
#define LORA_BWD_STATIC_SCRATCH_BYTES ((size_t)8 << 20) /* 8 MiB */

int lora_linear_bwd_static(const uint16_t *X, const uint16_t *W, const uint16_t *A, const uint16_t *B,
                           float scale, double p_drop, uint64_t seed, const float *U_save,
                           const uint16_t *dY, uint16_t *dX, float *dA, float *dB, int64_t T,
                           int64_t d_in, int64_t d_out, int32_t r, const uint32_t *keep_bits,
                           lora_stream_t stream);

/* ------------------------------------------------------------------------
 * Fused adapter switching (the merge path): W_l <- W_l + sum_j c_j·A_{l,a_j}·B_{l,a_j}
 * for every layer l of a stack, in place, in one pass over the weights.
 *
 * Source: "AdaFuse: Accelerating Dynamic Adapter Inference via Token-Level
 * Pre-Gating and Fused Kernel Optimization", 方法详解, 关键设计 item 2 (fused
 * adapter switching: unmerge the previous token's adapters with negative weights
 * and merge the current ones with positive weights as one concatenated update)
 * and item 3 (all layers' merges as one batched launch, added in place into
 * the backbone).
 *
 * lora_switch_create — a switch context for a stack of L layers.
 *   ranks_host  int32[n_adapters]: every layer holds the same adapters with these
 *               ranks (1 .. LORA_MAX_RANK), in the pool layout of lora_linear_fwd
 *   L, d_in, d_out   layers and each layer's weight shape (multiples of 8, >= 8;
 *               L*d_in <= 2^30)
 *   max_terms   most terms an apply may pass, 1 .. LORA_SWITCH_MAX_TERMS
 * The context owns device scratch of about L*ceil(d_in/128)*ceil(K/64)*16 KB,
 * K = 2*max_terms*(largest rank rounded up to 16), plus small tables and two
 * pinned host staging buffers, until lora_switch_destroy. It belongs to the
 * device current at this call.
 * Errors: LORA_ERR_ARG, LORA_ERR_RANK, LORA_ERR_NOMEM, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA.
 *
 * lora_switch_apply — the update, asynchronous on `stream`.
 *   W       bf16 [L, d_in, d_out] DEVICE, updated in place:
 *           W[l,i,j] <- bf16(W[l,i,j] + sum_j c_j * sum_{k < r_a} A_pool_l[off_a + k][i] * B_pool_l[off_a + k][j])
 *           with the sum in fp32 and one rounding (nearest even) to bf16
 *   A_pool  bf16 [L, R, d_in]   layer l's pool at A_pool + l*R*d_in (R = sum of ranks)
 *   B_pool  bf16 [L, R, d_out]  layer l's pool at B_pool + l*R*d_out
 *   term_adapter_host int32[n_terms], term_coef_host float[n_terms] (host): term j
 *           adds c_j·A_a·B_a of adapter a = term_adapter_host[j], c_j =
 *           term_coef_host[j]; for a switch, the previous adapters with
 *           c = -gate*scale and the current ones with c = +gate*scale. The same
 *           terms apply to every layer.
 *   n_terms 1 .. max_terms
 * The host arrays may be freed on return (they are staged in pinned memory the
 * context owns and copied on `stream`). Two applies with one context must be
 * ordered (they share its scratch). c_j·A enters the tensor cores as a hi and a
 * lo bf16 part, so the weighted factor keeps about 16 bits.
 * Errors: LORA_ERR_ARG (null or misaligned pointer, n_terms out of range, another
 * device current), LORA_ERR_ID (a term's adapter out of range), LORA_ERR_CUDA.
 * ------------------------------------------------------------------------ */
#define LORA_SWITCH_MAX_TERMS 64
typedef struct lora_switch *lora_switch_t;

int lora_switch_create(const int32_t *ranks_host, int32_t n_adapters, int64_t L, int64_t d_in, int64_t d_out,
                       int32_t max_terms, lora_switch_t *out);
int lora_switch_apply(lora_switch_t sw, uint16_t *W, const uint16_t *A_pool, const uint16_t *B_pool,
                      const int32_t *term_adapter_host, const float *term_coef_host, int32_t n_terms,
                      lora_stream_t stream);
/* Free the context (waits for its staging copies; the caller must not free a
 * context that queued work still uses). NULL is ignored. */
void lora_switch_destroy(lora_switch_t sw);

/* Batched tall-skinny QR of adapter factors: the FlashTSQR factor construction
 * of post-hoc compression in "LoRAForge：压缩与执行协同，让多LoRA服务更高效"
 * (FlashTSQR section and the terms note on TSQR: a QR of many matrices with far
 * more rows than columns, each cut into row blocks whose local QRs are merged,
 * parallel across modules and across row blocks). A = Q·R for each of `batch`
 * matrices A (m x n): Q (m x n) with orthonormal columns, R (n x n) upper
 * triangular with a non-negative diagonal (so the factorisation is the unique
 * one when A has full column rank). fp32 arithmetic (Householder reflections
 * on row tiles of 128, a binary tree of stacked R pairs above them).
 *   F             bf16 DEVICE, read only: element (i, j) of matrix b (row i < m,
 *                 column j < n) at F[b*batch_stride + j*ld + i], i.e. column j
 *                 is a row of an adapter pool (A_pool or B_pool rows of one
 *                 adapter of rank n: A's m = d_in, B^T's m = d_out)
 *   ld            elements between consecutive columns, >= m
 *   batch_stride  elements between consecutive matrices, >= 0
 *   batch, m, n   1 <= n <= 64, n <= m <= 2^31, batch * m * n <= 2^40
 *   R             fp32 DEVICE [batch][n][n] row-major (zeros below the diagonal), caller-owned
 *   Q             fp32 DEVICE [batch][n][m], column j of matrix b at Q + (b*n + j)*m
 *                 (the layout of F), caller-owned; NULL computes R only
 *   workspace     DEVICE scratch of lora_tsqr_workspace_size(batch, m, n, Q != NULL)
 *                 bytes (may be 0 bytes: then NULL is accepted), caller-owned;
 *                 used until the call's kernels complete on `stream`
 * Stream-ordered; returns once the launches are queued. A zero column gives a
 * zero diagonal entry of R (and a column of Q that is still orthonormal to the
 * others).
 * Errors: LORA_ERR_ARG (null F or R, sizes out of range, ld < m),
 * LORA_ERR_WORKSPACE (workspace missing or too small), LORA_ERR_UNSUPPORTED,
 * LORA_ERR_CUDA. */
size_t lora_tsqr_workspace_size(int64_t batch, int64_t m, int32_t n, int want_q);
int lora_tsqr(const uint16_t *F, int64_t ld, int64_t batch_stride, int64_t batch, int64_t m, int32_t n, float *R,
              float *Q, void *workspace, size_t workspace_bytes, lora_stream_t stream);

/* Post-hoc compression of adapter modules ("LoRAForge：压缩与执行协同，让多LoRA
 * 服务更高效": section 核心设计, the retained-rank representation and the
 * LoRAForge-U / LoRAForge-S allocation policies; section FlashTSQR, the factor
 * construction; the note on spectral energy). A module's update A·B (A: d_in x r,
 * B: r x d_out) is, with A = Q_A·R_A and B^T = Q_B·R_B (lora_tsqr's QR),
 * Q_A·M·Q_B^T with the r x r core M = R_A·R_B^T = U·diag(sigma)·V^T: sigma is the
 * update's spectrum, and A'·B' with A' = Q_A·U_k·diag(sigma_k)^½ and
 * B' = diag(sigma_k)^½·V_k^T·Q_B^T is its best rank-k approximation. Three
 * stream-ordered calls:
 *
 * lora_compress_spectra: the factor QRs and the core SVD (one-sided Jacobi, fp32)
 * of a group of n_modules modules that share d_in, d_out and r.
 *   A_rows     bf16 DEVICE: module b's A as r pool rows of d_in at A_rows + b*a_bstride
 *              (row j = column j of A, the layout of A_pool)
 *   B_rows     bf16 DEVICE: module b's B as r pool rows of d_out at B_rows + b*b_bstride
 *   r          1 .. 64, r <= d_in, r <= d_out
 *   sigma      fp32 DEVICE [n_modules][r], caller-owned: the spectrum, descending
 *   workspace  DEVICE, lora_compress_workspace_size(n_modules, d_in, d_out, r) bytes,
 *              caller-owned: it holds the factorisation for lora_compress_export
 *              (about 4·n_modules·r·(d_in + d_out) bytes); keep it until then
 *
 * lora_compress_allocate: the retained rank of each of n_modules modules (of any
 * groups: sigma rows padded with zeros to r_max), on the device.
 *   sigma [n_modules][r_max] fp32, ranks [n_modules] int32, costs [n_modules] int64
 *              (parameters per retained rank, d_in + d_out): DEVICE
 *   policy     0: LoRAForge-U, k_b = clamp(ceil(keep·r_b), min(k_floor, r_b), r_b);
 *              1: LoRAForge-S, a budget of floor(keep·sum r_b·c_b) parameters:
 *              every module first keeps min(k_floor, r_b) ranks, then ranks are
 *              taken by the largest (sigma_bi² / sum_j sigma_bj²) / c_b (float32;
 *              equal values by module, then rank index) while their costs fit,
 *              up to the first that does not
 *   keep       in [0, 1]; k_floor >= 0
 *   k          int32 DEVICE [n_modules]; offsets int64 DEVICE [n_modules + 1] (the
 *              exclusive prefix sum of k: each module's first row in new pools)
 *   workspace  DEVICE, lora_compress_allocate_workspace_size(n_modules, r_max)
 *              bytes (policy 1 only; may be NULL for policy 0)
 *
 * lora_compress_export: the truncated factors of a group, written rank-exact:
 * module b's A' as k[b] rows (k[b] <= r; more are not written) of d_in at row
 * offsets[b] of A_new, B' as k[b] rows
 * of d_out at row offsets[b] of B_new (bf16, caller-owned DEVICE pools). sigma,
 * k, offsets are this group's (pointers to its first module); the workspace
 * is the one lora_compress_spectra filled for this group (it is not changed,
 * so several exports may follow one spectra call).
 *
 * Errors: LORA_ERR_ARG (null pointers, sizes out of range, policy, keep),
 * LORA_ERR_WORKSPACE, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA. */
size_t lora_compress_workspace_size(int64_t n_modules, int64_t d_in, int64_t d_out, int32_t r);
int lora_compress_spectra(const uint16_t *A_rows, int64_t a_bstride, const uint16_t *B_rows, int64_t b_bstride,
                          int64_t n_modules, int64_t d_in, int64_t d_out, int32_t r, float *sigma, void *workspace,
                          size_t workspace_bytes, lora_stream_t stream);
size_t lora_compress_allocate_workspace_size(int64_t n_modules, int32_t r_max);
int lora_compress_allocate(const float *sigma, const int32_t *ranks, const int64_t *costs, int64_t n_modules,
                           int32_t r_max, int32_t policy, double keep, int32_t k_floor, int32_t *k, int64_t *offsets,
                           void *workspace, size_t workspace_bytes, lora_stream_t stream);
int lora_compress_export(const float *sigma, const int32_t *k, const int64_t *offsets, int64_t n_modules, int64_t d_in,
                         int64_t d_out, int32_t r, uint16_t *A_new, uint16_t *B_new, void *workspace,
                         size_t workspace_bytes, lora_stream_t stream);

/* Test hook: write the dropout mask the forward and backward use (dropout on
 * the LoRA-branch input, one of the small ops the LoRAFusion explainer lists in
 * section 解决什么真问题, item 1; the drop rule is the one under lora_linear_fwd).
 *   mask_dev  uint8 [T, d_in] device: 1 where X[t, i] is dropped, else 0.
 * Errors: LORA_ERR_ARG, LORA_ERR_CUDA. */
int lora_dropout_mask(uint64_t seed, double p_drop, int64_t T, int64_t d_in, uint8_t *mask_dev,
                      lora_stream_t stream);

/* The same mask as keep bits, for lora_linear_fwd / lora_linear_bwd's
 * keep_bits argument: word t*ceil(d_in/32) + w of bits_dev (u32, DEVICE,
 * 4-byte aligned, caller-owned) holds columns 32w .. 32w+31 of token t, bit i
 * set iff column 32w+i is KEPT; bits past d_in are 0. One pass of the generator
 * over the T x d_in elements, so that the forward's shrink, the backward's dX
 * epilogue and its dA contraction read the mask instead of each re-deriving it
 * (the dropout definition is the one under lora_linear_fwd's p_drop; the pages
 * fix no generator, this one is a reading of them, not a counterpart).
 * Errors: LORA_ERR_ARG, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA. */
int lora_dropout_keep_bits(uint64_t seed, double p_drop, int64_t T, int64_t d_in, uint32_t *bits_dev,
                           lora_stream_t stream);

/* The seed that gives rows t0 .. t0+T-1 of a [T_global, d_in] input the dropout
 * mask they have in the global input under `seed`: a data-parallel rank whose
 * batch is those rows of a global batch passes it to lora_linear_fwd,
 * lora_linear_bwd and lora_dropout_keep_bits and indexes its rows from 0. The
 * mask's generator state for element index n is seed + (n + 1)·g (g the
 * generator's increment, arithmetic mod 2^64), so shifting n by t0·d_in is
 * adding t0·d_in·g to the seed. Host only (no CUDA call); t0 >= 0, d_in >= 1,
 * else returns `seed` unchanged. No counterpart in the pages (the pages fix no
 * generator and no sharding). */
uint64_t lora_dropout_seed_for_rows(uint64_t seed, int64_t t0, int64_t d_in);

/* Test hook for failure detection: launch one thread that waits on an mbarrier
 * nothing will complete, with a wait limit of `limit_us` microseconds (1 ..
 * 10^6). The wait runs out, sets LORA_DEV_TIMEOUT in the status word and the
 * kernel returns normally, so the context stays usable; `*waited_ok_dev`
 * (device int) receives 0. This is the same bounded wait every kernel of the
 * library uses on its pipeline barriers.
 * Errors: LORA_ERR_ARG, LORA_ERR_CUDA. */
int lora_selftest_bounded_wait(uint32_t limit_us, int *waited_ok_dev, lora_stream_t stream);

/* Synchronise `stream`, then read and clear the current device's status word.
 * No counterpart in the pages (this library's failure reporting).
 *   status_host  receives the LORA_DEV_* bits (0 if all kernels ran cleanly); may be NULL
 * Returns LORA_OK if the word was 0, LORA_ERR_DEVICE if any bit was set,
 * LORA_ERR_CUDA if the synchronisation failed. */
int lora_device_status(lora_stream_t stream, uint32_t *status_host);

/* Static string for a status code (never NULL). No counterpart in the pages. */
const char *lora_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* LORA_B200_H */
