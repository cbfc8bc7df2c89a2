"""Seeded synthetic inputs for the multi-adapter LoRA linear layer.

This module only draws numbers: it holds none of the layer's arithmetic, so
both the CPU oracle (``oracle/``) and the CUDA path can consume its arrays
without sharing any compute code.

Workloads (sizes and distributions as stated for the heterogeneous LoRA layer
Y[t] = X[t]·W + s_a·(X[t]·A_a)·B_a, where a is token t's adapter):

  tiny      T=64, d_in=d_out=256, ranks {4,8,8,16}, s=16/r, ids uniform over 4
  decode    T=256, 4096x4096, 64 adapters of rank 16, s=2, ids uniform over 64
  prefill   T=8192, 4096->11008, 200 adapters, ranks from {8,16,32,64},
            Zipf(1.0) adapter per 512-token request, s=16/r
  fleet     T=4096, 4096x4096, 1000 adapters, ranks uniform 1..21, row k of B_a
            scaled by 1/k, Zipf(1.2) adapter per token, s=16/r
  finetune  T=16384, 4096x4096, 1 adapter of rank 16, s=2, dropout p=0.1,
            plus an upstream gradient dY ~ N(0,1)
  fleet_finetune  the fleet batch with dropout p=0.1 and dY ~ N(0,1): one
            fine-tuning step of all its adapters at once

Readings where the pages are silent:
  * X ~ N(0,1), W ~ N(0,1/d_in), A ~ N(0,1/d_in), B_a ~ N(0,1/r_a) for every
    workload (only the tiny and decode workloads state it).
  * s_a = 16/r_a where no scale is given (prefill, fleet).
  * Zipf is finite: P(k) ∝ k^-alpha over k=1..N, adapter id k-1; ranks are drawn
    independently of popularity.
  * "ranks 1..21" is read as uniform over the integers 1..21 inclusive.
  * Every array is drawn from numpy's default_rng(seed) in fp32 in the fixed
    order ranks, ids, X, W, A, B, dY and rounded to bf16 (round to nearest
    even). bf16 arrays are returned as their uint16 bit patterns.

Factor layout ("rank-exact pool", S-LoRA page, Unified Paging section: a rank-R
weight occupies R vectors of the hidden size): adapter a owns rows
[off_a, off_a + r_a) of A_pool (each row a column of A_a, i.e. A_a^T, length
d_in) and of B_pool (rows of B_a, length d_out), with off_a the exclusive
prefix sum of the ranks in adapter-id order. Nothing is padded.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

WORKLOADS = ("tiny", "decode", "prefill", "fleet", "finetune", "fleet_finetune")


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Spec:
    name: str
    T: int
    d_in: int
    d_out: int
    n_adapters: int
    rank_choice: tuple            # ("fixed", r) | ("set", (..)) | ("range", lo, hi) | ("list", (..))
    ids: tuple                    # ("uniform",) | ("zipf_request", alpha, req_len) | ("zipf_token", alpha) | ("single",)
    scale: object                 # float, or "16/r"
    b_row_decay: bool = False     # multiply row k (1-based) of B_a by 1/k
    p_drop: float = 0.0
    with_dy: bool = False
    seed: int = 0
    mask_seed: int = 0


SPECS = {
    "tiny": Spec("tiny", 64, 256, 256, 4, ("list", (4, 8, 8, 16)), ("uniform",), "16/r"),
    "decode": Spec("decode", 256, 4096, 4096, 64, ("fixed", 16), ("uniform",), 2.0),
    "prefill": Spec("prefill", 8192, 4096, 11008, 200, ("set", (8, 16, 32, 64)),
                    ("zipf_request", 1.0, 512), "16/r"),
    "fleet": Spec("fleet", 4096, 4096, 4096, 1000, ("range", 1, 21), ("zipf_token", 1.2),
                  "16/r", b_row_decay=True),
    "finetune": Spec("finetune", 16384, 4096, 4096, 1, ("fixed", 16), ("single",), 2.0,
                     p_drop=0.1, with_dy=True),
    # the fleet batch as one multi-adapter fine-tuning step (every adapter trained)
    "fleet_finetune": Spec("fleet_finetune", 4096, 4096, 4096, 1000, ("range", 1, 21), ("zipf_token", 1.2),
                           "16/r", b_row_decay=True, p_drop=0.1, with_dy=True),
}


@dataclass
class Inputs:
    spec: Spec
    T: int
    d_in: int
    d_out: int
    ranks: np.ndarray        # int32 [n_adapters]
    ids: np.ndarray          # int32 [T]
    scale: np.ndarray        # float32 [n_adapters]
    X: np.ndarray            # uint16 (bf16 bits) [T, d_in]
    W: np.ndarray            # uint16 [d_in, d_out]
    A_pool: np.ndarray       # uint16 [sum r, d_in]   (rows = columns of A_a)
    B_pool: np.ndarray       # uint16 [sum r, d_out]  (rows of B_a)
    dY: np.ndarray | None    # uint16 [T, d_out]
    p_drop: float
    mask_seed: int
    offsets: np.ndarray = field(default=None)  # int64 [n_adapters+1] exclusive prefix of ranks

    @property
    def n_adapters(self) -> int:
        return int(self.ranks.shape[0])


def _zipf_probs(n: int, alpha: float) -> np.ndarray:
    k = np.arange(1, n + 1, dtype=np.float64)
    w = k ** (-alpha)
    return w / w.sum()


def _normal_bf16(rng, shape, std) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def make_inputs(spec: Spec | str, *, T: int | None = None, d_in: int | None = None,
                d_out: int | None = None, n_adapters: int | None = None,
                seed: int | None = None, with_dy: bool | None = None,
                p_drop: float | None = None) -> Inputs:
    """Draw one workload. Keyword overrides shrink a workload for quick tests
    while keeping its rank/id/scale recipe."""
    if isinstance(spec, str):
        spec = SPECS[spec]
    T = spec.T if T is None else T
    d_in = spec.d_in if d_in is None else d_in
    d_out = spec.d_out if d_out is None else d_out
    n = spec.n_adapters if n_adapters is None else n_adapters
    seed = spec.seed if seed is None else seed
    with_dy = spec.with_dy if with_dy is None else with_dy
    p = spec.p_drop if p_drop is None else p_drop
    rng = np.random.default_rng(seed)

    kind = spec.rank_choice[0]
    if kind == "fixed":
        ranks = np.full(n, spec.rank_choice[1], dtype=np.int32)
    elif kind == "list":
        lst = np.array(spec.rank_choice[1], dtype=np.int32)
        ranks = np.resize(lst, n).astype(np.int32)
    elif kind == "set":
        ranks = rng.choice(np.array(spec.rank_choice[1], dtype=np.int32), size=n).astype(np.int32)
    elif kind == "range":
        lo, hi = spec.rank_choice[1], spec.rank_choice[2]
        ranks = rng.integers(lo, hi + 1, size=n, dtype=np.int32)
    else:
        raise ValueError(kind)

    ik = spec.ids[0]
    if ik == "uniform":
        ids = rng.integers(0, n, size=T, dtype=np.int32)
    elif ik == "zipf_request":
        alpha, req = spec.ids[1], spec.ids[2]
        n_req = -(-T // req)
        req_ids = rng.choice(n, size=n_req, p=_zipf_probs(n, alpha)).astype(np.int32)
        ids = np.repeat(req_ids, req)[:T].astype(np.int32)
    elif ik == "zipf_token":
        ids = rng.choice(n, size=T, p=_zipf_probs(n, spec.ids[1])).astype(np.int32)
    elif ik == "single":
        ids = np.zeros(T, dtype=np.int32)
    else:
        raise ValueError(ik)

    if spec.scale == "16/r":
        scale = (np.float32(16.0) / ranks.astype(np.float32)).astype(np.float32)
    else:
        scale = np.full(n, spec.scale, dtype=np.float32)

    offsets = np.zeros(n + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(ranks, dtype=np.int64)
    R = int(offsets[-1])

    X = _normal_bf16(rng, (T, d_in), 1.0)
    W = _normal_bf16(rng, (d_in, d_out), float(np.sqrt(1.0 / d_in)))
    A_pool = _normal_bf16(rng, (R, d_in), float(np.sqrt(1.0 / d_in)))
    braw = rng.standard_normal((R, d_out), dtype=np.float32)
    rowscale = np.empty(R, dtype=np.float32)
    for a in range(n):
        r = int(ranks[a])
        o = int(offsets[a])
        std = np.float32(np.sqrt(1.0 / r))
        if spec.b_row_decay:
            rowscale[o:o + r] = std / np.arange(1, r + 1, dtype=np.float32)
        else:
            rowscale[o:o + r] = std
    braw *= rowscale[:, None]
    B_pool = f32_to_bf16_bits(braw)
    dY = _normal_bf16(rng, (T, d_out), 1.0) if with_dy else None
    return Inputs(spec=spec, T=T, d_in=d_in, d_out=d_out, ranks=ranks, ids=ids,
                  scale=scale, X=X, W=W, A_pool=A_pool, B_pool=B_pool, dY=dY,
                  p_drop=float(p), mask_seed=spec.mask_seed, offsets=offsets)


def integer_inputs(T: int, d_in: int, d_out: int, ranks, ids, seed: int = 0,
                   lo: int = -3, hi: int = 3) -> Inputs:
    """Small-integer-valued inputs with s=1: every product and partial sum is an
    exact integer in fp32, so any correct implementation agrees bit for bit."""
    rng = np.random.default_rng(seed)
    ranks = np.asarray(ranks, dtype=np.int32)
    ids = np.asarray(ids, dtype=np.int32)
    n = ranks.shape[0]
    offsets = np.zeros(n + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(ranks)
    R = int(offsets[-1])

    def ints(shape):
        return f32_to_bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32))

    spec = Spec("integer", T, d_in, d_out, n, ("list", tuple(int(r) for r in ranks)),
                ("uniform",), 1.0)
    return Inputs(spec=spec, T=T, d_in=d_in, d_out=d_out, ranks=ranks, ids=ids,
                  scale=np.ones(n, dtype=np.float32), X=ints((T, d_in)), W=ints((d_in, d_out)),
                  A_pool=ints((R, d_in)), B_pool=ints((R, d_out)), dY=ints((T, d_out)),
                  p_drop=0.0, mask_seed=0, offsets=offsets)


def make_rank_inputs(spec: Spec | str, rank: int, **kw) -> Inputs:
    """Rank `rank`'s share of a data-parallel run: the same layer (ranks, scales,
    W, A_pool, B_pool) on every rank, and a batch of its own (ids, X, dY) drawn
    with the workload's recipe. Rank 0's batch is the workload's own draw. The
    ranks' batches are read as consecutive shards of one global batch (rank r
    holds global rows r*T .. r*T + T - 1); the dropout seed stays the global
    one, and the caller derives the seed of its rows from it."""
    if isinstance(spec, str):
        spec = SPECS[spec]
    base = make_inputs(spec, **kw)
    if rank == 0:
        return base
    kw2 = dict(kw)
    kw2["seed"] = (spec.seed if kw.get("seed") is None else kw["seed"]) + 7919 * rank
    other = make_inputs(spec, **kw2)
    return Inputs(spec=spec, T=base.T, d_in=base.d_in, d_out=base.d_out, ranks=base.ranks, ids=other.ids,
                  scale=base.scale, X=other.X, W=base.W, A_pool=base.A_pool, B_pool=base.B_pool, dY=other.dY,
                  p_drop=base.p_drop, mask_seed=base.mask_seed, offsets=base.offsets)


def factor_stack(batch: int, m: int, n: int, *, seed: int = 0, decay: float = 1.0) -> np.ndarray:
    """Adapter factors as a stack of pools, for the tall-skinny QR: bf16 bit
    patterns [batch, n, m], matrix b's column j in row [b, j] (an adapter pool's
    row layout). Entries N(0, 1/m); column j scaled by decay**j (decay < 1 gives
    the decaying spectrum of a trained factor: condition number about decay**(1-n))."""
    rng = np.random.default_rng(seed)
    F = rng.standard_normal((batch, n, m)).astype(np.float32) / np.float32(np.sqrt(m))
    F *= (np.float32(decay) ** np.arange(n, dtype=np.float32))[None, :, None]
    return f32_to_bf16_bits(F)


def module_factors(n: int, r: int, d_in: int, d_out: int, *, seed: int = 0, decay=(0.6, 0.95)):
    """Trained-like factors of n modules for post-hoc compression, as bf16 bit
    patterns in pool-row layout: A_rows [n, r, d_in] with entries N(0, 1/d_in)
    (LoRA's A scale) and B_rows [n, r, d_out] with entries N(0, 1) times
    decay_b**j on row j, decay_b uniform in `decay` per module, so the modules'
    spectra fall off at different rates (the spread a spectral budget reads)."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((n, r, d_in)).astype(np.float32) / np.float32(np.sqrt(d_in))
    dec = rng.uniform(decay[0], decay[1], size=n).astype(np.float32)
    B = rng.standard_normal((n, r, d_out)).astype(np.float32)
    B *= dec[:, None, None] ** np.arange(r, dtype=np.float32)[None, :, None]
    return f32_to_bf16_bits(A), f32_to_bf16_bits(B)
