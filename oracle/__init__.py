"""CPU oracle for the multi-adapter LoRA linear layer (ctypes wrapper).

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(the CUDA library and its binding) never imports it and shares no code with it.

Functions follow the definitions cited in ``lora_oracle.c``; all arithmetic
is fp64 over exactly widened bf16 inputs. Parity pins live in
``tests/test_oracle.py``.
"""

from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lora_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_u64 = ctypes.c_uint64
_dbl = ctypes.c_double
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_splitmix64_at.restype = _u64
        L.oracle_splitmix64_at.argtypes = [_u64, _u64]
        L.oracle_splitmix64_next.restype = _u64
        L.oracle_splitmix64_next.argtypes = [ctypes.POINTER(_u64)]
        L.oracle_drop_threshold.restype = _u64
        L.oracle_drop_threshold.argtypes = [_dbl]
        L.oracle_mask.restype = None
        L.oracle_mask.argtypes = [_u64, _dbl, _i64, _i64, _vp]
        L.oracle_plan.restype = ctypes.c_int
        L.oracle_plan.argtypes = [_vp, _i64, _i32, _vp, _vp, _vp]
        L.oracle_fwd.restype = None
        L.oracle_fwd.argtypes = [_i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _dbl, _u64, _vp, _i64, _vp, _vp, _i64]
        L.oracle_bwd.restype = None
        L.oracle_bwd.argtypes = [_i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _dbl, _u64, _vp, _vp, _i64, _vp, _vp, _vp]
        L.oracle_switch.restype = None
        L.oracle_switch.argtypes = [_i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp]
        L.oracle_qr.restype = None
        L.oracle_qr.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_num_threads.argtypes = []
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def splitmix64_at(seed: int, n: int) -> int:
    return int(lib().oracle_splitmix64_at(seed & (2**64 - 1), n))


def splitmix64_stream(seed: int, count: int) -> list[int]:
    st = _u64(seed & (2**64 - 1))
    return [int(lib().oracle_splitmix64_next(ctypes.byref(st))) for _ in range(count)]


def drop_threshold(p: float) -> int:
    return int(lib().oracle_drop_threshold(float(p)))


def mask(seed: int, p: float, T: int, d_in: int) -> np.ndarray:
    """uint8 [T, d_in]: 1 where the LoRA-branch input element is dropped."""
    out = np.empty((T, d_in), dtype=np.uint8)
    lib().oracle_mask(seed, float(p), T, d_in, _p(out))
    return out


def plan(ids, n_adapters: int):
    """(perm int32[T], segments int32[n_seg, 3] of (adapter, start, length))."""
    ids = _c(ids, np.int32)
    T = ids.shape[0]
    perm = np.empty(T, dtype=np.int32)
    seg = np.empty((max(1, min(T, n_adapters)), 3), dtype=np.int32)
    ns = _i32(0)
    rc = lib().oracle_plan(_p(ids), T, n_adapters, _p(perm), _p(seg), ctypes.cast(ctypes.pointer(ns), _vp))
    if rc != 0:
        raise ValueError("adapter id out of range")
    return perm, seg[: ns.value].copy()


def _common(inp):
    return (_c(inp.ids, np.int32), _c(inp.ranks, np.int32), _c(inp.scale, np.float32),
            _c(inp.X, np.uint16), _c(inp.W, np.uint16), _c(inp.A_pool, np.uint16),
            _c(inp.B_pool, np.uint16))


def forward(inp, rows=None, p=None, seed=None, want_u=False):
    """Y (fp64 [n_rows, d_out]) and optionally U (fp64 [n_rows, r_max]) for the
    given original token rows (default: all)."""
    ids, ranks, scale, X, W, A, B = _common(inp)
    rows = np.arange(inp.T, dtype=np.int64) if rows is None else _c(rows, np.int64)
    p = inp.p_drop if p is None else p
    seed = inp.mask_seed if seed is None else seed
    Y = np.empty((rows.shape[0], inp.d_out), dtype=np.float64)
    rmax = int(ranks.max()) if ranks.size else 1
    U = np.empty((rows.shape[0], rmax), dtype=np.float64) if want_u else None
    lib().oracle_fwd(inp.T, inp.d_in, inp.d_out, ranks.shape[0], _p(ids), _p(ranks), _p(scale),
                     _p(X), _p(W), _p(A), _p(B), float(p), seed, _p(rows), rows.shape[0],
                     _p(Y), _p(U), rmax)
    return (Y, U) if want_u else Y


def backward(inp, rows=None, p=None, seed=None, dY=None, want_dAB=True):
    """dX rows (fp64 [n_rows, d_in]), dA_pool (fp64 [sum r, d_in]) and
    dB_pool (fp64 [sum r, d_out])."""
    ids, ranks, scale, X, W, A, B = _common(inp)
    dY = _c(inp.dY if dY is None else dY, np.uint16)
    rows = np.arange(inp.T, dtype=np.int64) if rows is None else _c(rows, np.int64)
    p = inp.p_drop if p is None else p
    seed = inp.mask_seed if seed is None else seed
    R = int(ranks.sum())
    dX = np.empty((rows.shape[0], inp.d_in), dtype=np.float64)
    dA = np.empty((R, inp.d_in), dtype=np.float64) if want_dAB else None
    dB = np.empty((R, inp.d_out), dtype=np.float64) if want_dAB else None
    lib().oracle_bwd(inp.T, inp.d_in, inp.d_out, ranks.shape[0], _p(ids), _p(ranks), _p(scale),
                     _p(X), _p(W), _p(A), _p(B), float(p), seed, _p(dY), _p(rows), rows.shape[0],
                     _p(dX), _p(dA), _p(dB))
    return dX, dA, dB


def switch(W, A_pool, B_pool, ranks, term_adapter, term_coef):
    """Fused adapter switch of every layer (see oracle_switch): W uint16 bf16 bits
    [L, d_in, d_out], A_pool [L, R, d_in], B_pool [L, R, d_out]; returns the
    unrounded fp64 [L, d_in, d_out]."""
    W = _c(W, np.uint16)
    L, d_in, d_out = W.shape
    ranks = _c(ranks, np.int32)
    ta = _c(term_adapter, np.int32)
    tc = _c(term_coef, np.float64)
    out = np.empty((L, d_in, d_out), dtype=np.float64)
    lib().oracle_switch(L, d_in, d_out, ranks.shape[0], _p(ranks), _p(W), _p(_c(A_pool, np.uint16)),
                        _p(_c(B_pool, np.uint16)), ta.shape[0], _p(ta), _p(tc), _p(out))
    return out


def qr(A, want_q=True):
    """Householder QR of each matrix of A (fp64 [batch, m, n], or [m, n]): R
    [batch, n, n] and Q [batch, m, n] (see oracle_qr)."""
    A = np.asarray(A, dtype=np.float64)
    single = A.ndim == 2
    A = _c(A[None] if single else A, np.float64)
    b, m, n = A.shape
    R = np.empty((b, n, n), dtype=np.float64)
    Q = np.empty((b, m, n), dtype=np.float64) if want_q else None
    lib().oracle_qr(b, m, n, _p(A), _p(R), _p(Q))
    if single:
        return R[0], (Q[0] if want_q else None)
    return R, Q


# --------------------------------------------------------------------------- post-hoc compression
# "LoRAForge：压缩与执行协同，让多LoRA服务更高效": post-hoc compression keeps a
# module's update A·B (A: d_in x r, B: r x d_out) in a retained rank k (核心设计:
# the explicit retained-rank representation; FlashTSQR section: the factor
# construction by QR; the spectral-energy note: a module's singular values and
# their cumulative energy). The steps below are that reading, in fp64.

def compress_spectra(A_rows, B_rows):
    """Factor construction and spectrum of each module: A_rows [n, r, d_in] and
    B_rows [n, r, d_out] (bf16 bits, or floats), module b's A = A_rows[b]^T and
    B = B_rows[b]. A = Q_A·R_A and B^T = Q_B·R_B (Householder, oracle_qr), so
    A·B = Q_A·(R_A·R_B^T)·Q_B^T with orthonormal Q_A, Q_B: the singular values of
    A·B are those of the r x r core M = R_A·R_B^T. Returns (sigma [n, r]
    descending, U, V [n, r, r] with M = U·diag(sigma)·V^T, Q_A [n, d_in, r],
    Q_B [n, d_out, r]). The SVD of the small core is numpy's (a library step)."""
    def f64(a):
        a = np.asarray(a)
        if a.dtype == np.uint16:
            a = (a.astype(np.uint32) << 16).view(np.float32)
        return a.astype(np.float64)
    A = f64(A_rows).transpose(0, 2, 1)
    Bt = f64(B_rows).transpose(0, 2, 1)
    RA, QA = qr(A)
    RB, QB = qr(Bt)
    M = RA @ RB.transpose(0, 2, 1)
    U, s, Vt = np.linalg.svd(M)
    return s, U, Vt.transpose(0, 2, 1), QA, QB


def allocate(sigma, ranks, costs, policy: str, keep: float, k_floor: int):
    """Retained ranks of n modules (LoRAForge article, 核心设计: LoRAForge-U, the
    same retention ratio for every module; LoRAForge-S, a budget spent by each
    module's cumulative spectral energy). The rule, in float32 arithmetic so that
    a caller holding the same float32 singular values decides identically:
      U: k_b = clamp(ceil(keep * r_b), floor_b, r_b), floor_b = min(k_floor, r_b).
      S: the budget P = floor(keep * sum_b r_b * c_b) parameters (c_b = the
         parameters per retained rank of module b, d_in + d_out); every module
         first keeps floor_b ranks; each further rank i >= floor_b of module b
         scores g = (sigma_bi^2 / E_b) / c_b, E_b = sum_j sigma_bj^2 (summed in
         j order; g = 0 when E_b = 0); the ranks are taken in the order of g
         (largest first; equal g by module, then by i) while their costs fit in
         P - sum floor_b * c_b, up to the first that does not fit. g falls with
         i, so a module keeps a prefix of its ranks.
    sigma: float32 [n, r_max] (descending in each row, zeros past r_b); ranks,
    costs: [n] integers. Returns k [n] (int32) and offsets [n + 1] (int64, the
    exclusive prefix sum of k: each module's first row in the new pools)."""
    sigma = np.asarray(sigma, dtype=np.float32)
    ranks = np.asarray(ranks, dtype=np.int64)
    costs = np.asarray(costs, dtype=np.int64)
    n = sigma.shape[0]
    floors = np.minimum(ranks, k_floor)
    if policy == "U":
        k = np.array([min(int(ranks[b]), max(int(floors[b]), math.ceil(keep * int(ranks[b]))))
                      for b in range(n)], dtype=np.int64)
    elif policy == "S":
        budget = math.floor(keep * float(int((ranks * costs).sum())))
        left = budget - int((floors * costs).sum())
        items = []  # (key, b, i, cost)
        for b in range(n):
            e = np.float32(0.0)
            for j in range(int(ranks[b])):
                e = np.float32(e + np.float32(sigma[b, j]) * np.float32(sigma[b, j]))
            for i in range(int(floors[b]), int(ranks[b])):
                sq = np.float32(np.float32(sigma[b, i]) * np.float32(sigma[b, i]))
                g = np.float32(np.float32(sq / e) / np.float32(costs[b])) if e > 0 else np.float32(0.0)
                items.append((int(np.array(g, dtype=np.float32).view(np.uint32)), b, i, int(costs[b])))
        k = floors.copy()
        total = 0
        for key, b, i, c in sorted(items, key=lambda t: (-t[0], t[1], t[2])):
            if total + c > left:
                break
            total += c
            k[b] += 1
    else:
        raise ValueError(policy)
    offsets = np.concatenate([[0], np.cumsum(k)]).astype(np.int64)
    return k.astype(np.int32), offsets


def export(sigma, U, V, QA, QB, k):
    """The truncated factors of each module: A'_b = Q_A·U_k·diag(sqrt(sigma_k))
    (d_in x k) and B'_b = diag(sqrt(sigma_k))·V_k^T·Q_B^T (k x d_out), so that
    A'_b·B'_b is the best rank-k approximation of A_b·B_b (Eckart-Young).
    Returns lists of fp64 arrays, A' as pool rows [k, d_in], B' [k, d_out]."""
    A_new, B_new = [], []
    for b in range(sigma.shape[0]):
        kb = int(k[b])
        sq = np.sqrt(sigma[b, :kb])
        A_new.append(((QA[b] @ U[b][:, :kb]) * sq[None, :]).T)
        B_new.append(((QB[b] @ V[b][:, :kb]) * sq[None, :]).T)
    return A_new, B_new
