"""Pins for the CPU oracle: each test checks the oracle against something other
than itself (a published vector, an exact computation, a closed form, an
invariant, a different formula, or brute force), chosen so that a dropped term,
a wrong index or a transposed operand fails at least one of them.

CPU only (no GPU marker)."""

from __future__ import annotations

import dataclasses
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from lora_adapter_execution_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(b):
    return wl.bf16_bits_to_f32(b).astype(np.float64)


def bf(x):
    return wl.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def small(name="tiny", **kw):
    return wl.make_inputs(name, **kw)


def merged_reference(inp, rows=None):
    """Y via the merged-weight form X·(W + s_a·A_a·B_a) (S-LoRA article,
    batching section, formula 1), numpy fp64 matmul: a different formula from
    the oracle's unmerged X·W + s·(X·A)·B (formula 2)."""
    X, W, A, B = f32(inp.X), f32(inp.W), f32(inp.A_pool), f32(inp.B_pool)
    rows = np.arange(inp.T) if rows is None else np.asarray(rows)
    Y = np.empty((rows.size, inp.d_out))
    for q, t in enumerate(rows):
        a = int(inp.ids[t])
        o, r = int(inp.offsets[a]), int(inp.ranks[a])
        Wm = W + float(inp.scale[a]) * (A[o:o + r].T @ B[o:o + r])
        Y[q] = X[t] @ Wm
    return Y


# ------------------------------------------------------------------ SplitMix64

def test_splitmix64_published_vectors():
    want = []
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                i, v = line.split()
                want.append((int(i), int(v, 16)))
    stream = oracle.splitmix64_stream(0, len(want))
    for i, v in want:
        assert stream[i] == v
        assert oracle.splitmix64_at(0, i) == v


def test_splitmix64_direct_index_matches_stream():
    for seed in (0, 1, 12345, 2**63 + 7):
        s = oracle.splitmix64_stream(seed, 50)
        assert [oracle.splitmix64_at(seed, n) for n in range(50)] == s


def test_drop_threshold_exact():
    for p in (0.1, 0.5, 0.25, 1e-3, 0.9):
        assert oracle.drop_threshold(p) == int(Fraction(p) * 2**64)
    assert oracle.drop_threshold(0.0) == 0
    assert oracle.drop_threshold(0.5) == 2**63


def test_mask_fraction_binomial():
    T, d, p = 512, 512, 0.1
    m = oracle.mask(0, p, T, d)
    n = m.size
    frac = m.mean()
    sigma = np.sqrt(p * (1 - p) / n)
    assert abs(frac - p) < 5 * sigma
    assert oracle.mask(0, 0.0, 8, 16).sum() == 0
    # different seeds give different masks
    assert (oracle.mask(1, p, 64, 64) != oracle.mask(0, p, 64, 64)).any()


def test_mask_element_definition():
    # element (t, col) is the (t*d_in + col)-th generator output compared to the threshold
    T, d, p, seed = 3, 7, 0.3, 99
    m = oracle.mask(seed, p, T, d)
    thr = int(Fraction(p) * 2**64)
    stream = oracle.splitmix64_stream(seed, T * d)
    want = np.array([1 if h < thr else 0 for h in stream], dtype=np.uint8).reshape(T, d)
    assert (m == want).all()


# ------------------------------------------------------------------ plan

@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "fleet", "finetune"])
def test_plan_matches_stable_sort(name):
    spec = wl.SPECS[name]
    inp = wl.make_inputs(spec, d_in=16, d_out=16)  # plan depends on ids only
    perm, seg = oracle.plan(inp.ids, inp.n_adapters)
    want = sorted(range(inp.T), key=lambda t: (int(inp.ids[t]), t))
    assert perm.tolist() == want
    assert (np.argsort(inp.ids, kind="stable") == perm).all()
    # segments: ascending adapter, contiguous, lengths = counts, no empty segment
    counts = np.bincount(inp.ids, minlength=inp.n_adapters)
    used = np.nonzero(counts)[0]
    assert seg[:, 0].tolist() == used.tolist()
    assert seg[:, 2].tolist() == counts[used].tolist()
    starts = np.concatenate([[0], np.cumsum(counts[used])[:-1]])
    assert seg[:, 1].tolist() == starts.tolist()


def test_plan_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.plan(np.array([0, 4, 1], dtype=np.int32), 4)
    with pytest.raises(ValueError):
        oracle.plan(np.array([-1], dtype=np.int32), 4)


def test_workload_statistics():
    # the recipe reproduces the segment statistics the workloads imply
    dec = wl.make_inputs("decode", d_in=16, d_out=16)
    _, seg = oracle.plan(dec.ids, 64)
    assert 55 <= seg.shape[0] <= 64
    pre = wl.make_inputs("prefill", d_in=16, d_out=16)
    _, seg = oracle.plan(pre.ids, 200)
    assert all(int(s[2]) % 512 == 0 for s in seg)
    assert set(np.unique(pre.ranks)).issubset({8, 16, 32, 64})
    fl = wl.make_inputs("fleet", d_in=16, d_out=16)
    assert fl.ranks.min() >= 1 and fl.ranks.max() <= 21


# ------------------------------------------------------------------ forward

@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("decode", dict(T=40, d_in=64, d_out=48, n_adapters=8)),
    ("prefill", dict(T=64, d_in=32, d_out=80, n_adapters=10)),
    ("fleet", dict(T=50, d_in=48, d_out=40, n_adapters=30)),
])
def test_forward_merged_equivalence(name, kw):
    inp = wl.make_inputs(name, **kw)
    Y = oracle.forward(inp)
    Ym = merged_reference(inp)
    assert np.allclose(Y, Ym, rtol=1e-12, atol=1e-12 * np.abs(Ym).max())


def test_forward_B_zero_is_base_exactly():
    inp = small(T=16, d_in=32, d_out=24)
    inp = dataclasses.replace(inp, B_pool=np.zeros_like(inp.B_pool))
    Y = oracle.forward(inp)
    # integer-free check: compare with numpy fp64 X·W; bf16 products are exact
    # in fp64 and the sums here are short, so agreement is to rounding only
    ref = f32(inp.X) @ f32(inp.W)
    assert np.allclose(Y, ref, rtol=1e-14, atol=1e-14)
    iinp = wl.integer_inputs(8, 16, 12, [3, 5], [0, 1, 1, 0, 1, 0, 0, 1])
    iinp = dataclasses.replace(iinp, B_pool=np.zeros_like(iinp.B_pool))
    assert (oracle.forward(iinp) == f32(iinp.X) @ f32(iinp.W)).all()


def test_forward_token_permutation_invariance():
    inp = small()
    rng = np.random.default_rng(5)
    pi = rng.permutation(inp.T)
    inp2 = dataclasses.replace(inp, X=inp.X[pi].copy(), ids=inp.ids[pi].copy())
    assert (oracle.forward(inp2) == oracle.forward(inp)[pi]).all()


def test_forward_adapter_relabel_invariance():
    inp = small()
    n = inp.n_adapters
    sigma = np.array([2, 0, 3, 1])          # new label of old adapter a is sigma[a]
    inv = np.argsort(sigma)                  # old adapter holding new label b
    ranks2 = inp.ranks[inv]
    scale2 = inp.scale[inv]
    A2 = np.concatenate([inp.A_pool[inp.offsets[a]:inp.offsets[a + 1]] for a in inv])
    B2 = np.concatenate([inp.B_pool[inp.offsets[a]:inp.offsets[a + 1]] for a in inv])
    off2 = np.concatenate([[0], np.cumsum(ranks2)])
    inp2 = dataclasses.replace(inp, ids=sigma[inp.ids].astype(np.int32), ranks=ranks2.astype(np.int32),
                               scale=scale2, A_pool=A2, B_pool=B2, offsets=off2)
    assert n == 4
    assert (oracle.forward(inp2) == oracle.forward(inp)).all()


def test_forward_rank1_closed_form():
    T, d_in, d_out = 12, 20, 18
    inp = wl.make_inputs("tiny", T=T, d_in=d_in, d_out=d_out, n_adapters=3)
    ranks = np.array([1, 1, 1], dtype=np.int32)
    ei = [3, 11, 19]   # A_a = e_i (column i of the input)
    ej = [0, 7, 17]    # B_a = e_j^T
    A = np.zeros((3, d_in), dtype=np.float32)
    B = np.zeros((3, d_out), dtype=np.float32)
    for a in range(3):
        A[a, ei[a]] = 1.0
        B[a, ej[a]] = 1.0
    scale = np.array([0.5, 2.0, -3.0], dtype=np.float32)
    inp = dataclasses.replace(inp, ranks=ranks, scale=scale, A_pool=bf(A), B_pool=bf(B),
                              offsets=np.arange(4))
    Y = oracle.forward(inp)
    X = f32(inp.X)
    ref = X @ f32(inp.W)
    for t in range(T):
        a = inp.ids[t]
        ref[t, ej[a]] += float(scale[a]) * X[t, ei[a]]
    assert np.allclose(Y, ref, rtol=1e-14, atol=1e-14)


def test_forward_integer_brute_force():
    # pure-Python integer arithmetic on a tiny case: the exact answer
    T, d_in, d_out = 6, 10, 9
    ranks = [2, 3, 1]
    ids = [2, 0, 1, 1, 0, 2]
    inp = wl.integer_inputs(T, d_in, d_out, ranks, ids, seed=3)
    X = f32(inp.X).astype(int).tolist()
    W = f32(inp.W).astype(int).tolist()
    A = f32(inp.A_pool).astype(int).tolist()
    B = f32(inp.B_pool).astype(int).tolist()
    off = [0, 2, 5, 6]
    Y, U = oracle.forward(inp, want_u=True)
    for t in range(T):
        a = ids[t]
        u = [sum(X[t][i] * A[off[a] + k][i] for i in range(d_in)) for k in range(ranks[a])]
        for j in range(d_out):
            y = sum(X[t][i] * W[i][j] for i in range(d_in))
            y += sum(u[k] * B[off[a] + k][j] for k in range(ranks[a]))
            assert Y[t, j] == y
        assert U[t, :ranks[a]].tolist() == u
        assert (U[t, ranks[a]:] == 0).all()


def test_forward_dropout_branch_only():
    # p > 0 changes only the LoRA term; with B = 0 the result is the base exactly
    inp = small(T=20, d_in=40, d_out=24, p_drop=0.3)
    z = dataclasses.replace(inp, B_pool=np.zeros_like(inp.B_pool))
    assert (oracle.forward(z) == oracle.forward(z, p=0.0)).all()
    # U with dropout equals (mask-zeroed, 1/(1-p)-scaled X)·A_a
    _, U = oracle.forward(inp, want_u=True)
    m = oracle.mask(inp.mask_seed, inp.p_drop, inp.T, inp.d_in)
    Xd = f32(inp.X) * np.where(m == 1, 0.0, 1.0 / (1.0 - inp.p_drop))
    A = f32(inp.A_pool)
    for t in range(inp.T):
        a = inp.ids[t]
        o, r = int(inp.offsets[a]), int(inp.ranks[a])
        assert np.allclose(U[t, :r], Xd[t] @ A[o:o + r].T, rtol=1e-12, atol=1e-12)


def test_forward_row_subset_consistent():
    inp = small()
    rows = np.array([5, 0, 63, 17])
    assert (oracle.forward(inp, rows=rows) == oracle.forward(inp)[rows]).all()


# ------------------------------------------------------------------ backward

def _loss(inp, dY, **kw):
    return float((oracle.forward(inp, **kw) * f32(dY)).sum())


def _bump(arr_bits, idx, delta):
    f = wl.bf16_bits_to_f32(arr_bits).copy()
    f[idx] += delta
    out = bf(f)
    assert wl.bf16_bits_to_f32(out)[idx] == f[idx]
    return out


@pytest.mark.parametrize("p", [0.0, 0.25])
def test_backward_unit_step_differences(p):
    """The loss L = <dY, Y> is linear in X, in A (B fixed) and in B (A fixed),
    so a unit step on an integer input gives the exact partial derivative:
    L(v + e) - L(v) = dL/dv. Checked against the oracle's backward."""
    T, d_in, d_out = 5, 8, 7
    ranks, ids = [2, 3], [1, 0, 1, 1, 0]
    inp = wl.integer_inputs(T, d_in, d_out, ranks, ids, seed=11)
    inp = dataclasses.replace(inp, scale=np.array([2.0, -1.5], dtype=np.float32), p_drop=p,
                              mask_seed=4)
    dX, dA, dB = oracle.backward(inp)
    L0 = _loss(inp, inp.dY)
    tol = 1e-9
    for (t, i) in [(0, 0), (2, 5), (4, 7), (3, 1)]:
        L1 = _loss(dataclasses.replace(inp, X=_bump(inp.X, (t, i), 1.0)), inp.dY)
        assert abs((L1 - L0) - dX[t, i]) <= tol * max(1.0, abs(dX[t, i]))
    for (row, i) in [(0, 0), (1, 7), (2, 3), (4, 4)]:
        L1 = _loss(dataclasses.replace(inp, A_pool=_bump(inp.A_pool, (row, i), 1.0)), inp.dY)
        assert abs((L1 - L0) - dA[row, i]) <= tol * max(1.0, abs(dA[row, i]))
    for (row, j) in [(0, 0), (1, 6), (3, 2), (4, 5)]:
        L1 = _loss(dataclasses.replace(inp, B_pool=_bump(inp.B_pool, (row, j), 1.0)), inp.dY)
        assert abs((L1 - L0) - dB[row, j]) <= tol * max(1.0, abs(dB[row, j]))


def test_backward_merged_dX():
    # p = 0: dX = dY·(W + s_a A_a B_a)^T per token (merged form)
    inp = wl.make_inputs("tiny", T=24, d_in=32, d_out=40, with_dy=True)
    dX, _, _ = oracle.backward(inp, want_dAB=False)
    X, W, A, B, dY = (f32(v) for v in (inp.X, inp.W, inp.A_pool, inp.B_pool, inp.dY))
    for t in range(inp.T):
        a = inp.ids[t]
        o, r = int(inp.offsets[a]), int(inp.ranks[a])
        Wm = W + float(inp.scale[a]) * (A[o:o + r].T @ B[o:o + r])
        assert np.allclose(dX[t], dY[t] @ Wm.T, rtol=1e-12, atol=1e-12)


def test_backward_adjoint_identity():
    # <dY, J·delta> = <J^T·dY, delta> for a random direction delta in X, A, B
    inp = wl.make_inputs("finetune", T=16, d_in=24, d_out=20, p_drop=0.2)
    dX, dA, dB = oracle.backward(inp)
    rng = np.random.default_rng(9)
    # L is linear in X, so the loss difference along any direction equals the
    # inner product with dX; the direction is whatever bf16 step was representable
    step = (rng.integers(-2, 3, size=inp.X.shape) * 0.25).astype(np.float32)
    Xp = bf(wl.bf16_bits_to_f32(inp.X) + step)
    dirX = f32(Xp) - f32(inp.X)
    lhs = _loss(dataclasses.replace(inp, X=Xp), inp.dY) - _loss(inp, inp.dY)
    rhs = float((dX * dirX).sum())
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(rhs))
    assert dA.shape == (16, 24) and dB.shape == (16, 20)


def test_backward_single_adapter_closed_forms():
    # single adapter, p = 0: dB = s·U^T·dY and dA = X^T·dU with dU = s·dY·B^T
    inp = wl.make_inputs("finetune", T=20, d_in=16, d_out=12, p_drop=0.0)
    dX, dA, dB = oracle.backward(inp)
    X, A, B, dY = (f32(v) for v in (inp.X, inp.A_pool, inp.B_pool, inp.dY))
    s = float(inp.scale[0])
    U = X @ A.T
    dU = s * dY @ B.T
    assert np.allclose(dB, s * U.T @ dY, rtol=1e-12, atol=1e-12)
    assert np.allclose(dA, dU.T @ X, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ adapter switch (merge path)
def switch_inputs(L=2, d_in=24, d_out=16, ranks=(3, 5, 2, 4), seed=0, ints=False):
    """Stacked per-layer weights and factor pools, each layer its own pool with
    the same adapter offsets."""
    rng = np.random.default_rng(seed)
    ranks = np.asarray(ranks, dtype=np.int32)
    R = int(ranks.sum())
    if ints:
        draw = lambda shape: bf(rng.integers(-3, 4, size=shape).astype(np.float32))  # noqa: E731
    else:
        draw = lambda shape: bf(rng.standard_normal(shape).astype(np.float32))  # noqa: E731
    return ranks, draw((L, d_in, d_out)), draw((L, R, d_in)), draw((L, R, d_out))


def test_switch_rank1_closed_form():
    """A rank-1 adapter whose A column is e_i and B row is e_j changes exactly
    W[l, i, j] by its coefficient, in every layer, and nothing else."""
    ranks, W, A, B = switch_inputs(L=3, ranks=(1, 2))
    A[:] = 0
    B[:] = 0
    A[:, 0, 5] = bf(1.0)
    B[:, 0, 7] = bf(1.0)
    out = oracle.switch(W, A, B, ranks, [0], [-2.5])
    want = f32(W).copy()
    want[:, 5, 7] -= 2.5
    assert np.array_equal(out, want)


def test_switch_matches_numpy_sum_of_outer_products():
    """Per layer, W + sum_j c_j · A_j^T·B_j with A_j^T the pool rows of adapter j
    transposed (numpy fp64 matmul, a different order of summation)."""
    ranks, W, A, B = switch_inputs(L=3, d_in=40, d_out=28, ranks=(3, 5, 2, 4), seed=1)
    terms, coefs = [1, 3, 0], [-0.75, 1.25, 0.5]
    out = oracle.switch(W, A, B, ranks, terms, coefs)
    off = np.concatenate([[0], np.cumsum(ranks)])
    for l in range(3):
        want = f32(W[l]).copy()
        for a, c in zip(terms, coefs):
            Al, Bl = f32(A[l, off[a]:off[a + 1]]), f32(B[l, off[a]:off[a + 1]])
            want += c * (Al.T @ Bl)
        np.testing.assert_allclose(out[l], want, rtol=1e-12, atol=1e-12)


def test_switch_fused_equals_unmerge_then_merge_and_round_trip():
    """The fused switch (unmerge the previous adapters with negative weights and
    merge the current ones in one update) equals the two updates applied one
    after the other; and unmerging what was merged gives W back. Integer inputs
    make every step exact, so both hold bit for bit."""
    ranks, W, A, B = switch_inputs(L=2, ranks=(3, 5, 2, 4), ints=True, seed=2)
    prev, cur = ([0, 2], [2.0, 1.0]), ([1, 3], [1.0, 3.0])
    fused = oracle.switch(W, A, B, ranks, prev[0] + cur[0], [-c for c in prev[1]] + cur[1])
    step1 = oracle.switch(W, A, B, ranks, prev[0], [-c for c in prev[1]])
    assert np.abs(step1).max() < 256  # exact in bf16
    step2 = oracle.switch(bf(step1), A, B, ranks, cur[0], cur[1])
    assert np.array_equal(fused, step2)
    back = oracle.switch(bf(oracle.switch(W, A, B, ranks, *cur)), A, B, ranks, cur[0], [-c for c in cur[1]])
    assert np.array_equal(back, f32(W))


def test_switch_merged_weight_reproduces_the_unmerged_forward():
    """Merging an adapter with coefficient s_a into W (one layer) and running the
    plain product X·W' gives the oracle's unmerged forward for tokens of that
    adapter (S-LoRA article, batching: formula 1 against formula 2). Integer
    inputs: exact."""
    inp = wl.integer_inputs(20, 32, 24, [4, 6], np.ones(20, dtype=np.int32), seed=3, lo=-2, hi=2)
    inp = dataclasses.replace(inp, scale=np.array([1.0, 3.0], dtype=np.float32))
    Wm = oracle.switch(inp.W[None], inp.A_pool[None], inp.B_pool[None], inp.ranks, [1], [3.0])[0]
    assert np.array_equal(f32(inp.X) @ Wm, oracle.forward(inp))


# ------------------------------------------------------------------ tall-skinny QR (FlashTSQR)
def test_qr_reconstructs_and_is_orthonormal():
    """Q·R = A, Q^T·Q = I and R upper triangular, on tall random matrices."""
    rng = np.random.default_rng(5)
    A = rng.standard_normal((3, 300, 24))
    R, Q = oracle.qr(A)
    for b in range(3):
        np.testing.assert_allclose(Q[b] @ R[b], A[b], atol=1e-12)
        np.testing.assert_allclose(Q[b].T @ Q[b], np.eye(24), atol=1e-12)
        assert np.all(np.tril(R[b], -1) == 0)


def test_qr_matches_numpy_up_to_row_signs():
    """R is unique up to the sign of each row (Q up to the sign of each column):
    the oracle's R against numpy's (LAPACK) after making both diagonals positive."""
    rng = np.random.default_rng(6)
    A = rng.standard_normal((200, 17))
    R, Q = oracle.qr(A)
    Qn, Rn = np.linalg.qr(A)
    s, sn = np.sign(np.diag(R)), np.sign(np.diag(Rn))
    np.testing.assert_allclose(s[:, None] * R, sn[:, None] * Rn, atol=1e-12)
    np.testing.assert_allclose(Q * s[None, :], Qn * sn[None, :], atol=1e-12)


def test_qr_gram_identity_and_orthogonal_columns():
    """R^T·R = A^T·A (the Gram matrix); and a matrix whose columns are orthogonal
    with norms d_j has |R| = diag(d)."""
    rng = np.random.default_rng(7)
    A = rng.standard_normal((150, 12))
    R, _ = oracle.qr(A, want_q=False)
    np.testing.assert_allclose(R.T @ R, A.T @ A, rtol=1e-12, atol=1e-10)
    Qo, _ = np.linalg.qr(rng.standard_normal((150, 12)))
    d = np.arange(1, 13, dtype=np.float64)
    R2, _ = oracle.qr(Qo * d[None, :], want_q=False)
    np.testing.assert_allclose(np.abs(R2), np.diag(d), atol=1e-12)


# --------------------------------------------------------------------------- post-hoc compression
def _factor_modules(n, r, d_in, d_out, seed, decay=0.8):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((n, r, d_in)) / np.sqrt(d_in)
    B = rng.standard_normal((n, r, d_out)) * (decay ** np.arange(r))[None, :, None]
    return A, B


def test_compress_spectra_equal_the_singular_values_of_the_dense_product():
    # the QR-core route against numpy's SVD of the explicit d_in x d_out product
    A, B = _factor_modules(3, 6, 50, 40, seed=1)
    s, U, V, QA, QB = oracle.compress_spectra(A, B)
    for b in range(3):
        dense = A[b].T @ B[b]
        ref = np.linalg.svd(dense, compute_uv=False)[:6]
        assert np.allclose(s[b], ref, rtol=1e-10, atol=1e-12)
        # the core's factors rebuild the product
        assert np.allclose(QA[b] @ U[b] @ np.diag(s[b]) @ V[b].T @ QB[b].T, dense, atol=1e-12)


def test_compress_export_full_rank_and_eckart_young():
    A, B = _factor_modules(2, 8, 64, 48, seed=2)
    s, U, V, QA, QB = oracle.compress_spectra(A, B)
    for k in (8, 5, 1):
        An, Bn = oracle.export(s, U, V, QA, QB, np.array([k, k]))
        for b in range(2):
            dense = A[b].T @ B[b]
            approx = An[b].T @ Bn[b]
            err2 = np.linalg.norm(dense - approx) ** 2
            assert np.isclose(err2, float((s[b, k:] ** 2).sum()), rtol=1e-9, atol=1e-20)
            # the factors are balanced: A'^T A' = B' B'^T = diag(sigma_k)
            assert np.allclose(An[b] @ An[b].T, np.diag(s[b, :k]), atol=1e-12)
            assert np.allclose(Bn[b] @ Bn[b].T, np.diag(s[b, :k]), atol=1e-12)


def test_allocate_uniform_by_hand():
    sig = np.ones((3, 16), dtype=np.float32)
    k, off = oracle.allocate(sig, [16, 8, 5], [100, 100, 100], "U", 0.25, 1)
    assert k.tolist() == [4, 2, 2] and off.tolist() == [0, 4, 6, 8]   # ceil(4), ceil(2), ceil(1.25)
    k, _ = oracle.allocate(sig, [16, 8, 5], [100, 100, 100], "U", 0.25, 3)
    assert k.tolist() == [4, 3, 3]
    k, _ = oracle.allocate(sig, [16, 8, 5], [100, 100, 100], "U", 1.0, 1)
    assert k.tolist() == [16, 8, 5]


def _score(sig, b, i, cost):
    e = np.float32(0)
    for j in range(sig.shape[1]):
        e = np.float32(e + np.float32(sig[b, j] * sig[b, j]))
    return float(np.float32(np.float32(np.float32(sig[b, i] * sig[b, i]) / e) / np.float32(cost)))


def test_allocate_spectral_is_the_best_energy_per_budget_by_brute_force():
    # equal costs and no ties: the kept set must be the allocation of the
    # largest total score among all allocations within the budget
    import itertools
    rng = np.random.default_rng(5)
    for trial in range(25):
        n = 3
        ranks = rng.integers(2, 6, size=n)
        sig = np.zeros((n, 5), dtype=np.float32)
        for b in range(n):
            sig[b, :ranks[b]] = np.sort(rng.uniform(0.05, 3.0, size=ranks[b]).astype(np.float32))[::-1]
        costs = np.full(n, 10)
        keep = float(rng.uniform(0.2, 0.9))
        k, _ = oracle.allocate(sig, ranks, costs, "S", keep, 1)
        budget = math.floor(keep * float(int((ranks * costs).sum())))
        best, best_k = -1.0, None
        for ks in itertools.product(*[range(1, int(r) + 1) for r in ranks]):
            if sum(ks) * 10 > max(budget, n * 10):
                continue
            tot = sum(_score(sig, b, i, 10) for b in range(n) for i in range(1, ks[b]))
            if tot > best + 1e-12:
                best, best_k = tot, ks
        got = sum(_score(sig, b, i, 10) for b in range(n) for i in range(1, k[b]))
        assert np.isclose(got, best, rtol=0, atol=1e-9), (trial, k.tolist(), best_k)


def test_allocate_spectral_invariants():
    rng = np.random.default_rng(6)
    n, r = 40, 16
    ranks = rng.integers(4, r + 1, size=n)
    costs = rng.integers(200, 900, size=n)
    sig = np.zeros((n, r), dtype=np.float32)
    for b in range(n):
        sig[b, :ranks[b]] = np.sort(rng.exponential(1.0, size=ranks[b]).astype(np.float32))[::-1]
    prev = None
    for keep in (1 / 12, 0.2, 0.5, 0.9):
        k, off = oracle.allocate(sig, ranks, costs, "S", keep, 1)
        budget = math.floor(keep * float(int((ranks * costs).sum())))
        assert (k >= np.minimum(ranks, 1)).all() and (k <= ranks).all()
        assert int((k * costs).sum()) <= max(budget, int((np.minimum(ranks, 1) * costs).sum()))
        assert off[0] == 0 and (np.diff(off) == k).all()
        if prev is not None:
            assert (k >= prev).all()  # a larger budget never removes a rank
        prev = k
    # concentrated energy keeps fewer ranks than a flat spectrum at the same budget
    s2 = np.zeros((2, 8), dtype=np.float32)
    s2[0] = [10, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1]
    s2[1] = [1, 1, 1, 1, 1, 1, 1, 1]
    k, _ = oracle.allocate(s2, [8, 8], [100, 100], "S", 0.5, 1)
    assert k[0] < k[1]
