"""GPU parity of the batched tall-skinny QR (lora_tsqr) against the fp64
oracle's Householder QR, with both made unique by a non-negative diagonal of R
(the oracle's rows of R and columns of Q flipped where its diagonal is
negative).

Tolerances, from the fp32 arithmetic (unit roundoff u = 2^-24 = 6e-8): the
reconstruction ||Q·R - A|| / ||A|| and the loss of orthogonality
max|Q^T·Q - I| are backward errors of Householder QR, bounded by a small
multiple of (tile rows + tree depth·n)·u whatever the conditioning: 5e-5
leaves a factor of about 2 over 255·u + 6·64·u. R and Q themselves differ
from the exact factors by about the condition number times that, so the
elementwise comparison with the oracle uses 1e-4 (relative Frobenius) on
well-conditioned factors and 2e-3 on the decaying-spectrum case (condition
number about 50)."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from lora_adapter_execution_b200 import workloads as wl

from helpers import dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

BACKWARD = 5e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lora_adapter_execution_b200 as lora
    lora.load_library()
    yield
    assert lora.device_status() == 0


def as_matrices(bits):
    """[batch, n, m] bf16 bits -> fp64 [batch, m, n] (the matrices A_b)."""
    return wl.bf16_bits_to_f32(bits).astype(np.float64).transpose(0, 2, 1)


def oracle_unique(A):
    R, Q = oracle.qr(A)
    d = np.where(np.diagonal(R, axis1=1, axis2=2) < 0, -1.0, 1.0)
    return R * d[:, :, None], Q * d[:, None, :]


def run(F, want_q=True):
    import lora_adapter_execution_b200 as lora
    b, n, m = F.shape
    R = torch.full((b, n, n), float("nan"), dtype=torch.float32, device="cuda")
    Q = torch.full((b, n, m), float("nan"), dtype=torch.float32, device="cuda") if want_q else None
    lora.tsqr(F, R, Q)
    assert lora.device_status() == 0
    return R.double().cpu().numpy(), (Q.double().cpu().numpy().transpose(0, 2, 1) if want_q else None)


def rel_fro(got, ref):
    return np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)


def check_backward(A, R, Q, what):
    assert np.isfinite(R).all() and np.isfinite(Q).all(), what
    assert (np.diagonal(R, axis1=1, axis2=2) >= 0).all(), f"{what}: negative diagonal"
    assert np.allclose(np.tril(R, -1), 0.0), f"{what}: R not upper triangular"
    rec = max(rel_fro(Q[i] @ R[i], A[i]) for i in range(A.shape[0]))
    orth = max(np.abs(Q[i].T @ Q[i] - np.eye(Q.shape[2])).max() for i in range(A.shape[0]))
    assert rec <= BACKWARD, f"{what}: reconstruction {rec:.2e}"
    assert orth <= BACKWARD, f"{what}: orthogonality {orth:.2e}"
    return rec, orth


CASES = {
    # (batch, m, n, decay): one leaf and m == n; leaves 128 + 72; 8 leaves at
    # n = 1 (the warp build's narrowest columns); 6 leaves at n = 64 (the CTA
    # build); odd leaf counts (9 -> 5 -> 3 -> 2 -> 1 at m = 1111)
    "square_64": (2, 64, 64, 1.0),
    "one_leaf": (3, 200, 24, 1.0),
    "two_leaves": (3, 300, 16, 1.0),
    "seven_leaves_n1": (4, 1000, 1, 1.0),
    "five_leaves_n64": (2, 700, 64, 1.0),
    "ragged_n": (5, 1111, 37, 1.0),
    "many": (64, 520, 16, 1.0),
    # a last leaf of one row (m = 129) and one shorter than n on the CTA build
    "short_leaf": (3, 129, 16, 1.0),
    "short_leaf_cta": (2, 140, 33, 1.0),
    "n8": (5, 1000, 8, 1.0),
    "n32": (3, 2000, 32, 1.0),
}


@pytest.mark.parametrize("case", list(CASES))
def test_tsqr_vs_oracle(case):
    b, m, n, decay = CASES[case]
    bits = wl.factor_stack(b, m, n, seed=11, decay=decay)
    A = as_matrices(bits)
    R, Q = run(dev_bf16(bits))
    Rr, Qr = oracle_unique(A)
    assert rel_fro(R, Rr) <= 1e-4, f"R {rel_fro(R, Rr):.2e}"
    assert rel_fro(Q, Qr) <= 1e-4, f"Q {rel_fro(Q, Qr):.2e}"
    check_backward(A, R, Q, case)


def test_tsqr_decaying_spectrum():
    bits = wl.factor_stack(4, 900, 64, seed=5, decay=0.94)  # condition number about 50
    A = as_matrices(bits)
    R, Q = run(dev_bf16(bits))
    Rr, Qr = oracle_unique(A)
    assert rel_fro(R, Rr) <= 2e-3 and rel_fro(Q, Qr) <= 2e-3
    check_backward(A, R, Q, "decay")


def test_tsqr_r_only_matches():
    bits = wl.factor_stack(6, 777, 32, seed=2)
    F = dev_bf16(bits)
    R1, _ = run(F, want_q=False)
    R2, _ = run(F, want_q=True)
    assert np.array_equal(R1, R2)  # the same up pass either way


def test_tsqr_strided_pool_view():
    # one adapter's rows (rank 24 at row offset 8) of a stack of 4 layers' pools
    L, Rtot, d = 4, 40, 520
    pool_bits = wl.factor_stack(L, d, Rtot, seed=9)  # [L, 40, 520]
    pool = dev_bf16(pool_bits)
    F = pool[:, 8:32, :]
    assert not F.is_contiguous() and F.stride(2) == 1
    R, Q = run(F)
    A = as_matrices(pool_bits[:, 8:32, :])
    Rr, Qr = oracle_unique(A)
    assert rel_fro(R, Rr) <= 1e-4 and rel_fro(Q, Qr) <= 1e-4


def test_tsqr_rank_deficient():
    # a zero column and a repeated column: R's diagonal has zeros, Q stays
    # orthonormal and Q·R still reproduces A
    bits = wl.factor_stack(2, 400, 8, seed=4)
    bits[:, 3, :] = 0
    bits[:, 6, :] = bits[:, 1, :]
    A = as_matrices(bits)
    R, Q = run(dev_bf16(bits))
    assert np.all(np.abs(R[:, 3, 3]) <= 1e-6)
    check_backward(A, R, Q, "rank deficient")


def test_tsqr_full_size_properties_and_samples():
    # the bench's factor workload (4096 x 16 factors), properties on every
    # matrix, the oracle on a few
    b, m, n = 256, 4096, 16
    bits = wl.factor_stack(b, m, n, seed=1, decay=0.97)
    R, Q = run(dev_bf16(bits))
    A = as_matrices(bits)
    check_backward(A, R, Q, "full")
    pick = [0, 117, 255]
    Rr, Qr = oracle_unique(A[pick])
    assert rel_fro(R[pick], Rr) <= 1e-4 and rel_fro(Q[pick], Qr) <= 1e-4


def test_tsqr_rejects_bad_arguments():
    import lora_adapter_execution_b200 as lora
    F = dev_bf16(wl.factor_stack(1, 100, 65))
    with pytest.raises(lora.LoraError):
        lora.tsqr(F, torch.empty(1, 65, 65, device="cuda"))  # n > 64
    F = dev_bf16(wl.factor_stack(1, 10, 16))
    with pytest.raises(lora.LoraError):
        lora.tsqr(F, torch.empty(1, 16, 16, device="cuda"))  # m < n
