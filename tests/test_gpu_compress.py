"""GPU parity of post-hoc compression (lora_compress_spectra, _allocate, _export)
against the fp64 oracle.

Tolerances: the spectrum comes from fp32 Householder QRs (backward error a
small multiple of n·u ~ 1e-6 relative to the factors) and an fp32 one-sided
Jacobi SVD (orthogonality to 4e-7), so each sigma is within about 1e-5 of the
module's largest; the test allows 1e-4·sigma_max. The allocation is an integer
decision made in float32 on both sides from the same float32 spectrum: exact.
The exported factors are bf16 (relative rounding 2^-9 per element), so their
product is checked at the layer's own tolerance (relative Frobenius 5e-3)."""

from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from lora_adapter_execution_b200 import workloads as wl

from helpers import check_close, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lora_adapter_execution_b200 as lora
    lora.load_library()
    yield
    assert lora.device_status() == 0


def f64(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def spectra(A_bits, B_bits):
    import lora_adapter_execution_b200 as lora
    comp = lora.Compressor(dev_bf16(A_bits), dev_bf16(B_bits))
    assert lora.device_status() == 0
    return comp


@pytest.mark.parametrize("n,r,d_in,d_out", [(6, 16, 300, 264), (3, 8, 1000, 520), (2, 37, 260, 129),
                                            (4, 64, 640, 384), (3, 1, 200, 150)])
def test_spectra_vs_oracle(n, r, d_in, d_out):
    A, B = wl.module_factors(n, r, d_in, d_out, seed=r)
    comp = spectra(A, B)
    s = comp.sigma.double().cpu().numpy()
    ref, *_ = oracle.compress_spectra(f64(A), f64(B))
    assert (np.diff(s, axis=1) <= 0).all(), "not descending"
    err = np.abs(s - ref) / np.maximum(ref[:, :1], 1e-30)
    assert err.max() <= 1e-4, f"sigma off by {err.max():.2e} of sigma_max"


@pytest.mark.parametrize("policy,keep,floor", [("S", 1 / 12, 1), ("S", 0.3, 2), ("S", 0.0, 1), ("S", 1.0, 0),
                                               ("U", 0.25, 1), ("U", 1 / 12, 2), ("U", 1.0, 1)])
def test_allocate_matches_oracle_bit_exact(policy, keep, floor):
    import lora_adapter_execution_b200 as lora
    # a spectrum from the GPU itself, plus heterogeneous ranks and costs
    A, B = wl.module_factors(40, 16, 256, 192, seed=7)
    comp = spectra(A, B)
    rng = np.random.default_rng(3)
    ranks = rng.integers(1, 17, size=40).astype(np.int32)
    costs = rng.choice([448, 8192, 15104], size=40).astype(np.int64)
    sig = comp.sigma.cpu().numpy().copy()
    for b in range(40):
        sig[b, ranks[b]:] = 0.0
    k, off = lora.compress_allocate(torch.from_numpy(sig).cuda(), torch.from_numpy(ranks).cuda(),
                                    torch.from_numpy(costs).cuda(), policy, keep, floor)
    assert lora.device_status() == 0
    kr, offr = oracle.allocate(sig, ranks, costs, policy, keep, floor)
    assert np.array_equal(k.cpu().numpy(), kr), (k.cpu().numpy(), kr)
    assert np.array_equal(off.cpu().numpy(), offr)


def test_allocate_large_and_ties_bit_exact():
    # many modules, and exact ties (flat spectra): the order by module, then rank
    import lora_adapter_execution_b200 as lora
    rng = np.random.default_rng(9)
    n, r = 3000, 16
    sig = np.sort(rng.exponential(1.0, size=(n, r)).astype(np.float32), axis=1)[:, ::-1].copy()
    sig[::7] = 1.0  # flat modules
    ranks = np.full(n, r, dtype=np.int32)
    costs = np.full(n, 8192, dtype=np.int64)
    for keep in (1 / 12, 0.5):
        k, off = lora.compress_allocate(torch.from_numpy(sig).cuda(), torch.from_numpy(ranks).cuda(),
                                        torch.from_numpy(costs).cuda(), "S", keep, 1)
        kr, offr = oracle.allocate(sig, ranks, costs, "S", keep, 1)
        assert np.array_equal(k.cpu().numpy(), kr) and np.array_equal(off.cpu().numpy(), offr)


def export_group(comp, k, off, rows):
    A_new = torch.zeros(rows, comp.d_in, dtype=torch.bfloat16, device="cuda")
    B_new = torch.zeros(rows, comp.d_out, dtype=torch.bfloat16, device="cuda")
    comp.export(torch.from_numpy(k).cuda(), torch.from_numpy(off).cuda(), A_new, B_new)
    return host_f64(A_new), host_f64(B_new)


@pytest.mark.parametrize("policy,keep,r", [("S", 0.3, 16), ("U", 1.0, 16), ("S", 1 / 12, 16),
                                           # the way down's other builds: the warp build's widest
                                           # columns (r <= 32) and the CTA build (r > 32)
                                           ("S", 0.4, 24), ("U", 1.0, 40), ("S", 0.3, 64)])
def test_export_vs_oracle_truncation(policy, keep, r):
    import lora_adapter_execution_b200 as lora
    n, d_in, d_out = 5, 520, 264
    A, B = wl.module_factors(n, r, d_in, d_out, seed=11)
    comp = spectra(A, B)
    sig = comp.sigma.cpu().numpy()
    ranks = np.full(n, r, dtype=np.int32)
    costs = np.full(n, d_in + d_out, dtype=np.int64)
    k, off = oracle.allocate(sig, ranks, costs, policy, keep, 1)
    An, Bn = export_group(comp, k, off, int(off[-1]))
    assert lora.device_status() == 0
    s, U, V, QA, QB = oracle.compress_spectra(f64(A), f64(B))
    Ar, Br = oracle.export(s, U, V, QA, QB, k)
    for b in range(n):
        rows = slice(int(off[b]), int(off[b + 1]))
        got = An[rows].T @ Bn[rows]
        ref = Ar[b].T @ Br[b]
        check_close(got, ref, f"module {b} (k={k[b]})")
        if k[b] == r:  # nothing dropped: the original update
            check_close(got, f64(A[b]).T @ f64(B[b]), f"module {b} full rank")


def test_export_two_groups_into_shared_pools():
    import lora_adapter_execution_b200 as lora
    d_in, d_out = 384, 256
    A1, B1 = wl.module_factors(3, 8, d_in, d_out, seed=1)
    A2, B2 = wl.module_factors(4, 16, d_in, d_out, seed=2)
    c1, c2 = spectra(A1, B1), spectra(A2, B2)
    sig = np.zeros((7, 16), dtype=np.float32)
    sig[:3, :8] = c1.sigma.cpu().numpy()
    sig[3:] = c2.sigma.cpu().numpy()
    ranks = np.array([8] * 3 + [16] * 4, dtype=np.int32)
    costs = np.full(7, d_in + d_out, dtype=np.int64)
    k, off = lora.compress_allocate(torch.from_numpy(sig).cuda(), torch.from_numpy(ranks).cuda(),
                                    torch.from_numpy(costs).cuda(), "S", 0.35, 1)
    rows = int(off[-1].item())
    A_new = torch.zeros(rows, d_in, dtype=torch.bfloat16, device="cuda")
    B_new = torch.zeros(rows, d_out, dtype=torch.bfloat16, device="cuda")
    c1.export(k[:3], off[:3], A_new, B_new)
    c2.export(k[3:], off[3:7], A_new, B_new)
    assert lora.device_status() == 0
    kh, oh = k.cpu().numpy(), off.cpu().numpy()
    An, Bn = host_f64(A_new), host_f64(B_new)
    for grp, (A, B, b0) in enumerate(((A1, B1, 0), (A2, B2, 3))):
        s, U, V, QA, QB = oracle.compress_spectra(f64(A), f64(B))
        Ar, Br = oracle.export(s, U, V, QA, QB, kh[b0:b0 + A.shape[0]])
        for j in range(A.shape[0]):
            rows_b = slice(int(oh[b0 + j]), int(oh[b0 + j + 1]))
            check_close(An[rows_b].T @ Bn[rows_b], Ar[j].T @ Br[j], f"group {grp} module {j}")


def test_exported_pools_serve_the_forward():
    """The export's rank-exact pools are a serving fleet: the forward over them
    matches the oracle forward over the same pools."""
    import dataclasses
    import lora_adapter_execution_b200 as lora
    n, r, d_in, d_out = 12, 16, 256, 264
    A, B = wl.module_factors(n, r, d_in, d_out, seed=21)
    comp = spectra(A, B)
    ranks = np.full(n, r, dtype=np.int32)
    costs = np.full(n, d_in + d_out, dtype=np.int64)
    k, off = lora.compress_allocate(comp.sigma, torch.from_numpy(ranks).cuda(), torch.from_numpy(costs).cuda(),
                                    "S", 0.25, 1)
    rows = int(off[-1].item())
    A_new = torch.zeros(rows, d_in, dtype=torch.bfloat16, device="cuda")
    B_new = torch.zeros(rows, d_out, dtype=torch.bfloat16, device="cuda")
    comp.export(k, off[:n], A_new, B_new)
    inp = wl.make_inputs("tiny", T=400, d_in=d_in, d_out=d_out, n_adapters=n)
    kh = k.cpu().numpy().astype(np.int32)
    inp = dataclasses.replace(inp, ranks=kh, offsets=off.cpu().numpy(),
                              A_pool=A_new.view(torch.int16).cpu().numpy().view(np.uint16),
                              B_pool=B_new.view(torch.int16).cpu().numpy().view(np.uint16),
                              scale=np.full(n, 2.0, dtype=np.float32))
    plan = lora.Plan(inp.ids, inp.ranks, d_in, d_out)
    Y = torch.empty(inp.T, d_out, dtype=torch.bfloat16, device="cuda")
    lora.linear_fwd(plan, dev_bf16(inp.X), dev_bf16(inp.W), A_new, B_new, torch.from_numpy(inp.scale).cuda(), Y)
    assert lora.device_status() == 0
    plan.destroy()
    check_close(host_f64(Y), oracle.forward(inp), "Y over exported pools")
