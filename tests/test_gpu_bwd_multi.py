"""GPU parity of the multi-adapter backward (lora_linear_bwd_multi) against the
fp64 oracle's backward, which is multi-adapter by definition.

Same tolerance as the forward (bf16 I/O, fp32 accumulation): rel-Frobenius
<= 5e-3, |err| <= 3e-2·max(1, |ref|) per element; integer-valued inputs
bit-exact. dA, dB are compared on the pool rows of adapters that own tokens
(the call writes no other rows)."""

from __future__ import annotations

import dataclasses

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


def run_multi(inp, keep_bits=False):
    """Forward (U_save) then the multi-adapter backward through the C ABI."""
    import lora_adapter_execution_b200 as lora
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W, A, B, dY = (dev_bf16(v) for v in (inp.X, inp.W, inp.A_pool, inp.B_pool, inp.dY))
    scale = torch.from_numpy(inp.scale).cuda()
    bits = None
    if keep_bits:
        bits = torch.empty(inp.T, -(-inp.d_in // 32), dtype=torch.int32, device="cuda")
        lora.dropout_keep_bits(inp.mask_seed, inp.p_drop, bits, inp.d_in)
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    U = torch.empty(inp.T, plan.r_max, dtype=torch.float32, device="cuda")
    lora.linear_fwd(plan, X, W, A, B, scale, Y, p_drop=inp.p_drop, seed=inp.mask_seed, U_save=U, keep_bits=bits)
    R = plan.pool_rows
    dX = torch.empty(inp.T, inp.d_in, dtype=torch.bfloat16, device="cuda")
    dA = torch.full((R, inp.d_in), float("nan"), dtype=torch.float32, device="cuda")
    dB = torch.full((R, inp.d_out), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(lora.bwd_multi_workspace_size(plan), dtype=torch.uint8, device="cuda")
    lora.linear_bwd_multi(plan, X, W, A, B, scale, U, dY, dX, dA, dB, ws, p_drop=inp.p_drop, seed=inp.mask_seed,
                          keep_bits=bits)
    assert lora.device_status() == 0
    plan.destroy()
    return host_f64(dX), host_f64(dA), host_f64(dB)


def used_rows(inp):
    rows = [np.arange(inp.offsets[a], inp.offsets[a + 1]) for a in np.unique(inp.ids)]
    return np.concatenate(rows)


def check_multi(inp, got, what, rows=None):
    dX, dA, dB = got
    rdX, rdA, rdB = oracle.backward(inp, rows=rows)
    u = used_rows(inp)
    check_close(dX if rows is None else dX[rows], rdX, f"{what} dX")
    check_close(dA[u], rdA[u], f"{what} dA")
    check_close(dB[u], rdB[u], f"{what} dB")


CASES = {
    # mixed adapters in every tile (sorted copies of X and dY), ranks 1..21
    "fleet_small": dict(name="fleet", kw=dict(T=700, d_in=320, d_out=296, n_adapters=90)),
    # requests of consecutive tokens (no gather): pieces cut where the original order jumps
    "prefill_small": dict(name="prefill", kw=dict(T=2100, d_in=256, d_out=392, n_adapters=12)),
    # one adapter: long segment, several pieces and their reduction
    "single": dict(name="finetune", kw=dict(T=2600, d_in=264, d_out=200)),
    "decode_small": dict(name="decode", kw=dict(T=300, d_in=328, d_out=264, n_adapters=40)),
    # ~200 short segments dealt into ~18 ranges: each CTA's range holds many pieces
    "fleet_ranges": dict(name="fleet", kw=dict(T=1500, d_in=2048, d_out=1024, n_adapters=300)),
}


@pytest.mark.parametrize("p", [0.0, 0.1])
@pytest.mark.parametrize("case", list(CASES))
def test_bwd_multi_vs_oracle(case, p):
    c = CASES[case]
    inp = wl.make_inputs(c["name"], with_dy=True, p_drop=p, **c["kw"])
    inp = dataclasses.replace(inp, mask_seed=17)
    check_multi(inp, run_multi(inp), f"{case} p={p}")


@pytest.mark.parametrize("case", ["fleet_small", "prefill_small"])
def test_bwd_multi_keep_bits_identical(case):
    """Reading the mask from keep bits (sorted copies of them when the plan
    gathers) gives bit for bit what re-deriving it from the generator gives."""
    c = CASES[case]
    kw = dict(c["kw"], d_in=384)
    inp = wl.make_inputs(c["name"], with_dy=True, p_drop=0.2, **kw)
    a = run_multi(inp, keep_bits=False)
    b = run_multi(inp, keep_bits=True)
    u = used_rows(inp)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1][u], b[1][u]) and np.array_equal(a[2][u], b[2][u])
    check_multi(inp, b, case)


def test_bwd_multi_ranks_up_to_256():
    inp = wl.make_inputs("tiny", T=400, d_in=192, d_out=136, n_adapters=3, with_dy=True, p_drop=0.1)
    ranks = np.array([256, 1, 130], dtype=np.int32)
    off = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int64)
    rng = np.random.default_rng(3)
    A = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], inp.d_in)).astype(np.float32) / 14)
    B = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], inp.d_out)).astype(np.float32) / 8)
    inp = dataclasses.replace(inp, ranks=ranks, A_pool=A, B_pool=B, offsets=off,
                              scale=np.array([0.25, 3.0, -0.5], dtype=np.float32))
    check_multi(inp, run_multi(inp), "ranks 256/1/130")


def test_bwd_multi_integer_bit_exact():
    """Small integers, s = 1, no dropout: every sum is an exact integer in fp32,
    so dX is the oracle's value rounded once and dA, dB equal it exactly."""
    rng = np.random.default_rng(8)
    T, d_in, d_out = 520, 64, 48
    ranks = [16, 5, 32, 1, 9]
    ids = rng.integers(0, len(ranks), size=T)
    inp = wl.integer_inputs(T, d_in, d_out, ranks, ids, seed=6, lo=-2, hi=2)
    dX, dA, dB = run_multi(inp)
    rdX, rdA, rdB = oracle.backward(inp)
    want = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rdX.astype(np.float32))).astype(np.float64)
    u = used_rows(inp)
    assert (dX == want).all(), np.argwhere(dX != want)[:5]
    assert (dA[u] == rdA[u]).all() and (dB[u] == rdB[u]).all()


def test_bwd_multi_single_adapter_matches_single_adapter_backward():
    """With one adapter the multi-adapter path and lora_linear_bwd compute the
    same gradients (within the parity tolerance of each other)."""
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs("finetune", T=3000, d_in=256, d_out=264, p_drop=0.1)
    dX, dA, dB = run_multi(inp)
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W, A, B, dY = (dev_bf16(v) for v in (inp.X, inp.W, inp.A_pool, inp.B_pool, inp.dY))
    U = torch.empty(inp.T, 16, dtype=torch.float32, device="cuda")
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    lora.linear_fwd(plan, X, W, A, B, torch.from_numpy(inp.scale).cuda(), Y, p_drop=inp.p_drop,
                    seed=inp.mask_seed, U_save=U)
    sdX = torch.empty(inp.T, inp.d_in, dtype=torch.bfloat16, device="cuda")
    sdA = torch.empty(16, inp.d_in, dtype=torch.float32, device="cuda")
    sdB = torch.empty(16, inp.d_out, dtype=torch.float32, device="cuda")
    ws = torch.empty(lora.bwd_workspace_size(inp.T, inp.d_in, inp.d_out, 16), dtype=torch.uint8, device="cuda")
    lora.linear_bwd(X, W, A, B, float(inp.scale[0]), U, dY, sdX, sdA, sdB, ws, p_drop=inp.p_drop, seed=inp.mask_seed)
    assert lora.device_status() == 0
    plan.destroy()
    check_close(dX, host_f64(sdX), "dX vs single-adapter")
    check_close(dA, host_f64(sdA), "dA vs single-adapter")
    check_close(dB, host_f64(sdB), "dB vs single-adapter")


def test_bwd_multi_full_size_fleet_vs_oracle():
    """The fleet batch (4096 tokens of 1000 rank-1..21 adapters, 4096 x 4096) as
    a fine-tuning step with dropout: dA, dB over every used adapter row, dX on
    rows of every 128-row tile."""
    inp = wl.make_inputs("fleet", with_dy=True, p_drop=0.1)
    got = run_multi(inp)
    perm, _ = oracle.plan(inp.ids, inp.n_adapters)
    rng = np.random.default_rng(1)
    rows = np.unique(perm[[128 * m + int(rng.integers(128)) for m in range(inp.T // 128)]]).astype(np.int64)
    check_multi(inp, got, "fleet", rows=rows)
