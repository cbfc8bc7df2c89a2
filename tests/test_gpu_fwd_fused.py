"""GPU parity of the fused forward (lora_linear_fwd_fused: row gather, shrink
and fused GEMM in one cooperative launch) against the fp64 oracle, at the
forward's tolerance, and against the two-kernel forward."""

from __future__ import annotations

import dataclasses

import numpy as np
import pytest

import oracle
from lora_adapter_execution_b200 import workloads as wl

from helpers import check_close, dev_bf16, host_f64
from test_gpu_fwd import SMALL_CASES, tile_rows

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


def run(inp, fused=True, keep_bits=False):
    import lora_adapter_execution_b200 as lora
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W, A, B = (dev_bf16(v) for v in (inp.X, inp.W, inp.A_pool, inp.B_pool))
    scale = torch.from_numpy(inp.scale).cuda()
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    U = torch.full((inp.T, plan.r_max), float("nan"), dtype=torch.float32, device="cuda")
    bits = None
    if keep_bits:
        bits = torch.empty(inp.T, -(-inp.d_in // 32), dtype=torch.int32, device="cuda")
        lora.dropout_keep_bits(inp.mask_seed, inp.p_drop, bits, inp.d_in)
    f = lora.linear_fwd_fused if fused else lora.linear_fwd
    f(plan, X, W, A, B, scale, Y, p_drop=inp.p_drop, seed=inp.mask_seed, U_save=U, keep_bits=bits)
    assert lora.device_status() == 0
    plan.destroy()
    return host_f64(Y), host_f64(U)


@pytest.mark.parametrize("case", [c for c in SMALL_CASES if c != "rank_256"])
def test_fused_small_vs_oracle(case):
    c = SMALL_CASES[case]
    inp = wl.make_inputs(c["name"], **c["kw"])
    Y, U = run(inp)
    Yr, Ur = oracle.forward(inp, want_u=True)
    check_close(Y, Yr, f"{case} Y")
    check_close(U, Ur[:, :U.shape[1]], f"{case} U")


@pytest.mark.parametrize("keep_bits", [False, True])
def test_fused_dropout_vs_oracle(keep_bits):
    inp = wl.make_inputs("fleet", T=520, d_in=256, d_out=264, n_adapters=60, p_drop=0.1)
    inp = dataclasses.replace(inp, mask_seed=1234)
    Y, U = run(inp, keep_bits=keep_bits)
    Yr, Ur = oracle.forward(inp, want_u=True)
    check_close(Y, Yr, "Y")
    check_close(U, Ur[:, :U.shape[1]], "U")


@pytest.mark.parametrize("name", ["decode", "fleet", "prefill"])
def test_fused_full_size_vs_oracle_and_two_kernel_forward(name):
    inp = wl.make_inputs(name)
    Y, U = run(inp)
    Y2, U2 = run(inp, fused=False)
    rows = np.arange(inp.T) if name == "decode" else tile_rows(inp)[0]
    Yr, Ur = oracle.forward(inp, rows=rows, want_u=True)
    check_close(Y[rows], Yr, f"{name} Y")
    check_close(U[rows], Ur[:, :U.shape[1]], f"{name} U")
    check_close(Y, Y2, f"{name} fused vs two kernels")


def test_fused_repeatable_bitwise():
    inp = wl.make_inputs("fleet", T=900, d_in=256, d_out=264, n_adapters=100)
    a = run(inp)
    b = run(inp)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()
