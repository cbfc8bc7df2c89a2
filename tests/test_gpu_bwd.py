"""GPU parity of the single-adapter backward (dU -> dX GEMM with the masked
adapter term -> token contractions for dA, dB) against the fp64 oracle."""

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


def run_fwd_bwd(inp, keep_bits=False, outputs=False, seed=None):
    """Forward (for U_save) then backward, all through the C ABI; with
    keep_bits the dropout mask is written once and read by both."""
    import lora_adapter_execution_b200 as lora
    r = int(inp.ranks[0])
    if seed is not None:
        inp = dataclasses.replace(inp, mask_seed=seed)
    bits = None
    if keep_bits:
        bits = torch.empty(inp.T, -(-inp.d_in // 32), dtype=torch.int32, device="cuda")
        lora.dropout_keep_bits(inp.mask_seed, inp.p_drop, bits, inp.d_in)
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W = dev_bf16(inp.X), dev_bf16(inp.W)
    A, B = dev_bf16(inp.A_pool), dev_bf16(inp.B_pool)
    dY = dev_bf16(inp.dY)
    scale = torch.from_numpy(inp.scale).cuda()
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    U = torch.empty(inp.T, r, dtype=torch.float32, device="cuda")
    lora.linear_fwd(plan, X, W, A, B, scale, Y, p_drop=inp.p_drop, seed=inp.mask_seed, U_save=U, keep_bits=bits)
    dX = torch.empty(inp.T, inp.d_in, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(r, inp.d_in, dtype=torch.float32, device="cuda")
    dB = torch.empty(r, inp.d_out, dtype=torch.float32, device="cuda")
    ws = torch.empty(lora.bwd_workspace_size(inp.T, inp.d_in, inp.d_out, r), dtype=torch.uint8, device="cuda")
    lora.linear_bwd(X, W, A, B, float(inp.scale[0]), U, dY, dX, dA, dB, ws, p_drop=inp.p_drop,
                    seed=inp.mask_seed, keep_bits=bits)
    assert lora.device_status() == 0
    plan.destroy()
    if outputs:
        return [t.cpu() for t in (Y, U, dX, dA, dB)]
    return host_f64(dX), host_f64(dA), host_f64(dB)


@pytest.mark.parametrize("kw", [
    dict(T=390, d_in=264, d_out=200, p_drop=0.1),
    dict(T=1000, d_in=520, d_out=264, p_drop=0.3),
    dict(T=700, d_in=256, d_out=256, p_drop=0.0),
])
def test_keep_bits_path_identical(kw):
    """Reading the mask from keep bits gives bit-identical Y, U, dX, dA, dB to
    re-deriving it from the generator in every kernel."""
    inp = wl.make_inputs("finetune", **kw)
    a = run_fwd_bwd(inp, keep_bits=False, outputs=True)
    b = run_fwd_bwd(inp, keep_bits=True, outputs=True)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int32) if x.dtype == torch.float32 else x.view(torch.int16),
                           y.view(torch.int32) if y.dtype == torch.float32 else y.view(torch.int16))


@pytest.mark.parametrize("kw", [
    dict(T=390, d_in=264, d_out=200, p_drop=0.0),
    dict(T=390, d_in=264, d_out=200, p_drop=0.1),
    dict(T=1000, d_in=520, d_out=264, p_drop=0.3),
])
def test_bwd_small_vs_oracle(kw):
    inp = wl.make_inputs("finetune", **kw)
    dX, dA, dB = run_fwd_bwd(inp)
    rdX, rdA, rdB = oracle.backward(inp)
    check_close(dX, rdX, "dX")
    check_close(dA, rdA, "dA")
    check_close(dB, rdB, "dB")


@pytest.mark.parametrize("r", [1, 5, 8, 21, 32, 64, 100, 256])
def test_bwd_ranks(r):
    inp = wl.make_inputs("finetune", T=300, d_in=256, d_out=136, p_drop=0.1)
    rng = np.random.default_rng(r)
    A = wl.f32_to_bf16_bits(rng.standard_normal((r, inp.d_in)).astype(np.float32) / 16)
    B = wl.f32_to_bf16_bits(rng.standard_normal((r, inp.d_out)).astype(np.float32) / np.sqrt(r))
    inp = dataclasses.replace(inp, ranks=np.array([r], dtype=np.int32), A_pool=A, B_pool=B,
                              offsets=np.array([0, r]))
    dX, dA, dB = run_fwd_bwd(inp)
    rdX, rdA, rdB = oracle.backward(inp)
    check_close(dX, rdX, f"dX r={r}")
    check_close(dA, rdA, f"dA r={r}")
    check_close(dB, rdB, f"dB r={r}")


def test_bwd_full_finetune_vs_oracle():
    inp = wl.make_inputs("finetune")
    dX, dA, dB = run_fwd_bwd(inp)
    rng = np.random.default_rng(0)
    # a random row of every 128-row tile, the tiles' first and last rows
    n_tiles = inp.T // 128
    rows = np.unique(np.concatenate([[128 * m + int(rng.integers(128)) for m in range(n_tiles)],
                                     [0, 127, 128, inp.T - 1], rng.choice(inp.T, 40, replace=False)]))
    rdX, rdA, rdB = oracle.backward(inp, rows=rows.astype(np.int64))
    check_close(dX[rows], rdX, "dX")
    check_close(dA, rdA, "dA")
    check_close(dB, rdB, "dB")


def test_bwd_deterministic():
    inp = wl.make_inputs("finetune", T=2100, d_in=256, d_out=264, p_drop=0.1)
    a = run_fwd_bwd(inp)
    b = run_fwd_bwd(inp)
    for x, y in zip(a, b):
        assert (x == y).all()


@pytest.mark.parametrize("r", [16, 5])
def test_bwd_integer_bit_exact(r):
    """Small-integer inputs with s = 1 and no dropout: every product and partial
    sum of the backward is an exact integer in fp32 (and |U|, |dU| <= 256 are
    exact in bf16), so dX is exactly the oracle's value rounded once to bf16 and
    dA, dB equal the oracle's exactly."""
    rng = np.random.default_rng(21 + r)
    T, d_in, d_out = 300, 64, 48
    inp = wl.integer_inputs(T, d_in, d_out, [r], np.zeros(T, dtype=np.int32), seed=r, lo=-2, hi=2)
    dX, dA, dB = run_fwd_bwd(inp)
    rdX, rdA, rdB = oracle.backward(inp)
    assert np.abs(rdA).max() < 2**24 and np.abs(rdB).max() < 2**24
    want = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rdX.astype(np.float32))).astype(np.float64)
    assert (dX == want).all(), np.argwhere(dX != want)[:5]
    assert (dA == rdA).all() and (dB == rdB).all()
    del rng


@pytest.mark.parametrize("T,d_in,d_out,r,p", [(1, 8, 8, 3, 0.0), (1, 8, 8, 16, 0.5), (1, 4096, 4096, 16, 0.1),
                                              (70, 8, 24, 21, 0.2)])
def test_bwd_degenerate_sizes_vs_oracle(T, d_in, d_out, r, p):
    """The boundary's smallest sizes: one token, widths of 8."""
    inp = wl.make_inputs("finetune", T=T, d_in=d_in, d_out=d_out, p_drop=p)
    rng = np.random.default_rng(T + r)
    A = wl.f32_to_bf16_bits(rng.standard_normal((r, d_in)).astype(np.float32) / np.sqrt(d_in))
    B = wl.f32_to_bf16_bits(rng.standard_normal((r, d_out)).astype(np.float32) / np.sqrt(r))
    inp = dataclasses.replace(inp, ranks=np.array([r], dtype=np.int32), A_pool=A, B_pool=B,
                              offsets=np.array([0, r]))
    dX, dA, dB = run_fwd_bwd(inp)
    rdX, rdA, rdB = oracle.backward(inp)
    check_close(dX, rdX, "dX")
    check_close(dA, rdA, "dA")
    check_close(dB, rdB, "dB")


def test_bwd_data_parallel_shards_sum_to_the_union_batch():
    """Two shards of one global batch, each run with the seed that gives its rows
    the global dropout mask (lora_dropout_seed_for_rows): their dA, dB summed (the
    data-parallel all-reduce) match the oracle's gradient of the whole batch, and
    their dX rows the batch's rows."""
    import lora_adapter_execution_b200 as lora
    kw = dict(T=640, d_in=256, d_out=264, p_drop=0.1)
    shards = [wl.make_rank_inputs("finetune", r, **kw) for r in range(2)]
    outs = []
    for r, sh in enumerate(shards):
        seed = lora.dropout_seed_for_rows(sh.mask_seed, r * sh.T, sh.d_in)
        outs.append(run_fwd_bwd(sh, keep_bits=(r == 1), seed=seed))
    union = dataclasses.replace(shards[0], T=2 * kw["T"], ids=np.concatenate([s.ids for s in shards]),
                                X=np.concatenate([s.X for s in shards]), dY=np.concatenate([s.dY for s in shards]))
    rdX, rdA, rdB = oracle.backward(union)
    check_close(outs[0][1] + outs[1][1], rdA, "dA sum")
    check_close(outs[0][2] + outs[1][2], rdB, "dB sum")
    check_close(np.concatenate([outs[0][0], outs[1][0]]), rdX, "dX rows")
