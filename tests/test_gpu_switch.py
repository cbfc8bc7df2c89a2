"""GPU parity of the fused adapter switch (lora_switch_apply: every layer's
W += sum_j c_j·A_j·B_j in one pass, in place) against the fp64 oracle.

The GPU sums in fp32 (c·A as a hi and a lo bf16 part) and rounds the new weight
once to bf16; the oracle's value is exact. Bound per element: the rounding,
half a bf16 ulp (2^-9 relative), plus a fraction of an ulp for the fp32 sum and
the ~2^-17 relative error of the split weights, so |W_gpu - W_exact| <=
2^-8·|W_exact| + 1e-5·max|ΔW|; integer-valued inputs are bit-exact."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from lora_adapter_execution_b200 import workloads as wl

from helpers import check_close, dev_bf16, host_bits

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


def stack(L, d_in, d_out, ranks, seed=0, ints=False):
    rng = np.random.default_rng(seed)
    R = int(np.sum(ranks))
    if ints:
        def draw(shape, s=1.0):
            return wl.f32_to_bf16_bits(rng.integers(-3, 4, size=shape).astype(np.float32))
    else:
        def draw(shape, s=1.0):
            return wl.f32_to_bf16_bits((rng.standard_normal(shape) * s).astype(np.float32))
    return (draw((L, d_in, d_out), 1 / np.sqrt(d_in)), draw((L, R, d_in), 1 / np.sqrt(d_in)),
            draw((L, R, d_out), 1.0))


def run_switch(ranks, W, A, B, terms, coefs, max_terms=None):
    import lora_adapter_execution_b200 as lora
    L, d_in, d_out = W.shape
    sw = lora.Switch(ranks, L, d_in, d_out, max_terms or len(terms))
    Wd = dev_bf16(W)
    sw.apply(Wd, dev_bf16(A), dev_bf16(B), terms, coefs)
    assert lora.device_status() == 0
    sw.destroy()
    return host_bits(Wd)


def check_switch(got_bits, W, exact, what):
    got = wl.bf16_bits_to_f32(got_bits).astype(np.float64)
    delta = exact - wl.bf16_bits_to_f32(W).astype(np.float64)
    bound = 2.0**-8 * np.abs(exact) + 1e-5 * np.abs(delta).max()
    bad = np.abs(got - exact) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off, first {np.argwhere(bad)[:3].tolist()}"
    check_close(got - wl.bf16_bits_to_f32(W), delta, f"{what} update", rel_fro=5e-3, elem=3e-2)


@pytest.mark.parametrize("L,d_in,d_out,ranks,terms,coefs", [
    (3, 264, 200, [3, 16, 7, 21, 5], [0, 2, 1, 3], [-1.2, -0.8, 1.4, 0.6]),
    (2, 512, 768, [16] * 8, [5, 6, 2, 7], [-1.0, -0.5, 0.75, 1.25]),
    (1, 8, 8, [1, 2], [1], [3.0]),
    (2, 136, 72, [64, 33], [1, 0], [-0.5, 2.0]),
])
def test_switch_vs_oracle(L, d_in, d_out, ranks, terms, coefs):
    W, A, B = stack(L, d_in, d_out, ranks, seed=L + d_in)
    got = run_switch(ranks, W, A, B, terms, coefs)
    check_switch(got, W, oracle.switch(W, A, B, ranks, terms, coefs), f"L={L} {d_in}x{d_out}")


def test_switch_integer_bit_exact():
    """Integer weights, factors and coefficients: every product and sum is exact
    in fp32, so the new weight is exactly the oracle's value rounded once."""
    ranks = [4, 8, 5, 16]
    W, A, B = stack(2, 192, 264, ranks, seed=3, ints=True)
    terms, coefs = [0, 3, 1, 2], [-2.0, -1.0, 1.0, 3.0]
    got = run_switch(ranks, W, A, B, terms, coefs)
    want = wl.f32_to_bf16_bits(oracle.switch(W, A, B, ranks, terms, coefs).astype(np.float32))
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


def test_switch_unmerge_after_merge_restores_the_weights():
    """Merging and then unmerging the same adapters (the two halves of a switch)
    returns each weight to within one bf16 rounding of each step."""
    import lora_adapter_execution_b200 as lora
    ranks = [16] * 8
    W, A, B = stack(2, 256, 256, ranks, seed=9)
    sw = lora.Switch(ranks, 2, 256, 256, 4)
    Wd, Ad, Bd = dev_bf16(W), dev_bf16(A), dev_bf16(B)
    sw.apply(Wd, Ad, Bd, [1, 4], [0.7, 0.3])
    sw.apply(Wd, Ad, Bd, [1, 4], [-0.7, -0.3])
    assert lora.device_status() == 0
    sw.destroy()
    w0 = wl.bf16_bits_to_f32(W).astype(np.float64)
    got = wl.bf16_bits_to_f32(host_bits(Wd)).astype(np.float64)
    merged = np.abs(oracle.switch(W, A, B, ranks, [1, 4], [0.7, 0.3]))
    assert (np.abs(got - w0) <= 2.0**-8 * (np.abs(w0) + merged) + 1e-6).all()


def test_switch_full_size_layers_vs_oracle():
    """The decode-time switch of a 32-layer stack of 4096 x 4096 weights with 8
    rank-16 adapters per layer: unmerge two, merge two. Two layers (the first and
    the last) are checked against the oracle element by element."""
    L, d, ranks = 32, 4096, [16] * 8
    rng = np.random.default_rng(0)
    W = wl.f32_to_bf16_bits((rng.standard_normal((L, d, d), dtype=np.float32) / 64))
    A = wl.f32_to_bf16_bits((rng.standard_normal((L, 128, d), dtype=np.float32) / 64))
    B = wl.f32_to_bf16_bits((rng.standard_normal((L, 128, d), dtype=np.float32) / 4))
    terms, coefs = [2, 5, 0, 7], [-1.2, -0.8, 1.3, 0.7]
    got = run_switch(ranks, W, A, B, terms, coefs)
    for l in (0, L - 1):
        exact = oracle.switch(W[l:l + 1], A[l:l + 1], B[l:l + 1], ranks, terms, coefs)
        check_switch(got[l:l + 1], W[l:l + 1], exact, f"layer {l}")


def test_switch_argument_errors():
    import lora_adapter_execution_b200 as lora
    ranks = [4, 8]
    sw = lora.Switch(ranks, 1, 64, 64, 2)
    W, A, B = (dev_bf16(x) for x in stack(1, 64, 64, ranks))
    with pytest.raises(lora.LoraError) as e:
        sw.apply(W, A, B, [0, 2], [1.0, 1.0])  # adapter 2 does not exist
    assert e.value.code == -2
    with pytest.raises(lora.LoraError) as e:
        sw.apply(W, A, B, [0, 1, 0], [1.0, 1.0, 1.0])  # more terms than max_terms
    assert e.value.code == -1
    sw.destroy()
    assert lora.device_status() == 0
