"""GPU parity of the forward path (plan -> shrink -> fused tcgen05 GEMM) against
the fp64 CPU oracle, element by element, through the C ABI.

Tolerance (bf16 I/O, fp32 accumulation): rel-Frobenius <= 5e-3 and
|err| <= 3e-2 * max(1, |ref|) per element; bit-exact where the inputs make the
arithmetic exact; the plan and the dropout mask bit-exact."""

from __future__ import annotations

import dataclasses

import numpy as np
import pytest

import oracle
from lora_adapter_execution_b200 import workloads as wl

from helpers import check_close, dev_bf16, host_bits, host_f64

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


def run_fwd(inp, want_u=True, p=None, seed=None):
    import lora_adapter_execution_b200 as lora
    p = inp.p_drop if p is None else p
    seed = inp.mask_seed if seed is None else seed
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W = dev_bf16(inp.X), dev_bf16(inp.W)
    A, B = dev_bf16(inp.A_pool), dev_bf16(inp.B_pool)
    scale = torch.from_numpy(inp.scale).cuda()
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    rmax = plan.info()["r_max"]
    U = torch.full((inp.T, rmax), float("nan"), dtype=torch.float32, device="cuda") if want_u else None
    lora.linear_fwd(plan, X, W, A, B, scale, Y, p_drop=p, seed=seed, U_save=U)
    assert lora.device_status() == 0
    out = (host_f64(Y), host_f64(U) if want_u else None)
    plan.destroy()
    return out


SMALL_CASES = {
    # ragged everywhere: T not a multiple of 128, d_in not of 64, d_out not of 256
    "tiny": dict(name="tiny", kw={}),
    "decode_small": dict(name="decode", kw=dict(T=300, d_in=328, d_out=264, n_adapters=40)),
    "prefill_small": dict(name="prefill", kw=dict(T=1100, d_in=256, d_out=520, n_adapters=12)),
    "fleet_small": dict(name="fleet", kw=dict(T=700, d_in=320, d_out=296, n_adapters=200)),
    "finetune_small": dict(name="finetune", kw=dict(T=390, d_in=264, d_out=200, with_dy=False)),
    "rank_256": dict(name="tiny", kw=dict(T=200, d_in=192, d_out=136, n_adapters=3)),
}


@pytest.mark.parametrize("case", list(SMALL_CASES))
def test_fwd_small_vs_oracle(case):
    c = SMALL_CASES[case]
    inp = wl.make_inputs(c["name"], **c["kw"])
    if case == "rank_256":
        # extreme ranks: the maximum (256, four shrink pieces), 1, and a non-multiple of 16
        ranks = np.array([256, 1, 130], dtype=np.int32)
        off = np.concatenate([[0], np.cumsum(ranks)])
        rng = np.random.default_rng(3)
        A = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], inp.d_in)).astype(np.float32) / 14)
        B = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], inp.d_out)).astype(np.float32) / 8)
        inp = dataclasses.replace(inp, ranks=ranks, A_pool=A, B_pool=B, offsets=off,
                                  scale=np.array([0.25, 3.0, -0.5], dtype=np.float32))
    Y, U = run_fwd(inp)
    Yr, Ur = oracle.forward(inp, want_u=True)
    check_close(Y, Yr, f"{case} Y")
    check_close(U, Ur[:, :U.shape[1]], f"{case} U")


def test_fwd_dropout_small():
    inp = wl.make_inputs("fleet", T=520, d_in=256, d_out=264, n_adapters=60, p_drop=0.1)
    inp = dataclasses.replace(inp, mask_seed=1234)
    Y, U = run_fwd(inp)
    Yr, Ur = oracle.forward(inp, want_u=True)
    check_close(Y, Yr, "dropout Y")
    check_close(U, Ur[:, :U.shape[1]], "dropout U")


def test_fwd_integer_bit_exact():
    # |U| <= 64*4 = 256 (exact in bf16) and every fp32 partial sum is an exact
    # integer, so the GPU result is exactly the oracle's value rounded once.
    rng = np.random.default_rng(7)
    T, d_in, d_out = 260, 64, 272
    ranks = [16, 5, 32, 1]
    ids = rng.integers(0, 4, size=T)
    inp = wl.integer_inputs(T, d_in, d_out, ranks, ids, seed=5, lo=-2, hi=2)
    Y, U = run_fwd(inp)
    Yr, Ur = oracle.forward(inp, want_u=True)
    want = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(Yr.astype(np.float32))).astype(np.float64)
    assert np.abs(Yr).max() < 2**24
    assert (Y == want).all(), np.argwhere(Y != want)[:5]
    assert (U == Ur[:, :U.shape[1]]).all()


def test_fwd_B_zero_equals_base_gemm():
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs("decode", T=384, d_in=512, d_out=512, n_adapters=16)
    inp = dataclasses.replace(inp, B_pool=np.zeros_like(inp.B_pool))
    Y, _ = run_fwd(inp, want_u=False)
    Yb = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    lora.base_gemm(dev_bf16(inp.X), dev_bf16(inp.W), Yb)
    Yb = host_f64(Yb)
    # every tile's tokens are gathered in another order, but each output row is
    # the same dot products in the same K order: identical values
    assert (Y == Yb).all()
    check_close(Yb, oracle.forward(inp), "base")


def test_base_gemm_ragged_vs_oracle():
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs("decode", T=333, d_in=200, d_out=776, n_adapters=2)
    Yb = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    lora.base_gemm(dev_bf16(inp.X), dev_bf16(inp.W), Yb)
    z = dataclasses.replace(inp, B_pool=np.zeros_like(inp.B_pool))
    check_close(host_f64(Yb), oracle.forward(z), "base ragged")


def test_fwd_token_permutation_invariance():
    inp = wl.make_inputs("fleet", T=600, d_in=256, d_out=256, n_adapters=90)
    Y, _ = run_fwd(inp, want_u=False)
    pi = np.random.default_rng(2).permutation(inp.T)
    inp2 = dataclasses.replace(inp, X=inp.X[pi].copy(), ids=inp.ids[pi].copy())
    Y2, _ = run_fwd(inp2, want_u=False)
    check_close(Y2, Y[pi], "permuted")


def test_plan_on_device_matches_oracle():
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs("fleet", d_in=16, d_out=16)
    plan = lora.Plan(inp.ids, inp.ranks, 4096, 4096)
    perm, seg = plan.grouping()
    operm, oseg = oracle.plan(inp.ids, inp.n_adapters)
    assert (perm == operm).all() and (seg == oseg).all()


@pytest.mark.parametrize("p,seed", [(0.1, 0), (0.5, 77), (0.0, 3)])
def test_dropout_mask_bit_exact(p, seed):
    import lora_adapter_execution_b200 as lora
    T, d = 333, 264
    m = torch.empty(T, d, dtype=torch.uint8, device="cuda")
    lora.dropout_mask(seed, p, m)
    assert (m.cpu().numpy() == oracle.mask(seed, p, T, d)).all()


@pytest.mark.parametrize("p,seed,d", [(0.1, 0, 264), (0.5, 77, 200), (0.0, 3, 256), (0.3, 9, 37)])
def test_dropout_keep_bits_bit_exact(p, seed, d):
    """The keep bits (1 = kept) against the oracle's dropped mask, element by
    element; bits past d_in are 0."""
    import lora_adapter_execution_b200 as lora
    T = 301
    wpr = -(-d // 32)
    bits = torch.empty(T, wpr, dtype=torch.int32, device="cuda")
    lora.dropout_keep_bits(seed, p, bits, d)
    words = bits.cpu().numpy().view(np.uint32)
    unpacked = ((words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(T, wpr * 32)
    keep = 1 - oracle.mask(seed, p, T, d).astype(np.uint32)
    assert (unpacked[:, :d] == keep).all()
    assert (unpacked[:, d:] == 0).all()


def test_plan_rebuild_matches_fresh_plan():
    """A plan rebuilt for another batch (smaller: buffers reused; larger:
    reallocated) gives bit-identical Y to a freshly built plan, and its grouping
    equals the oracle's."""
    import lora_adapter_execution_b200 as lora
    first = wl.make_inputs("fleet", T=700, d_in=256, d_out=264, n_adapters=90, seed=1)
    plan = lora.Plan(first.ids, first.ranks, first.d_in, first.d_out)
    for T, seed in [(300, 2), (1500, 3)]:
        inp = wl.make_inputs("fleet", T=T, d_in=256, d_out=264, n_adapters=90, seed=seed)
        plan.rebuild(inp.ids, ranks=inp.ranks)
        perm, seg = plan.grouping()
        operm, oseg = oracle.plan(inp.ids, inp.n_adapters)
        assert (perm == operm).all() and (seg == oseg).all()
        X, W, A, B = dev_bf16(inp.X), dev_bf16(inp.W), dev_bf16(inp.A_pool), dev_bf16(inp.B_pool)
        scale = torch.from_numpy(inp.scale).cuda()
        Y1 = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
        Y2 = torch.empty_like(Y1)
        lora.linear_fwd(plan, X, W, A, B, scale, Y1)
        fresh = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
        lora.linear_fwd(fresh, X, W, A, B, scale, Y2)
        torch.cuda.synchronize()
        fresh.destroy()
        assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    plan.destroy()
    assert lora.device_status() == 0


def tile_rows(inp, seed=0):
    """Original rows that hit every 128-row tile of the plan's sorted order (one
    random row per tile, plus the tile's first and last row), and every row of
    the tile with the largest augmented K (the most adapters and ranks); the
    grouping comes from the oracle's plan."""
    perm, seg = oracle.plan(inp.ids, inp.n_adapters)
    T = inp.T
    n_tiles = -(-T // 128)
    kaug = np.zeros(n_tiles, dtype=np.int64)
    for a, start, length in seg:
        kc = -(-int(inp.ranks[a]) // 16) * 16
        for m in range(start // 128, (start + length - 1) // 128 + 1):
            kaug[m] += 2 * kc
    rng = np.random.default_rng(seed)
    pos = [int(rng.integers(128 * m, min(T, 128 * m + 128))) for m in range(n_tiles)]
    pos += [128 * m for m in range(n_tiles)] + [min(T, 128 * m + 128) - 1 for m in range(n_tiles)]
    heavy = int(np.argmax(kaug))
    pos += list(range(128 * heavy, min(T, 128 * heavy + 128)))
    return np.unique(perm[np.array(pos)]).astype(np.int64), heavy, int(kaug[heavy])


@pytest.mark.parametrize("name", ["decode", "prefill", "fleet", "finetune"])
def test_fwd_full_size_vs_oracle(name):
    inp = wl.make_inputs(name, with_dy=False)
    Y, U = run_fwd(inp)
    if name == "decode":
        rows = np.arange(inp.T)
    else:
        rows, heavy, kaug = tile_rows(inp)
        assert len(rows) >= -(-inp.T // 128)
    Yr, Ur = oracle.forward(inp, rows=rows, want_u=True)
    check_close(Y[rows], Yr, f"{name} Y")
    check_close(U[rows], Ur[:, :U.shape[1]], f"{name} U")


def test_fwd_full_size_matches_merged_weights():
    """The merged form of the S-LoRA article's batching section: Y[t] equals
    X[t]·(W + s_a·A_a·B_a) with the adapter merged into the weight (numpy fp64,
    a different formula from the oracle's), on the decode batch's tokens of ten
    adapters."""
    inp = wl.make_inputs("decode")
    Y, _ = run_fwd(inp, want_u=False)
    X = wl.bf16_bits_to_f32(inp.X).astype(np.float64)
    W = wl.bf16_bits_to_f32(inp.W).astype(np.float64)
    A = wl.bf16_bits_to_f32(inp.A_pool).astype(np.float64)
    B = wl.bf16_bits_to_f32(inp.B_pool).astype(np.float64)
    for a in np.unique(inp.ids)[:10]:
        o, r = int(inp.offsets[a]), int(inp.ranks[a])
        Wm = W + float(inp.scale[a]) * A[o:o + r].T @ B[o:o + r]
        rows = np.flatnonzero(inp.ids == a)
        check_close(Y[rows], X[rows] @ Wm, f"merged adapter {a}")


@pytest.mark.parametrize("T,d_in,d_out,ranks", [(1, 8, 8, [3]), (1, 4096, 4096, [16, 5]), (5, 8, 8, [1, 16, 2]),
                                                (130, 8, 16, [4, 21])])
def test_fwd_degenerate_sizes_vs_oracle(T, d_in, d_out, ranks):
    """The boundary's smallest sizes: one token, and widths of 8."""
    inp = wl.make_inputs("tiny", T=T, d_in=d_in, d_out=d_out, n_adapters=len(ranks))
    ranks = np.array(ranks, dtype=np.int32)
    off = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int64)
    rng = np.random.default_rng(11)
    A = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], d_in)).astype(np.float32) / np.sqrt(d_in))
    B = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], d_out)).astype(np.float32))
    ids = rng.integers(0, len(ranks), size=T).astype(np.int32)
    inp = dataclasses.replace(inp, ranks=ranks, ids=ids, A_pool=A, B_pool=B, offsets=off,
                              scale=(16.0 / ranks).astype(np.float32))
    Y, U = run_fwd(inp)
    Yr, Ur = oracle.forward(inp, want_u=True)
    check_close(Y, Yr, "Y")
    check_close(U, Ur[:, :U.shape[1]], "U")


def test_fwd_absent_adapter_factors_never_reach_a_token():
    """Rank 4 and 7 adapters read 16-row slices of B_pool whose remaining rows are
    the next adapters' rows; with Inf and NaN in those adapters (which have no
    token in the batch) every output stays finite and matches the oracle."""
    T, d_in, d_out = 300, 256, 264
    ranks = np.array([4, 16, 7, 21, 5], dtype=np.int32)
    off = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int64)
    rng = np.random.default_rng(4)
    ids = rng.choice([0, 2, 4], size=T).astype(np.int32)  # adapters 1 and 3 have no tokens
    inp = wl.make_inputs("tiny", T=T, d_in=d_in, d_out=d_out, n_adapters=5)
    A = wl.f32_to_bf16_bits(rng.standard_normal((off[-1], d_in)).astype(np.float32) / 16)
    Bf = rng.standard_normal((off[-1], d_out)).astype(np.float32) / 4
    Bf[off[1]:off[2]] = np.inf
    Bf[off[3]:off[4]] = np.nan
    inp = dataclasses.replace(inp, ranks=ranks, ids=ids, A_pool=A, B_pool=wl.f32_to_bf16_bits(Bf), offsets=off,
                              scale=np.full(5, 2.0, dtype=np.float32))
    Y, U = run_fwd(inp)
    assert np.isfinite(Y).all() and np.isfinite(U).all()
    clean = dataclasses.replace(inp, B_pool=wl.f32_to_bf16_bits(np.nan_to_num(Bf, nan=0.0, posinf=0.0)))
    check_close(Y, oracle.forward(clean), "Y next to non-finite absent adapters")


def test_fwd_repeatable_bitwise():
    inp = wl.make_inputs("fleet", T=900, d_in=256, d_out=264, n_adapters=100)
    Y1, U1 = run_fwd(inp)
    Y2, U2 = run_fwd(inp)
    assert (Y1 == Y2).all() and (U1 == U2).all()


def test_fwd_argument_errors():
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs("tiny")
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W = dev_bf16(inp.X), dev_bf16(inp.W)
    A, B = dev_bf16(inp.A_pool), dev_bf16(inp.B_pool)
    scale = torch.from_numpy(inp.scale).cuda()
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lora.LoraError):
        lora.linear_fwd(plan, X, W, A, B, scale, Y, p_drop=1.0)
    Xo = torch.empty(inp.T * inp.d_in + 1, dtype=torch.bfloat16, device="cuda")[1:].view(inp.T, inp.d_in)
    with pytest.raises(lora.LoraError):
        lora.linear_fwd(plan, Xo, W, A, B, scale, Y)
    host_plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out, host_only=True)
    with pytest.raises(lora.LoraError):
        lora.linear_fwd(host_plan, X, W, A, B, scale, Y)
    assert lora.device_status() == 0


@pytest.mark.parametrize("name,kw", [("decode", dict(T=300, d_in=328, d_out=264, n_adapters=40)),
                                     ("fleet", dict(T=700, d_in=320, d_out=296, n_adapters=200))])
def test_fwd_host_step_matches_device_forward(name, kw):
    """lora_linear_fwd_host (plan rebuilt from host ids, X copied in from pinned
    host memory, the forward, Y copied out) on two different batches through one
    plan: each step's host Y equals, bit for bit, lora_linear_fwd on device
    buffers with a plan built for that batch, and matches the oracle."""
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs(name, **kw)
    W, A, B = dev_bf16(inp.W), dev_bf16(inp.A_pool), dev_bf16(inp.B_pool)
    scale = torch.from_numpy(inp.scale).cuda()
    step_plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X_dev = torch.empty(inp.T, inp.d_in, dtype=torch.bfloat16, device="cuda")
    Y_dev = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    rng = np.random.default_rng(9)
    for it in range(2):
        ids = inp.ids if it == 0 else rng.integers(0, inp.n_adapters, size=inp.T).astype(np.int32)
        Xb = inp.X if it == 0 else wl.f32_to_bf16_bits(rng.standard_normal(inp.X.shape).astype(np.float32))
        X_host = torch.from_numpy(np.ascontiguousarray(Xb).view(np.int16)).view(torch.bfloat16).pin_memory()
        Y_host = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16).pin_memory()
        lora.linear_fwd_host(step_plan, ids, X_host, X_dev, W, A, B, scale, Y_dev, Y_host)
        torch.cuda.synchronize()
        assert lora.device_status() == 0
        ref_plan = lora.Plan(ids, inp.ranks, inp.d_in, inp.d_out)
        Y_ref = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
        lora.linear_fwd(ref_plan, dev_bf16(Xb), W, A, B, scale, Y_ref)
        torch.cuda.synchronize()
        ref_plan.destroy()
        assert torch.equal(Y_host.view(torch.int16), Y_ref.cpu().view(torch.int16)), f"{name} batch {it}"
        check_close(host_f64(Y_ref), oracle.forward(dataclasses.replace(inp, ids=ids, X=Xb)), f"{name} host step {it}")
    step_plan.destroy()
