"""The planner through the C ABI (host-only plans, no GPU) against the oracle's
stable grouping, bit for bit, plus the tile layout's invariants."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import lora_adapter_execution_b200 as lora
from lora_adapter_execution_b200 import workloads as wl


@pytest.mark.parametrize("name", wl.WORKLOADS)
def test_plan_bit_exact_vs_oracle(name):
    inp = wl.make_inputs(name, d_in=16, d_out=16)
    p = lora.Plan(inp.ids, inp.ranks, wl.SPECS[name].d_in, wl.SPECS[name].d_out, host_only=True)
    perm, seg = p.grouping()
    operm, oseg = oracle.plan(inp.ids, inp.n_adapters)
    assert (perm == operm).all()
    assert seg.shape == oseg.shape and (seg == oseg).all()
    info = p.info()
    used = np.unique(inp.ids)
    assert info["n_segments"] == used.size
    assert info["r_max"] == inp.ranks[used].max()
    assert info["sum_r_used"] == inp.ranks[used].sum()
    assert info["sum_r_tokens"] == inp.ranks[inp.ids].sum()
    assert info["n_tiles"] == -(-inp.T // 128)


def test_plan_fuzz():
    rng = np.random.default_rng(1)
    for _ in range(60):
        n = int(rng.integers(1, 50))
        T = int(rng.integers(1, 700))
        ranks = rng.integers(1, 257, size=n).astype(np.int32)
        if rng.random() < 0.5:
            ids = rng.integers(0, n, size=T).astype(np.int32)
        else:  # long runs
            ids = np.repeat(rng.integers(0, n, size=-(-T // 37)), 37)[:T].astype(np.int32)
        p = lora.Plan(ids, ranks, 64, 64, host_only=True)
        perm, seg = p.grouping()
        operm, oseg = oracle.plan(ids, n)
        assert (perm == operm).all() and (seg == oseg).all()
        info = p.info()
        # augmented K: every tile adds, per adapter present, twice its rank
        # rounded up to 16 (bf16 hi and lo parts of s*U)
        kaug = 0
        images = 0
        gathered = False
        for m in range(info["n_tiles"]):
            pos = perm[m * 128:(m + 1) * 128]
            kt = sum(2 * (-(-int(ranks[a]) // 16) * 16) for a in np.unique(ids[pos]))
            kaug += kt
            images += -(-kt // 64) * 16384
            gathered |= not (np.diff(pos) == 1).all()
        assert info["aug_k_total"] == kaug
        # scratch: the s*U images, then (if some tile's tokens are not consecutive
        # originals) a sorted copy of X (T x d_in bf16), 256-byte aligned
        want = images if not gathered else -(-images // 256) * 256 + T * 64 * 2
        assert info["scratch_bytes"] == want


def test_workload_tile_statistics():
    fl = wl.make_inputs("fleet", d_in=16, d_out=16)
    info = lora.Plan(fl.ids, fl.ranks, 4096, 4096, host_only=True).info()
    assert info["n_segments"] == 506 and info["sum_r_used"] == 5764
    pre = wl.make_inputs("prefill", d_in=16, d_out=16)
    info = lora.Plan(pre.ids, pre.ranks, 4096, 11008, host_only=True).info()
    assert info["n_segments"] == 14
