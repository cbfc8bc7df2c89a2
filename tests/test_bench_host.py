"""bench.py's host-side arithmetic, on CPU: the algorithmic bytes and flops that
the roofline divides by, recomputed from the inputs alone (numpy over the ids
and ranks, not the planner), and the planner's rank sums they use."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import lora_adapter_execution_b200 as lora  # noqa: E402
from lora_adapter_execution_b200 import workloads as wl  # noqa: E402


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("decode", {}), ("fleet", {"d_in": 256, "d_out": 264})])
def test_algorithmic_bytes_and_flops_from_first_principles(name, kw):
    inp = wl.make_inputs(name, **kw)  # fleet's ids and ranks at narrow widths
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out, host_only=True)
    info = plan.info()
    used = np.unique(inp.ids)
    r_used = int(inp.ranks[used].astype(np.int64).sum())
    r_tok = int(inp.ranks[inp.ids].astype(np.int64).sum())
    assert info["sum_r_used"] == r_used and info["sum_r_tokens"] == r_tok
    T, di, do = inp.T, inp.d_in, inp.d_out
    # the fused GEMM touches X, W, the used adapters' B rows, the s·U image's
    # source (counted with the shrink) and Y, each once, 2 bytes an element
    elems = T * di + di * do + sum(int(inp.ranks[a]) * do for a in used) + T * do
    # dense flops: the base product, then each token's rank-r expand
    flops = 2 * T * di * do + sum(2 * do * int(inp.ranks[a]) for a in inp.ids)
    gb, gf, lb, lf = bench.algorithmic(inp, info)
    assert gb == 2 * elems and gf == flops
    # the layer adds A's used rows and each token's rank-r shrink
    assert lb == 2 * (elems + sum(int(inp.ranks[a]) * di for a in used))
    assert lf == flops + sum(2 * di * int(inp.ranks[a]) for a in inp.ids)
    plan.destroy()


def test_decode_gemm_bytes_match_the_reported_figure():
    """The decode line's algorithmic bytes per launch: 2 B x (X 256x4096 + W
    4096x4096 + B rows of the used adapters x 4096 + Y 256x4096)."""
    inp = wl.make_inputs("decode")
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out, host_only=True)
    gb = bench.algorithmic(inp, plan.info())[0]
    r_used = int(inp.ranks[np.unique(inp.ids)].sum())
    assert gb == 2 * (256 * 4096 + 4096 * 4096 + r_used * 4096 + 256 * 4096)
    plan.destroy()


def test_reference_arm_prints_the_same_config_record():
    """Both arms describe the headline workload with one config record, computed
    from the inputs alone."""
    inp = wl.make_inputs("tiny")
    a = bench.config_record("tiny", inp, 1)
    b = bench.config_record("tiny", wl.make_inputs("tiny"), 1)
    assert a == b and a["workload"] == bench.WORKLOAD_TEXT["tiny"] and a["tokens_per_rank"] == 64


def test_backward_algorithmic_flops_match_the_fine_tuning_figure():
    """Fine-tuning: the base products of the forward and the dX GEMM (2 x 2·T·d²)
    plus the rank-16 terms come to about 1112 GFLOP per step."""
    inp = wl.make_inputs("finetune", with_dy=False, T=16384, d_in=64, d_out=64)
    T, d, r = 16384, 4096, 16
    inp.T, inp.d_in, inp.d_out = T, d, d
    _, fl = bench.algorithmic_bwd(inp, r)
    assert fl == 2 * T * d * d + 2 * T * r * 4 * d
    fwd = 2 * T * d * d + 2 * (d + d) * r * T
    assert abs((fl + fwd) / 1e9 - 1112.4) < 0.5


def test_default_runs_every_workload_with_the_fine_tuning_headline():
    a = bench.parse([])
    assert a.config == "all" and bench.HEADLINE == "finetune"
    assert set(bench.ORDER) | {"fleet_finetune"} == set(wl.WORKLOADS)
    assert bench.steps_for(bench.parse(["--steps", "20"]), "decode") == 20
