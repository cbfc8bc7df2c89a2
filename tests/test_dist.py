"""The multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

Weak scaling: every rank runs the same layer on a batch of its own, the step
time is the max over ranks of the device times, and the job's throughput counts
every rank's tokens. No GPU is needed for any of this."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from lora_adapter_execution_b200 import workloads as wl  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(1.5 + 2.0 * rank, world)
        inp = wl.make_rank_inputs("tiny", rank)
        q.put((rank, ms, int(inp.ids.sum()), float(np.asarray(inp.X, dtype=np.float64).sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_batches_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    # every rank sees the slowest rank's time
    assert [g[1] for g in got] == [3.5, 3.5]
    # the two ranks ran different batches
    assert got[0][2:] != got[1][2:]


def test_rank_inputs_share_the_layer():
    a = wl.make_rank_inputs("fleet", 0, T=300, d_in=64, d_out=64, n_adapters=40)
    b = wl.make_rank_inputs("fleet", 1, T=300, d_in=64, d_out=64, n_adapters=40)
    ref = wl.make_inputs("fleet", T=300, d_in=64, d_out=64, n_adapters=40)
    for f in ("ranks", "scale", "W", "A_pool", "B_pool", "offsets"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert np.array_equal(a.X, ref.X) and np.array_equal(a.ids, ref.ids)
    assert not np.array_equal(a.X, b.X)
    assert not np.array_equal(a.ids, b.ids)
    assert b.ids.min() >= 0 and b.ids.max() < len(b.ranks)
    assert a.mask_seed == b.mask_seed  # one global seed; each rank derives the seed of its rows


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(256, 10, 1, 2.0) == pytest.approx(256 * 10 / 2e-3)
    assert bench.job_throughput(256, 10, 4, 2.0) == pytest.approx(4 * 256 * 10 / 2e-3)
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def _rank_leaves(rank, world, port, q):
    """Rank 1 leaves between steps (after one agreed step, before the next
    all-reduce); rank 0 must learn of it through an error from its next
    collective within the short process-group timeout, not wait for good."""
    import datetime
    import time
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    first = bench.max_over_ranks(1.0 + rank, world)
    if rank == 1:
        q.put((rank, first, "left"))
        q.close()
        q.join_thread()  # the message is out before the process ends
        os._exit(0)  # leaves without joining the next step
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(1.0, world)
        outcome = "no error"
    except Exception as e:  # the backend's error type varies by version
        outcome = type(e).__name__
    q.put((rank, first, outcome, time.monotonic() - t0))
    q.close()
    q.join_thread()
    os._exit(0)


def test_rank_that_leaves_ends_the_next_collective_with_an_error():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_leaves, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=120) for _ in range(world)], key=lambda g: g[0])
    for p in procs:
        p.join(timeout=60)
    assert got[0][1] == got[1][1] == 2.0       # the step both ranks took agreed
    assert got[1][2] == "left"
    assert got[0][2] != "no error"             # rank 0's next collective failed ...
    assert got[0][3] < 60.0                    # ... within the timeout's bound, not forever


def test_rank_seed_gives_the_global_mask():
    """lora_dropout_seed_for_rows: rows t0.. of a rank's batch under the derived
    seed carry the mask the oracle assigns to global rows t0.. under the global
    seed (the oracle evaluates both sides; only the seed comes from the library)."""
    import lora_adapter_execution_b200 as lora
    import oracle
    T, d, p, seed = 40, 72, 0.3, 12345
    glob = oracle.mask(seed, p, 3 * T, d)
    for r in range(3):
        s_r = lora.dropout_seed_for_rows(seed, bench.rank_rows(r, T), d)
        assert np.array_equal(oracle.mask(s_r, p, T, d), glob[r * T:(r + 1) * T])
    assert lora.dropout_seed_for_rows(seed, 0, d) == seed


def _dp_rank(rank, world, port, q):
    """One data-parallel fine-tuning rank on CPU: the oracle's backward on this
    rank's shard (global rows rank*T..), then bench's gradient exchange."""
    import datetime
    import torch
    import torch.distributed as dist
    import lora_adapter_execution_b200 as lora
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        kw = dict(T=48, d_in=64, d_out=40, p_drop=0.25)
        inp = wl.make_rank_inputs("finetune", rank, **kw)
        s_r = lora.dropout_seed_for_rows(inp.mask_seed, bench.rank_rows(rank, inp.T), inp.d_in)
        import dataclasses
        dX, dA, dB = oracle.backward(dataclasses.replace(inp, mask_seed=s_r))
        grad = torch.from_numpy(np.concatenate([dA.ravel(), dB.ravel()]))
        bench.allreduce_grads(grad, world)
        q.put((rank, dX, grad.numpy().copy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_data_parallel_gradient_exchange_equals_the_union_batch_gloo():
    """Two gloo ranks, each with its shard of one global fine-tuning batch and the
    global dropout mask at its rows: after the all-reduce both hold the oracle's
    dA, dB of the whole batch, and each rank's dX rows are the batch's rows."""
    import dataclasses
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=180) for _ in range(world)], key=lambda g: g[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    kw = dict(T=48, d_in=64, d_out=40, p_drop=0.25)
    shards = [wl.make_rank_inputs("finetune", r, **kw) for r in range(world)]
    union = dataclasses.replace(shards[0], T=2 * shards[0].T, ids=np.concatenate([s.ids for s in shards]),
                                X=np.concatenate([s.X for s in shards]), dY=np.concatenate([s.dY for s in shards]))
    dX, dA, dB = oracle.backward(union)
    want = np.concatenate([dA.ravel(), dB.ravel()])
    for rank, rdX, grad in got:
        np.testing.assert_allclose(grad, want, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(rdX, dX[rank * 48:(rank + 1) * 48], rtol=1e-12, atol=1e-12)


def test_bench_gpus_2_starts_two_ranks_without_torchrun():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself (here the
    GPU-free dry run over gloo: one gradient exchange and one max over ranks)."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    import json
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["n_gpus"] == 2 and line["grad_sum"] == 3.0 and line["max_ms"] == 2.0
