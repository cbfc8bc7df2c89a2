"""Benchmark of the multi-adapter LoRA linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config all|NAME] [--impl lora|reference]

One step = one pass of the layer's whole hot path over one batch: the shrink
(U = (D ⊙ X)·A_a per token) and the fused tcgen05 GEMM (Y = X·W + s_a·U·B_a)
over a plan built once per batch and, for the fine-tuning workload, the
backward (dU -> dX GEMM -> dA, dB). Inputs are resident in HBM; steps rotate
over several input copies whose total exceeds the 126 MB L2, so no step reads
its operands from a warm L2. Steps are CUDA-graph replays timed with CUDA
events on the replay stream; a timed region is exactly K steps bracketed by a
barrier and a device synchronisation, repeated until the clock sampler has
seen it for a while, and the median region is reported (max over ranks).

With no --config every workload runs in one process and rank 0 prints ONE
JSON line: the fine-tuning workload (the largest single-GPU configuration,
forward + backward) is the headline (`value`, `roofline`, `e2e`,
`cpu_baseline`), and `configs` holds the same record for every workload.
`roofline` is the fused forward GEMM (the kernel the layer is built around),
timed alone in short bursts against the burst peak; `layer_roofline` is the
whole step, timed over long back-to-back regions, against the sustained peak.
`configs["switch"]` is the merge path (one fused adapter switch of a 32-layer
stack per step); `configs["factor_qr"]` the factor construction of post-hoc
compression (one batched tall-skinny QR of 2048 adapter factors per step);
`configs["compress"]` the whole LoRAForge-S export of 1024 modules per step.

`e2e` is the same metric through the public API with host buffers: per step
the plan is built from host ids, X (and dY) are copied from pinned host
memory, the layer runs, the result is copied back; consecutive steps overlap
(copy-in, compute and copy-out streams over two slots of buffers).

Multi-GPU: one process per GPU. Under torchrun each rank runs the layer on a
batch of its own (weak scaling). For the fine-tuning workload the ranks'
batches are shards of one global batch (data parallel): each step ends with
one NCCL all-reduce (sum) of the adapter gradients dA, dB, and each rank's
dropout mask is the global batch's mask at its rows. `--gpus N` without
torchrun re-executes this script under torchrun with N processes.

--impl reference times the CPU oracle (fp64 loops, all host cores) on a
bounded sample of the headline workload, with the same config record.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import socket
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lora_adapter_execution_b200 import workloads as wl  # noqa: E402

METRIC = "tokens/s per fused multi-LoRA linear at 1 B200; % of bf16 TC peak / HBM roofline"
L2_BYTES = 126 * 1024 * 1024
ORDER = ("tiny", "decode", "prefill", "fleet", "finetune")
HEADLINE = "finetune"
DEFAULT_STEPS = {"tiny": 2000, "decode": 3000, "prefill": 200, "fleet": 1000, "finetune": 100, "fleet_finetune": 200}
DEFAULT_WARMUP = 5
MIN_REGION_S = 0.3  # a timed region is repeated until this much device time has passed
CPU_BUDGET_S = {"headline": 12.0, "other": 5.0}
WORKLOAD_TEXT = {
    "tiny": "tiny: T=64, d_in=d_out=256, 4 adapters ranks {4,8,8,16}, s=16/r, ids uniform",
    "decode": "decode: T=256, d_in=d_out=4096, 64 adapters rank 16, s=2, ids uniform (unsorted)",
    "prefill": "prefill: T=8192, d_in=4096, d_out=11008, 200 adapters ranks {8,16,32,64}, Zipf(1.0) per 512-token request",
    "fleet": "fleet: T=4096, d_in=d_out=4096, 1000 adapters ranks 1..21, B rows x 1/k, Zipf(1.2) per token",
    "finetune": "finetune: T=16384, d_in=d_out=4096, 1 adapter rank 16, s=2, dropout 0.1; forward + backward",
    "fleet_finetune": ("fleet_finetune: the fleet batch (T=4096, 4096x4096, 1000 adapters ranks 1..21, Zipf(1.2) per "
                       "token) as one fine-tuning step of all its adapters, dropout 0.1; forward + multi-adapter "
                       "backward"),
}
# The fused GEMM, its launch and the plan tables that shape its work: a recorded
# ncu figure for the GEMM holds while the code of these files is unchanged.
KERNEL_SOURCES = ["lora_adapter_execution_b200/csrc/gemm.cuh", "lora_adapter_execution_b200/csrc/common.cuh",
                  "lora_adapter_execution_b200/csrc/internal.h", "lora_adapter_execution_b200/csrc/plan.cpp",
                  "lora_adapter_execution_b200/csrc/lora_b200.cu"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=DEFAULT_WARMUP)
    ap.add_argument("--config", default="all", choices=["all", *wl.WORKLOADS, "switch", "factor_qr", "compress"])
    ap.add_argument("--impl", default="lora", choices=["lora", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-layer", action="store_true",
                    help="time only the full step (no GEMM-alone, base or torch timings; for profiler runs)")
    ap.add_argument("--once", action="store_true",
                    help="one timed region per config, no repeats (for profiler runs)")
    ap.add_argument("--fwd", default="auto", choices=["auto", "fused", "two"],
                    help="the forward of the step: the faster of the two in a burst (auto), the one-launch fused "
                         "forward, or the two kernels")
    ap.add_argument("--dry-run", action="store_true",
                    help="no GPU: exercise the ranks' start-up and collectives over gloo and print a line")
    a = ap.parse_args(argv)
    a.warmup = max(3, a.warmup)
    return a


def steps_for(a, name):
    return a.steps if a.steps is not None else DEFAULT_STEPS[name]


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of the ranks' values (a device time): an all-reduce MAX over the
    process group, the value itself on one rank."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_grads(grad, world: int):
    """Data-parallel fine-tuning's one exchange: sum the ranks' adapter gradients
    (dA and dB, views of the one fp32 buffer `grad`) in place. Each rank's dA, dB
    is a sum over its own tokens, so the sum over ranks is the gradient of the
    global batch."""
    if world <= 1:
        return grad
    import torch.distributed as dist
    dist.all_reduce(grad, op=dist.ReduceOp.SUM)
    return grad


def rank_rows(rank: int, tokens_per_rank: int) -> int:
    """First global row of rank `rank`'s shard of the global batch."""
    return rank * tokens_per_rank


def job_throughput(tokens_per_rank: int, steps: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: every rank processed steps x tokens_per_rank tokens of
    its own batch (weak scaling) in ms, the max over ranks."""
    return world * tokens_per_rank * steps / (ms * 1e-3)


def n_copies_for(per_copy: int) -> int:
    return max(2, min(8, math.ceil(3 * L2_BYTES / per_copy)))


def copy_bytes(inp) -> int:
    T, di, do = inp.T, inp.d_in, inp.d_out
    per_copy = 2 * (T * di + di * do + T * do) + 2 * (di + do) * int(inp.offsets[-1])
    if inp.dY is not None:
        per_copy += 2 * (T * do + 2 * T * di)
    return per_copy


def config_record(name, inp, world):
    """The `config` object of a line: what the workload is and how it is run.
    Computed from the inputs alone, so both arms print the same record."""
    per_copy = copy_bytes(inp)
    n = n_copies_for(per_copy)
    ft = inp.dY is not None
    return {"workload": WORKLOAD_TEXT[name], "tokens_per_rank": inp.T,
            "l2": f"inputs rotate over {n} copies ({n * per_copy / 2**20:.0f} MiB > 126 MiB L2)",
            "parallelism": (f"dp{world} (shards of one global batch, all-reduce of dA, dB per step)" if ft
                            else f"dp{world} (independent batches, no collective)"),
            "plan": "built once per batch outside the timed region (reused by every layer)"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clocks and throttle reasons sampled during the timed region: NVML every
    2 ms (the device found by its UUID), else nvidia-smi every 100 ms. Reads only."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.nv = None
        self.samples = []  # (sm MHz, max sm MHz, reason bits)
        self.stop = threading.Event()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _poll(self):
        nv, h = self.nv
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), smax, get_reasons(h)))
            except Exception:
                break
            time.sleep(0.002)

    def __enter__(self):
        try:
            self.nv = self._nvml_handle()
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return self
        except Exception:
            self.nv = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.nv is not None:
            self.stop.set()
            self.t.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, smax, reasons, any_bits = [], None, set(), 0
        for mhz, mx, bits in self.samples:
            sm.append(float(mhz))
            smax = float(mx)
            any_bits |= int(bits)
            for n, b in self.REASONS.items():
                if bits & b:
                    reasons.add(n)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvml" if self.samples else ("nvidia-smi" if self.lines else None),
                "nvml_reason_bits": hex(any_bits) if self.samples else None}


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_src_sha():
    """Hash of the kernel sources' code: // comments, trailing blanks and empty
    lines are left out, so editing a comment keeps a recorded ncu figure valid."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        for line in open(os.path.join(ROOT, f), encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(config):
    """dram bytes per launch of the fused GEMM from a committed ncu capture, if the
    kernel source has not changed since (profiles/traffic.json)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(config)
    if not d or d.get("src_sha") != kernel_src_sha():
        return None
    return d.get("traffic_bytes_per_launch")


def algorithmic(inp, info):
    """Per-launch algorithmic bytes and flops of the fused GEMM, and of the whole
    layer (forward): bytes read or written at least once, flops of the dense math
    without block-diagonal padding."""
    T, di, do = inp.T, inp.d_in, inp.d_out
    R_used, R_tok = info["sum_r_used"], info["sum_r_tokens"]
    gemm_bytes = 2 * (T * di + di * do + do * R_used + T * do)
    gemm_flops = 2 * T * di * do + 2 * do * R_tok
    layer_bytes = 2 * (T * di + di * do + T * do + (di + do) * R_used)
    layer_flops = 2 * T * di * do + 2 * (di + do) * R_tok
    return gemm_bytes, gemm_flops, layer_bytes, layer_flops


def algorithmic_bwd_multi(inp, info):
    """The multi-adapter backward: reads X, W, dY, the used adapters' A, B rows
    and U, writes dX and the used gradient rows; flops of the dX GEMM and each
    token's rank-r terms (dU, its dX term, its dB and dA shares)."""
    T, di, do = inp.T, inp.d_in, inp.d_out
    R_used, R_tok = info["sum_r_used"], info["sum_r_tokens"]
    nbytes = (2 * (T * di + di * do + T * do + R_used * (di + do)) + 4 * T * info["r_max"] + 2 * T * di
              + 4 * R_used * (di + do))
    flops = 2 * T * do * di + 4 * (di + do) * R_tok
    return nbytes, flops


def algorithmic_bwd(inp, r):
    """Algorithmic bytes and flops of the single-adapter backward: reads X, W, dY,
    A, B, U, writes dX, dA, dB; flops of dU = s·dY·B^T, the dX GEMM with its adapter
    term, dB = s·U^T·dY and dA = (D⊙X)^T·dU."""
    T, di, do = inp.T, inp.d_in, inp.d_out
    nbytes = 2 * (T * di + di * do + T * do + r * (di + do)) + 4 * T * r + 2 * T * di + 4 * r * (di + do)
    flops = 2 * T * do * di + 2 * T * r * (do + di + do + di)
    return nbytes, flops


# ----------------------------------------------------------------------------- reference arm
def _oracle_runner(inp):
    """(run(n) -> seconds, what) for the oracle on n tokens of the workload: the
    forward of n evenly spaced tokens, or (fine-tuning) forward + backward of a
    sub-batch of the first n tokens."""
    import oracle
    if inp.dY is not None:
        def run(n):
            sub = wl.Inputs(spec=inp.spec, T=n, d_in=inp.d_in, d_out=inp.d_out, ranks=inp.ranks,
                            ids=inp.ids[:n].copy(), scale=inp.scale, X=inp.X[:n].copy(), W=inp.W,
                            A_pool=inp.A_pool, B_pool=inp.B_pool, dY=inp.dY[:n].copy(), p_drop=inp.p_drop,
                            mask_seed=inp.mask_seed, offsets=inp.offsets)
            t0 = time.perf_counter()
            oracle.forward(sub)
            oracle.backward(sub)
            return time.perf_counter() - t0
        return run, "forward+backward of the first {n} tokens (sub-batch of the same workload)"

    def run(n):
        rows = np.linspace(0, inp.T - 1, n).astype(np.int64)
        t0 = time.perf_counter()
        oracle.forward(inp, rows=rows)
        return time.perf_counter() - t0
    return run, "forward of {n} evenly spaced tokens of the batch"


def oracle_sample(inp, budget_s: float):
    """Time the oracle on a bounded sample of about budget_s seconds; returns
    (tokens, seconds, sample text)."""
    run, what = _oracle_runner(inp)
    n0 = 4
    dt = run(n0)
    n = int(max(1, min(inp.T, n0 * budget_s / max(dt, 1e-6))))
    dt = run(n)
    return n, dt, what.format(n=n)


def reference_name(a):
    return HEADLINE if a.config == "all" else a.config


def run_reference(a):
    rank, _, world = dist_env()
    if rank != 0:
        return
    import oracle
    name = reference_name(a)
    if name not in wl.WORKLOADS:
        # the merge path and the factor QR have oracle CPU baselines inside their
        # own entries (cpu_baseline); the reference arm times the layer workloads
        print(json.dumps({"impl": "reference", "unavailable": f"--impl reference times the layer workloads; "
                          f"{name}'s oracle baseline is its entry's cpu_baseline"}), flush=True)
        return
    inp = wl.make_inputs(name)
    oracle.build()
    cores = oracle.num_threads()
    # the whole run (warm-up + K steps) takes about 90 s of oracle time: each
    # step is a bounded sample sized once from a calibration run
    K = steps_for(a, name)
    run, what = _oracle_runner(inp)
    per_step = 90.0 / max(1, K + a.warmup)
    n0 = 2
    dt0 = run(n0)
    n = int(max(1, min(inp.T, n0 * per_step / max(dt0, 1e-6))))
    for _ in range(a.warmup):
        run(n)
    tok = 0
    secs = 0.0
    for _ in range(K):
        secs += run(n)
        tok += n
    v = tok / secs
    sample = what.format(n=n)
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
           "steps": K, "warmup": a.warmup, "ms_per_step": 1e3 * secs / K,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_record(name, inp, world),
           "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- lora arm
class Ctx:
    """What the per-workload measurements share: the device, the process group,
    the replay stream and the arguments."""

    def __init__(self, a):
        import torch
        import torch.distributed as dist
        import lora_adapter_execution_b200 as lora
        self.a = a
        self.rank, self.local_rank, self.world = dist_env()
        torch.cuda.set_device(self.local_rank)
        self.dev = torch.device("cuda", self.local_rank)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=self.dev)
        lora.load_library()
        self.stream = torch.cuda.Stream(device=self.dev)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def timed(self, step, K, min_s=MIN_REGION_S):
        """Device ms of exactly K calls of step() (graph replays), each region
        bracketed by a barrier and a synchronisation; at least 3 regions, repeated
        until min_s seconds of device time have passed; returns the median region
        (max over ranks) and the number of regions."""
        import torch
        for i in range(self.a.warmup):
            step(i)
        torch.cuda.synchronize()
        regions = []
        total = 0.0
        while True:
            self.barrier()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(self.stream):
                e0.record(self.stream)
                for i in range(K):
                    step(i)
                e1.record(self.stream)
            torch.cuda.synchronize()
            self.barrier()
            ms = e0.elapsed_time(e1)
            regions.append(ms)
            total += ms * 1e-3
            # every rank takes the same decision (the max over ranks of the total)
            done = len(regions) >= 3 and max_over_ranks(total, self.world, self.dev) >= min_s
            if done or len(regions) >= 2000:
                break
        return max_over_ranks(float(np.median(regions)), self.world, self.dev), len(regions)


def measure(name, cx, cpu_budget):
    """Every figure of one workload: the step's throughput, the fused GEMM's and
    the layer's roofline fractions, e2e through the public API, the CPU baseline."""
    import torch
    import torch.distributed as dist
    import lora_adapter_execution_b200 as lora

    a, dev, world, rank = cx.a, cx.dev, cx.world, cx.rank
    inp = wl.make_rank_inputs(name, rank)
    T, di, do = inp.T, inp.d_in, inp.d_out
    finetune = inp.dY is not None
    multi = finetune and inp.n_adapters > 1  # every adapter of a mixed batch trained at once
    K = steps_for(a, name)
    # data parallel: this rank's rows are global rows rank*T.. of one batch, so
    # its dropout mask is the global mask there
    mask_seed = lora.dropout_seed_for_rows(inp.mask_seed, rank_rows(rank, T), di) if finetune else inp.mask_seed

    def d(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    per_copy = copy_bytes(inp)
    n_copies = n_copies_for(per_copy)
    plan = lora.Plan(inp.ids, inp.ranks, di, do)
    info = plan.info()
    r_max = info["r_max"]
    scale = torch.from_numpy(inp.scale).to(dev)
    r = int(inp.ranks[0])
    copies = []
    for c in range(n_copies):
        cp = dict(X=d(inp.X), W=d(inp.W), A=d(inp.A_pool), B=d(inp.B_pool),
                  Y=torch.empty(T, do, dtype=torch.bfloat16, device=dev),
                  U=torch.empty(T, r_max, dtype=torch.float32, device=dev) if finetune else None)
        if multi:
            R = plan.pool_rows
            grad = torch.empty(R * (di + do), dtype=torch.float32, device=dev)  # dA_pool | dB_pool
            cp.update(dY=d(inp.dY), dX=torch.empty(T, di, dtype=torch.bfloat16, device=dev), grad=grad,
                      dA=grad[: R * di].view(R, di), dB=grad[R * di:].view(R, do),
                      ws=torch.empty(lora.bwd_multi_workspace_size(plan), dtype=torch.uint8, device=dev),
                      bits=torch.empty(T, -(-di // 32), dtype=torch.int32, device=dev))
        elif finetune:
            grad = torch.empty(r * (di + do), dtype=torch.float32, device=dev)  # dA | dB, one all-reduce
            cp.update(dY=d(inp.dY), dX=torch.empty(T, di, dtype=torch.bfloat16, device=dev), grad=grad,
                      dA=grad[: r * di].view(r, di), dB=grad[r * di:].view(r, do),
                      ws=torch.empty(lora.bwd_workspace_size(T, di, do, r), dtype=torch.uint8, device=dev),
                      bits=torch.empty(T, -(-di // 32), dtype=torch.int32, device=dev))
        copies.append(cp)

    # One graph per copy; the plan (and its scratch) is shared, steps run in
    # order. Copy c holds step c's batch; with dropout each copy's keep bits are
    # written on a second stream during the previous step's forward GEMM (the
    # bits kernel needs no shared memory and fits beside the GEMM's CTAs), and
    # that stream is joined before the step ends.
    masked = finetune and inp.p_drop > 0
    side = torch.cuda.Stream(device=dev)
    ev_fork = torch.cuda.Event()
    ev_join = torch.cuda.Event()

    def step(c, fused=False):
        # the forward in two kernels (shrink, then the fused GEMM) or in one
        # launch (lora_linear_fwd_fused)
        cp, nxt = copies[c], (c + 1) % len(copies)
        bits = cp["bits"] if masked else None
        if not fused:
            lora.linear_shrink(plan, cp["X"], cp["A"], scale, p_drop=inp.p_drop, seed=mask_seed, U_save=cp["U"],
                               keep_bits=bits)
        cur = torch.cuda.current_stream()
        if masked:
            ev_fork.record(cur)
            side.wait_event(ev_fork)
            with torch.cuda.stream(side):
                lora.dropout_keep_bits(mask_seed, inp.p_drop, copies[nxt]["bits"], di)
            ev_join.record(side)
        if fused:
            lora.linear_fwd_fused(plan, cp["X"], cp["W"], cp["A"], cp["B"], scale, cp["Y"], p_drop=inp.p_drop,
                                  seed=mask_seed, U_save=cp["U"], keep_bits=bits)
        else:
            lora.fused_gemm(plan, cp["X"], cp["W"], cp["B"], cp["Y"])
        if multi:
            lora.linear_bwd_multi(plan, cp["X"], cp["W"], cp["A"], cp["B"], scale, cp["U"], cp["dY"], cp["dX"],
                                  cp["dA"], cp["dB"], cp["ws"], p_drop=inp.p_drop, seed=mask_seed, keep_bits=bits)
        elif finetune:
            lora.linear_bwd(cp["X"], cp["W"], cp["A"], cp["B"], float(inp.scale[0]), cp["U"], cp["dY"], cp["dX"],
                            cp["dA"], cp["dB"], cp["ws"], p_drop=inp.p_drop, seed=mask_seed, keep_bits=bits)
        if masked:
            cur.wait_event(ev_join)

    # launches of this library per step: [row gather] + shrink + fused GEMM; the
    # backward: dU shrink, [U padding copy], dX GEMM, 2 contractions per 64-rank
    # group, 2 reductions; the keep bits of the next copy
    n_groups = -(-r // 64)
    launches_per_step = 2 + int(info["gathers_x"])
    if multi:
        # [X, dY (, keep bits) sorted copies], U sorted, dU shrink, dX GEMM, 2
        # contractions, [2 partial reductions], the keep bits
        bits_gathered = info["gathers_x"] and masked and (-(-di // 32)) % 4 == 0
        launches_per_step += (2 * info["gathers_x"] + int(bits_gathered) + 4 + 2 * int(plan_partial_rows(plan) > 0)
                              + int(masked))
    elif finetune:
        launches_per_step += 2 + int(r % 16 != 0) + 2 * n_groups + 2 + int(masked)
    torch.cuda.synchronize()
    with torch.cuda.stream(cx.stream):
        if masked:  # every copy's keep bits exist before its first step
            for c in range(len(copies)):
                lora.dropout_keep_bits(mask_seed, inp.p_drop, copies[c]["bits"], di)
        step(0)  # the first call sets kernel attributes outside any capture
    torch.cuda.synchronize()
    fused_error = None
    try:
        with torch.cuda.stream(cx.stream):
            step(0, fused=True)
        torch.cuda.synchronize()
        assert lora.device_status() == 0
    except Exception as e:  # the device refused the cooperative launch: two kernels only
        fused_error = f"{type(e).__name__}: {e}"
    graphs, fgraphs, ggraphs, bgraphs = [], [], [], []
    for c, cp in enumerate(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cx.stream):
            step(c)
        graphs.append(g)
        if fused_error is None:
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1, stream=cx.stream):
                step(c, fused=True)
            fgraphs.append(g1)
        if not a.no_layer:
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=cx.stream):
                lora.fused_gemm(plan, cp["X"], cp["W"], cp["B"], cp["Y"])
            ggraphs.append(g2)
            g3 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g3, stream=cx.stream):
                lora.base_gemm(cp["X"], cp["W"], cp["Y"])
            bgraphs.append(g3)
    torch.cuda.synchronize()
    assert lora.device_status() == 0

    def replay(gs, exchange=False):
        def f(i):
            gs[i % len(gs)].replay()
            if exchange:  # the data-parallel gradient exchange, on the replay stream
                allreduce_grads(copies[i % len(gs)]["grad"], world)
        return f

    ms_torch = ms_gemm = ms_base = ms_step_burst = ms_fused_burst = None
    if not a.no_layer:
        # the kernels alone, first, on a GPU that has idled: three regions of K
        # launches each (a burst, as the burst peak was taken)
        def burst(gs):
            time.sleep(0.2)
            return cx.timed(replay(gs), K, 0.0)[0]
        ms_step_burst = burst(graphs) if not (finetune and not multi and world > 1) else None
        ms_fused_burst = burst(fgraphs) if fgraphs and not (finetune and not multi and world > 1) else None
        ms_gemm = burst(ggraphs)
        ms_base = burst(bgraphs)
        assert lora.device_status() == 0
        # torch.matmul base for the overhead reference (cuBLAS, same shape and rotation)
        with torch.cuda.stream(cx.stream):
            torch.matmul(copies[0]["X"], copies[0]["W"], out=copies[0]["Y"])  # cuBLAS handle outside capture
        torch.cuda.synchronize()
        tgraphs = []
        for cp in copies:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cx.stream):
                torch.matmul(cp["X"], cp["W"], out=cp["Y"])
            tgraphs.append(g)
        ms_torch = burst(tgraphs)
        del ggraphs, bgraphs, tgraphs

    # the step's forward: whichever path ran faster in the burst (the same
    # choice on every rank: the max over ranks of each path's time)
    use_fused = (ms_fused_burst is not None and ms_step_burst is not None and ms_fused_burst < ms_step_burst)
    if a.fwd != "auto":
        use_fused = a.fwd == "fused" and bool(fgraphs)
    if use_fused:
        graphs, launches_per_step = fgraphs, launches_per_step - 1 - int(info["gathers_x"])
    with ClockSampler(cx.local_rank) as clk:
        ms_total, n_regions = cx.timed(replay(graphs, finetune and not multi and world > 1), K,
                                   0.0 if a.once else MIN_REGION_S)
    clocks = clk.summary()
    value = job_throughput(T, K, world, ms_total)
    entry = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
             "warmup": a.warmup, "ms_per_step": ms_total / K, "higher_is_better": True, "scaling": "weak",
             "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
             "config": config_record(name, inp, world),
             "timing": (f"CUDA-graph replays, CUDA events on the replay stream; median of {n_regions} regions of "
                        f"exactly {K} steps, max over ranks"),
             "gpu_launches": launches_per_step * K,
             "forward": ("one fused launch (lora_linear_fwd_fused)" if use_fused
                         else "two kernels (lora_linear_shrink, lora_fused_gemm)"
                         + (f"; fused launch unavailable: {fused_error}" if fused_error else "")),
             "clocks": clocks}

    hbm, tc_burst, tc_sust, src = peaks()
    gb, gf, lb, lf = algorithmic(inp, info)
    t_step = ms_total * 1e-3 / K
    if multi:
        bb, bfl = algorithmic_bwd_multi(inp, info)
        lb, lf = lb + bb, lf + bfl
    elif finetune:
        bb, bfl = algorithmic_bwd(inp, r)
        lb, lf = lb + bb, lf + bfl
    if name in ("decode", "tiny"):
        ach = lb / t_step / 1e9
        entry["layer_roofline"] = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                                   "peak_kind": f"{src} hbm_gbs (copy)", "algorithmic_per_step": lb,
                                   "what": "the whole step (all launches) against the layer's algorithmic bytes"}
    else:
        # the step is timed over long back-to-back regions (the clock record shows
        # the power cap), so its peak is the sustained one
        ach = lf / t_step / 1e12
        peak = tc_sust or tc_burst
        entry["layer_roofline"] = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                                   "frac": ach / peak, "frac_of_burst": ach / tc_burst,
                                   "peak_kind": f"{src} bf16_tflops_sustained (the step runs {MIN_REGION_S} s and more "
                                                f"back to back); burst {tc_burst}",
                                   "algorithmic_per_step": lf,
                                   "what": "the whole step (all launches) against the layer's algorithmic flops"}

    if ms_gemm is not None:
        t_gemm = ms_gemm * 1e-3 / K
        if name in ("decode", "tiny"):
            ach = gb / t_gemm / 1e9
            roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                    "peak_kind": f"{src} hbm_gbs (burst copy)"}
        else:
            ach = gf / t_gemm / 1e12
            roof = {"bound": "tensor", "achieved": ach, "peak": tc_burst, "unit": "TFLOP/s", "frac": ach / tc_burst,
                    "peak_kind": f"{src} bf16_tflops (burst)"}
        roof.update({"traffic": recorded_traffic(name), "kernel": "lora_gemm_kernel (fused base + adapter GEMM)",
                     "algorithmic_per_launch": gb if roof["bound"] == "hbm" else gf,
                     "avg_launch_us": t_gemm * 1e6, "timed": f"alone, 3 regions of {K} launches (burst)",
                     "layer_frac": entry["layer_roofline"]["frac"]})
        entry["roofline"] = roof
        base_fwd = min(ms_base, ms_torch) * 1e-3 / K
        t_sb = min(x for x in (ms_step_burst, ms_fused_burst) if x) * 1e-3 / K if ms_step_burst else None
        entry["layer"] = {"fused_gemm_us": t_gemm * 1e6, "base_gemm_us": ms_base * 1e3 / K,
                          "torch_matmul_us": ms_torch * 1e3 / K, "step_us": t_step * 1e6,
                          "step_burst_us": t_sb * 1e6 if t_sb else None,
                          "step_burst_us_fused": ms_fused_burst * 1e3 / K if ms_fused_burst else None,
                          "overhead_vs_base": None if (finetune or not t_sb) else t_sb / base_fwd - 1.0,
                          "gemm_overhead_vs_own_base": ms_gemm / ms_base - 1.0,
                          "layer_alg_bytes": lb, "layer_alg_flops": lf,
                          "segments": info["n_segments"], "aug_k_total": info["aug_k_total"]}

    # ---- end to end through the public API with host buffers
    if not a.no_e2e:
        entry["e2e"] = measure_e2e(cx, inp, copies, scale, mask_seed, K)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N=1 only)
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        import oracle
        oracle.build()
        n, dt, sample = oracle_sample(inp, cpu_budget)
        entry["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
                                 "kind": "oracle", "sample": sample}

    for cp in copies:
        cp.clear()
    del graphs
    plan.destroy()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def plan_partial_rows(plan):
    """Whether the multi-adapter backward has segments of several pieces (then it
    launches two more reductions): a segment longer than 1024 sorted tokens, or
    one whose original tokens are not consecutive in a plan without a sorted copy."""
    perm, seg = plan.grouping()
    gathers = plan.info()["gathers_x"]
    for _, start, length in seg:
        if length > 1024:
            return 1
        if not gathers and length > 1 and np.any(np.diff(perm[start:start + length]) != 1):
            return 1
    return 0


def measure_e2e(cx, inp, copies, scale, mask_seed, K):
    """The metric through the public API with host buffers (see the module text)."""
    import torch
    import lora_adapter_execution_b200 as lora
    dev, world = cx.dev, cx.world
    T, di, do = inp.T, inp.d_in, inp.d_out
    finetune = inp.dY is not None
    pin_X = torch.from_numpy(inp.X.view(np.int16)).view(torch.bfloat16).pin_memory()
    h2d = pin_X.numel() * 2 + inp.ids.nbytes
    d2h = T * do * 2
    if finetune:
        pin_dY = torch.from_numpy(inp.dY.view(np.int16)).view(torch.bfloat16).pin_memory()
        h2d += pin_dY.numel() * 2
        d2h += T * di * 2
    Ke = max(3, min(K, 200 if not finetune else 20))

    fallback_note = ""
    if not finetune:
        # the forward workloads: one C-ABI call per step with host buffers; it
        # must first reproduce the device-buffer forward bit for bit on every
        # rank, else (or on any error) the steps below run as the
        # Python-orchestrated loop
        r = e2e_host_step_loop(cx, inp, copies, scale, mask_seed, Ke, h2d, d2h)
        if r is not None:
            return r
        fallback_note = "; the host-step call failed or did not reproduce the device forward, so this loop ran"

    # Steps run as a pipeline over two slots (device buffers, plan, pinned
    # results): step i copies its inputs in on one stream, computes on a second
    # and copies its results out on a third, so the copies of one step overlap
    # the compute of its neighbours. Each step still builds its plan from the
    # host ids and moves all of its own inputs and results.
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    slots = copies[:2]
    plans = [lora.Plan(inp.ids, inp.ranks, di, do, stream=s_in) for _ in range(2)]
    pin_Ys = [torch.empty(T, do, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pin_dXs = [torch.empty(T, di, dtype=torch.bfloat16).pin_memory() for _ in range(2)] if finetune else None
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "comp", "out")}

    def e2e_step(i):
        s = i % 2
        c, p = slots[s], plans[s]
        if i >= 2:
            s_in.wait_event(ev["comp"][s])  # step i - 2 is done with this slot's inputs and plan
        p.rebuild(inp.ids, stream=s_in)  # the batch's plan from its host ids (buffers reused)
        with torch.cuda.stream(s_in):
            c["X"].copy_(pin_X, non_blocking=True)
            if finetune:
                c["dY"].copy_(pin_dY, non_blocking=True)
            ev["in"][s].record(s_in)
        s_comp.wait_event(ev["in"][s])
        if i >= 2:
            s_comp.wait_event(ev["out"][s])  # step i - 2's results have left this slot
        with torch.cuda.stream(s_comp):
            bits = None
            if finetune and inp.p_drop > 0:
                bits = c["bits"]
                lora.dropout_keep_bits(mask_seed, inp.p_drop, bits, di, stream=s_comp)
            lora.linear_fwd(p, c["X"], c["W"], c["A"], c["B"], scale, c["Y"], p_drop=inp.p_drop,
                            seed=mask_seed, U_save=c["U"], keep_bits=bits)
            if finetune and inp.n_adapters > 1:
                lora.linear_bwd_multi(p, c["X"], c["W"], c["A"], c["B"], scale, c["U"], c["dY"], c["dX"],
                                      c["dA"], c["dB"], c["ws"], p_drop=inp.p_drop, seed=mask_seed, keep_bits=bits)
            elif finetune:
                lora.linear_bwd(c["X"], c["W"], c["A"], c["B"], float(inp.scale[0]), c["U"], c["dY"],
                                c["dX"], c["dA"], c["dB"], c["ws"], p_drop=inp.p_drop, seed=mask_seed,
                                keep_bits=bits)
                allreduce_grads(c["grad"], world)
            ev["comp"][s].record(s_comp)
        s_out.wait_event(ev["comp"][s])
        with torch.cuda.stream(s_out):
            pin_Ys[s].copy_(c["Y"], non_blocking=True)
            if finetune:
                pin_dXs[s].copy_(c["dX"], non_blocking=True)
            ev["out"][s].record(s_out)

    def drain():
        for st in (s_in, s_comp, s_out):
            st.synchronize()

    for i in range(2):
        e2e_step(i)
    drain()
    cx.barrier()
    t0 = time.perf_counter()
    for i in range(Ke):
        e2e_step(2 + i)
    drain()
    dt = time.perf_counter() - t0
    for p in plans:
        p.destroy()
    dt = max_over_ranks(dt, world, dev)
    return {"value": job_throughput(T, Ke, world, dt * 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": Ke,
            "what": "per step: plan from host ids + H2D of X (pinned)" + (" and dY" if finetune else "")
                    + " + forward" + (" + backward + gradient all-reduce" if finetune else "")
                    + " + D2H of the result; steps pipelined over two slots (copy-in, compute and"
                    " copy-out streams); host wall clock over the steps" + fallback_note}


def e2e_host_step_loop(cx, inp, copies, scale, mask_seed, Ke, h2d, d2h):
    """The forward workloads' e2e through lora_linear_fwd_host: each step is one
    call with host buffers (the plan rebuilt from the host ids, X copied in from
    pinned host memory, the forward, Y copied out to pinned host memory), steps
    alternating over two streams with a plan and a buffer set each, so one
    step's copies overlap the other's kernels. The ranks first agree that the
    call's first result equals the device-buffer forward bit for bit on every
    rank (an all-reduce, taken by every rank whatever happened before it);
    otherwise it returns None and nothing is timed."""
    import torch
    import lora_adapter_execution_b200 as lora
    dev, world = cx.dev, cx.world
    T, di, do = inp.T, inp.d_in, inp.d_out
    streams, plans, pin_Ys = [], [], []
    slots = copies[:2]

    def step(i):
        s = i % 2
        c = slots[s]
        lora.linear_fwd_host(plans[s], inp.ids, pin_X, c["X"], c["W"], c["A"], c["B"], scale, c["Y"], pin_Ys[s],
                             p_drop=inp.p_drop, seed=mask_seed, U_save=c["U"], stream=streams[s])

    def drain():
        for st in streams:
            st.synchronize()

    ok = False
    try:
        pin_X = torch.from_numpy(inp.X.view(np.int16)).view(torch.bfloat16).pin_memory()
        streams = [torch.cuda.Stream(device=dev) for _ in range(2)]
        plans = [lora.Plan(inp.ids, inp.ranks, di, do, stream=st) for st in streams]
        pin_Ys = [torch.empty(T, do, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        for i in range(2):
            step(i)
        drain()
        # the first step's host result against the device-buffer forward of the same batch
        ref_plan = lora.Plan(inp.ids, inp.ranks, di, do)
        Y_ref = torch.empty(T, do, dtype=torch.bfloat16, device=dev)
        lora.linear_fwd(ref_plan, slots[0]["X"], slots[0]["W"], slots[0]["A"], slots[0]["B"], scale, Y_ref,
                        p_drop=inp.p_drop, seed=mask_seed)
        torch.cuda.synchronize(dev)
        ref_plan.destroy()
        ok = torch.equal(pin_Ys[0].view(torch.int16), Y_ref.cpu().view(torch.int16)) and lora.device_status() == 0
    except Exception:  # noqa: BLE001
        ok = False
    if max_over_ranks(0.0 if ok else 1.0, world, dev) > 0:
        drain()
        for p in plans:
            p.destroy()
        return None
    try:
        cx.barrier()
        t0 = time.perf_counter()
        for i in range(Ke):
            step(2 + i)
        drain()
        dt = time.perf_counter() - t0
    finally:
        drain()
        for p in plans:
            p.destroy()
    dt = max_over_ranks(dt, world, dev)
    return {"value": job_throughput(T, Ke, world, dt * 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": Ke,
            "what": "per step: one lora_linear_fwd_host call (plan from host ids, H2D of X from pinned host "
                    "memory, forward, D2H of Y into pinned host memory) on one of two streams, each with its "
                    "own plan and buffers; checked bit for bit against the device-buffer forward first; host "
                    "wall clock over the steps"}


SWITCH = dict(L=32, d=4096, n_adapters=8, rank=16, prev=(2, 5), cur=(0, 7), gates=((0.6, 0.4), (0.7, 0.3)),
              scale=2.0)
SWITCH_TEXT = ("adapter switch: 32 layers of 4096x4096 bf16 weights, 8 rank-16 adapters per layer (s=2); "
               "unmerge the previous token's top-2 and merge the current top-2 in one pass (4 terms)")


def switch_inputs(seed=0):
    """The switch workload: weights W ~ N(0, 1/d) and factor pools drawn like the
    layer's (A ~ N(0, 1/d), B ~ N(0, 1/r)), per layer, as bf16 bits."""
    c = SWITCH
    rng = np.random.default_rng(seed)
    L, d, R = c["L"], c["d"], c["n_adapters"] * c["rank"]
    W = wl.f32_to_bf16_bits(rng.standard_normal((L, d, d), dtype=np.float32) * np.float32(d ** -0.5))
    A = wl.f32_to_bf16_bits(rng.standard_normal((L, R, d), dtype=np.float32) * np.float32(d ** -0.5))
    B = wl.f32_to_bf16_bits(rng.standard_normal((L, R, d), dtype=np.float32) * np.float32(c["rank"] ** -0.5))
    terms = list(c["prev"]) + list(c["cur"])
    coefs = [-g * c["scale"] for g in c["gates"][0]] + [g * c["scale"] for g in c["gates"][1]]
    return W, A, B, terms, coefs


def measure_switch(cx, cpu_budget):
    """The merge path: one fused adapter switch of a whole layer stack per step,
    in place on the resident weights (HBM-bound: every weight is read and
    written once)."""
    import torch
    import lora_adapter_execution_b200 as lora
    a, dev = cx.a, cx.dev
    c = SWITCH
    K = a.steps if a.steps is not None else 50
    W, A, B, terms, coefs = switch_inputs()
    L, d, R = c["L"], c["d"], c["n_adapters"] * c["rank"]
    ranks = np.full(c["n_adapters"], c["rank"], dtype=np.int32)

    def dv(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)
    Wd, Ad, Bd = dv(W), dv(A), dv(B)
    sw = lora.Switch(ranks, L, d, d, len(terms))
    # the step alternates the switch and its inverse, so the weights stay near W
    neg = [-x for x in coefs]

    def step(i):
        sw.apply(Wd, Ad, Bd, terms, coefs if i % 2 == 0 else neg)
    with torch.cuda.stream(cx.stream):
        step(0)
        step(1)
    torch.cuda.synchronize()
    assert lora.device_status() == 0
    with ClockSampler(cx.local_rank) as clk:
        ms, n_regions = cx.timed(step, K, 0.0 if a.once else MIN_REGION_S)
    t = ms * 1e-3 / K
    hbm, _, _, src = peaks()
    nbytes = 2 * 2 * L * d * d + 2 * L * len(terms) * c["rank"] * 2 * d
    ach = nbytes / t / 1e9
    entry = {"metric": "fused adapter switches/s (every layer of the stack per switch)", "value": 1.0 / t,
             "unit": "switches/s", "n_gpus": cx.world, "steps": K, "warmup": a.warmup, "ms_per_step": t * 1e3,
             "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
             "config": {"workload": SWITCH_TEXT, "l2": f"weights {2 * L * d * d / 2**30:.1f} GiB > 126 MiB L2"},
             "timing": (f"eager calls of lora_switch_apply, CUDA events on the stream; median of {n_regions} regions "
                        f"of exactly {K} switches"),
             "gpu_launches": 2 * K, "clocks": clk.summary(),
             "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                          "peak_kind": f"{src} hbm_gbs (copy)", "traffic": None,
                          "kernel": "lora_switch_images_kernel + lora_gemm_kernel (merge mode), per switch",
                          "algorithmic_per_launch": nbytes, "avg_launch_us": t * 1e6,
                          "what": "bytes: every weight read and written once, the terms' factor rows read once"}}
    # e2e: the host holds the term list (adapters, gates); the step copies it in,
    # switches and reads one row of the last layer back
    pin = torch.empty(d, dtype=torch.bfloat16).pin_memory()
    torch.cuda.synchronize()
    cx.barrier()
    t0 = time.perf_counter()
    Ke = max(3, min(K, 50))
    for i in range(Ke):
        step(i)
        pin.copy_(Wd[L - 1, 0], non_blocking=True)
    torch.cuda.synchronize()
    dt = max_over_ranks(time.perf_counter() - t0, cx.world, dev)
    entry["e2e"] = {"value": Ke / dt, "unit": "switches/s", "h2d_bytes_per_step": 8 * len(terms),
                    "d2h_bytes_per_step": 2 * d, "steps": Ke,
                    "what": "per step: lora_switch_apply from host term arrays (staged and copied in) + D2H of one "
                            "weight row; host wall clock"}
    if cx.rank == 0 and cx.world == 1 and not a.no_cpu_baseline:
        import oracle
        oracle.build()
        run_layers = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < cpu_budget and run_layers < L:
            oracle.switch(W[run_layers:run_layers + 1], A[run_layers:run_layers + 1], B[run_layers:run_layers + 1],
                          ranks, terms, coefs)
            run_layers += 1
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": run_layers / L / dt, "unit": "switches/s", "cores": oracle.num_threads(),
                                 "kind": "oracle", "sample": f"{run_layers} of the {L} layers, scaled to one switch"}
    sw.destroy()
    del Wd, Ad, Bd
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


FACTOR = dict(batch=2048, m=4096, n=16, decay=0.97)
FACTOR_TEXT = ("factor QR: 2048 adapter factors of 4096 x 16 (1024 rank-16 modules, A and B^T of each; bf16 pool "
               "rows in, fp32 Q and R out)")


def measure_tsqr(cx, cpu_budget):
    """The factor construction of post-hoc compression: one batched tall-skinny
    QR (Q and R) of every factor per step; beside it torch.linalg.qr of the same
    matrices in fp32 (the matched library QR, context only)."""
    import torch
    import lora_adapter_execution_b200 as lora
    a, dev = cx.a, cx.dev
    c = FACTOR
    b, m, n = c["batch"], c["m"], c["n"]
    K = a.steps if a.steps is not None else 20
    bits = wl.factor_stack(b, m, n, seed=3, decay=c["decay"])
    F = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
    R = torch.empty(b, n, n, dtype=torch.float32, device=dev)
    Q = torch.empty(b, n, m, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, lora.tsqr_workspace_size(b, m, n, True)), dtype=torch.uint8, device=dev)
    levels = 1
    while (max(1, m // 128) if m >= 256 else 1) > (1 << (levels - 1)):
        levels += 1

    def step(i):
        lora.tsqr(F, R, Q, ws)
    with torch.cuda.stream(cx.stream):
        step(0)
    torch.cuda.synchronize()
    assert lora.device_status() == 0
    with ClockSampler(cx.local_rank) as clk:
        ms, n_regions = cx.timed(step, K, 0.0 if a.once else MIN_REGION_S)
    t = ms * 1e-3 / K
    hbm, _, _, src = peaks()
    nbytes = b * (m * n * 2 + m * n * 4 + n * n * 4)
    ach = nbytes / t / 1e9
    entry = {"metric": "adapter factors QR-factorised per second (Q and R)", "value": b / t, "unit": "factors/s",
             "n_gpus": cx.world, "steps": K, "warmup": a.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
             "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
             "config": {"workload": FACTOR_TEXT, "l2": f"factors {b * m * n * 2 / 2**20:.0f} MiB in, "
                                                       f"Q {b * m * n * 4 / 2**20:.0f} MiB out (> 126 MiB L2)"},
             "timing": (f"eager calls of lora_tsqr, CUDA events on the stream; median of {n_regions} regions of "
                        f"exactly {K} calls"),
             "gpu_launches": 2 * levels * K, "clocks": clk.summary(),
             "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                          "peak_kind": f"{src} hbm_gbs (copy)", "traffic": None,
                          "kernel": "lora_qr_factor_kernel + lora_qr_apply_kernel, all levels, per call",
                          "algorithmic_per_launch": nbytes, "avg_launch_us": t * 1e6,
                          "what": "bytes: the bf16 factors read once, Q and R (fp32) written once"}}
    # matched library QR: torch.linalg.qr of the same matrices (fp32, [b, m, n]);
    # not in profiler runs (--no-layer: it launches thousands of library kernels)
    A32 = F.float().transpose(1, 2).contiguous() if not a.no_layer else None
    try:
        if A32 is None:
            raise RuntimeError("skipped (--no-layer)")
        def lib_step(i):
            torch.linalg.qr(A32, mode="reduced")
        lms, _ = cx.timed(lib_step, max(3, K // 4), 0.0)
        entry["library_qr"] = {"what": "torch.linalg.qr(mode='reduced') of the same factors as fp32 [b, m, n]",
                               "ms_per_call": lms / max(3, K // 4), "factors_per_s": b / (lms * 1e-3 / max(3, K // 4))}
    except Exception as e:  # pragma: no cover - context only
        entry["library_qr"] = {"unavailable": str(e)[:200]}
    del A32
    # e2e: factors from pinned host memory, R back to the host
    if a.no_e2e:
        entry["e2e"] = None
        del F, R, Q, ws
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        return entry
    hF = torch.from_numpy(bits.view(np.int16)).pin_memory()
    hR = torch.empty(b, n, n, dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    cx.barrier()
    Ke = max(3, min(K, 10))
    t0 = time.perf_counter()
    for i in range(Ke):
        F.view(torch.int16).copy_(hF, non_blocking=True)
        step(i)
        hR.copy_(R, non_blocking=True)
    torch.cuda.synchronize()
    dt = max_over_ranks(time.perf_counter() - t0, cx.world, dev)
    entry["e2e"] = {"value": b * Ke / dt, "unit": "factors/s", "h2d_bytes_per_step": b * m * n * 2,
                    "d2h_bytes_per_step": b * n * n * 4, "steps": Ke,
                    "what": "per step: H2D of the bf16 factors (pinned) + lora_tsqr + D2H of R; host wall clock"}
    if cx.rank == 0 and cx.world == 1 and not a.no_cpu_baseline:
        import oracle
        oracle.build()
        cores = oracle.num_threads()
        cap = min(b, 64 * cores)
        A64 = wl.bf16_bits_to_f32(bits[:cap]).astype(np.float64).transpose(0, 2, 1)
        done = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < cpu_budget and done < cap:
            oracle.qr(A64[done:done + cores])  # one matrix per thread
            done += cores
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": done / dt, "unit": "factors/s", "cores": cores, "kind": "oracle",
                                 "sample": f"{done} of the {b} factors (Householder QR in fp64, Q and R)"}
    del F, R, Q, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


COMPRESS = dict(n=1024, r=16, d=4096, keep=1 / 12, floor=1)
COMPRESS_TEXT = ("post-hoc compression: 1024 rank-16 modules of 4096 x 4096 (32 layers x 4 projections x 8 "
                 "adapters), LoRAForge-S rank-floored 1/12 spectral export: spectra, allocation, truncated factors")


def measure_compress(cx, cpu_budget):
    """Post-hoc compression of a fleet's modules per step: the factor QRs and
    core SVDs (lora_compress_spectra), the spectral-budget allocation and the
    export of the truncated factors into new pools."""
    import torch
    import lora_adapter_execution_b200 as lora
    a, dev = cx.a, cx.dev
    c = COMPRESS
    n, r, d = c["n"], c["r"], c["d"]
    K = a.steps if a.steps is not None else 10
    A, B = wl.module_factors(n, r, d, d, seed=5)
    Ad = torch.from_numpy(A.view(np.int16)).to(dev).view(torch.bfloat16)
    Bd = torch.from_numpy(B.view(np.int16)).to(dev).view(torch.bfloat16)
    ranks = torch.full((n,), r, dtype=torch.int32, device=dev)
    costs = torch.full((n,), 2 * d, dtype=torch.int64, device=dev)
    A_new = torch.empty(n * r, d, dtype=torch.bfloat16, device=dev)
    B_new = torch.empty(n * r, d, dtype=torch.bfloat16, device=dev)
    state = {}

    def step(i):
        comp = lora.Compressor(Ad, Bd)
        k, off = lora.compress_allocate(comp.sigma, ranks, costs, "S", c["keep"], c["floor"])
        comp.export(k, off[:n], A_new, B_new)
        state["k"] = k
        state["comp"] = comp
    with torch.cuda.stream(cx.stream):
        step(0)
    torch.cuda.synchronize()
    assert lora.device_status() == 0
    kept = int(state["k"].sum().item())
    # tree levels of a 4096-row factor (leaves of 128): each factor goes up and
    # down them; + the core SVDs, the allocation and two root-block launches
    levels, nodes = 1, -(-d // 128)
    while nodes > 1:
        nodes, levels = -(-nodes // 2), levels + 1
    with ClockSampler(cx.local_rank) as clk:
        ms, n_regions = cx.timed(step, K, 0.0 if a.once else MIN_REGION_S)
    t = ms * 1e-3 / K
    hbm, _, _, src = peaks()
    nbytes = n * r * 2 * d * 2 + kept * 2 * d * 2
    ach = nbytes / t / 1e9
    entry = {"metric": "adapter modules compressed per second (spectra, allocation, export)", "value": n / t,
             "unit": "modules/s", "n_gpus": cx.world, "steps": K, "warmup": a.warmup, "ms_per_step": t * 1e3,
             "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
             "config": {"workload": COMPRESS_TEXT, "kept_ranks": kept, "of_ranks": n * r,
                        "l2": f"factors {n * r * 2 * d * 2 / 2**20:.0f} MiB in (> 126 MiB L2)"},
             "timing": (f"eager calls (workspace allocation included), CUDA events on the stream; median of "
                        f"{n_regions} regions of exactly {K} exports"),
             "gpu_launches": (4 * levels + 4) * K, "clocks": clk.summary(),
             "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                          "peak_kind": f"{src} hbm_gbs (copy)", "traffic": None,
                          "kernel": "all kernels of the export (tall-skinny QRs both ways, core SVDs, allocation)",
                          "algorithmic_per_launch": nbytes, "avg_launch_us": t * 1e6,
                          "what": "bytes: the modules' bf16 factors read once, the kept factors written once"}}
    if cx.rank == 0 and cx.world == 1 and not a.no_cpu_baseline:
        import oracle
        oracle.build()
        done = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < cpu_budget and done < n:
            Af = wl.bf16_bits_to_f32(A[done:done + 4]).astype(np.float64)
            Bf = wl.bf16_bits_to_f32(B[done:done + 4]).astype(np.float64)
            s_, U_, V_, QA_, QB_ = oracle.compress_spectra(Af, Bf)
            kk, _ = oracle.allocate(s_.astype(np.float32), np.full(len(Af), r), np.full(len(Af), 2 * d), "S",
                                    c["keep"], c["floor"])
            oracle.export(s_, U_, V_, QA_, QB_, kk)
            done += len(Af)
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": done / dt, "unit": "modules/s", "cores": oracle.num_threads(),
                                 "kind": "oracle", "sample": f"{done} of the {n} modules (allocation within each "
                                                             "batch of 4)"}
    del Ad, Bd, A_new, B_new, state
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


HEAD_KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config", "timing", "roofline", "layer_roofline", "gpu_launches",
             "clocks", "layer", "e2e", "cpu_baseline")


def run_lora(a):
    cx = Ctx(a)
    names = list(ORDER) if a.config == "all" else [a.config]
    entries = {}
    extra = {"switch": measure_switch, "factor_qr": measure_tsqr, "compress": measure_compress}
    for name in names:
        budget = CPU_BUDGET_S["headline" if name in (HEADLINE, a.config) else "other"]
        entries[name] = extra[name](cx, budget) if name in extra else measure(name, cx, budget)
    if a.config == "all":
        entries["fleet_finetune"] = measure("fleet_finetune", cx, CPU_BUDGET_S["other"])
        entries["switch"] = measure_switch(cx, CPU_BUDGET_S["other"])
        entries["factor_qr"] = measure_tsqr(cx, CPU_BUDGET_S["other"])
        entries["compress"] = measure_compress(cx, CPU_BUDGET_S["other"])
    head = entries[HEADLINE if a.config == "all" else a.config]
    out = {k: head[k] for k in HEAD_KEYS if k in head}
    if a.config == "all":
        out["headline"] = f"{HEADLINE} (the largest single-GPU configuration); every workload under configs"
        out["configs"] = entries
    if cx.rank == 0:
        print(json.dumps(out), flush=True)
    if cx.world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- launchers
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun_command(argv, n):
    """The command that runs this script with n processes (one per GPU) under
    torchrun on this node, with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.abspath(__file__), *argv]


def run_dry(a):
    """No GPU: each rank joins a gloo group, takes one data-parallel gradient
    exchange and the max over ranks of a time, and rank 0 prints a line."""
    import datetime
    import torch
    import torch.distributed as dist
    rank, _, world = dist_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    g = torch.full((4,), float(rank + 1), dtype=torch.float32)
    allreduce_grads(g, world)
    ms = max_over_ranks(1.0 + rank, world)
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "grad_sum": float(g[0]), "max_ms": ms}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    a = parse(argv)
    rank, _, world = dist_env()
    if a.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start N ranks of this script under torchrun
        r = subprocess.run(torchrun_command(argv, a.gpus))
        sys.exit(r.returncode)
    if a.gpus != world and rank == 0:
        print(f"bench.py: --gpus {a.gpus} but {world} process(es) (WORLD_SIZE); the line reports the processes "
              f"that ran", file=sys.stderr)
    if a.dry_run:
        run_dry(a)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_lora(a)


if __name__ == "__main__":
    main()
