"""lora_linear_bwd_static: the backward for callers that cannot allocate device
memory (for example when a framework or a serving process owns all of the
device's memory through its own allocator, or a host program gives a plugin no
allocator). It must give the same results as lora_linear_bwd with a
caller-provided workspace, call after call, while allocating nothing itself.

This file is collected last (pytest orders files by name), so that a failure
here never hides the results of the other GPU tests."""

from __future__ import annotations

import numpy as np
import pytest

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


def _forward(inp, bits=None):
    import lora_adapter_execution_b200 as lora
    r = int(inp.ranks[0])
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    X, W = dev_bf16(inp.X), dev_bf16(inp.W)
    A, B = dev_bf16(inp.A_pool), dev_bf16(inp.B_pool)
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    U = torch.empty(inp.T, r, dtype=torch.float32, device="cuda")
    lora.linear_fwd(plan, X, W, A, B, torch.from_numpy(inp.scale).cuda(), Y, p_drop=inp.p_drop,
                    seed=inp.mask_seed, U_save=U, keep_bits=bits)
    plan.destroy()
    return X, W, A, B, U, dev_bf16(inp.dY)


def _outputs(inp):
    r = int(inp.ranks[0])
    return (torch.empty(inp.T, inp.d_in, dtype=torch.bfloat16, device="cuda"),
            torch.empty(r, inp.d_in, dtype=torch.float32, device="cuda"),
            torch.empty(r, inp.d_out, dtype=torch.float32, device="cuda"))


def _same_bits(a, b):
    view = torch.int16 if a.dtype == torch.bfloat16 else torch.int32
    return torch.equal(a.view(view), b.view(view))


@pytest.mark.parametrize("kw,with_bits", [(dict(T=1500, d_in=520, d_out=264, p_drop=0.1), False),
                                          (dict(T=1024, d_in=512, d_out=256, p_drop=0.2), True)])
def test_static_scratch_backward_matches_workspace_backward(kw, with_bits):
    """Two calls in a row through the no-allocation entry point give bit for bit
    the results of lora_linear_bwd with a caller-allocated workspace: the same
    kernels run on the same scratch layout, only its address differs. The second
    case passes the dropout keep bits with d_in a multiple of 128, so the dA
    contraction stages them through the copy engine."""
    import lora_adapter_execution_b200 as lora
    inp = wl.make_inputs("finetune", **kw)
    bits = None
    if with_bits:
        bits = torch.empty(inp.T, -(-inp.d_in // 32), dtype=torch.int32, device="cuda")
        lora.dropout_keep_bits(inp.mask_seed, inp.p_drop, bits, inp.d_in)
    X, W, A, B, U, dY = _forward(inp, bits)
    s = float(inp.scale[0])
    assert lora.bwd_workspace_size(inp.T, inp.d_in, inp.d_out, int(inp.ranks[0])) <= (8 << 20)
    # reference: the existing entry point with a caller-allocated workspace
    ref = _outputs(inp)
    ws = torch.empty(lora.bwd_workspace_size(inp.T, inp.d_in, inp.d_out, int(inp.ranks[0])),
                     dtype=torch.uint8, device="cuda")
    lora.linear_bwd(X, W, A, B, s, U, dY, *ref, ws, p_drop=inp.p_drop, seed=inp.mask_seed, keep_bits=bits)
    assert lora.device_status() == 0
    # two calls in a row through the no-allocation entry point; the second one
    # runs on the scratch contents the first one left behind
    for call in range(2):
        got = _outputs(inp)
        lora.linear_bwd_static(X, W, A, B, s, U, dY, *got, p_drop=inp.p_drop, seed=inp.mask_seed, keep_bits=bits)
        assert lora.device_status() == 0
        for name, g, w in zip(("dX", "dA", "dB"), got, ref):
            assert _same_bits(g, w), f"call {call} {name} differs from the workspace backward"
    # and both agree with the oracle within the parity tolerance
    import oracle
    rdX, rdA, rdB = oracle.backward(inp)
    for name, g, w in zip(("dX", "dA", "dB"), got, (rdX, rdA, rdB)):
        check_close(host_f64(g), w, name)


def test_static_scratch_backward_rejects_oversized_requests():
    """A request whose scratch need exceeds the 8 MiB array is refused with
    LORA_ERR_WORKSPACE. The entry point checks the size before it reads any
    pointer or makes any CUDA call, so the 16-byte stand-in buffers passed here
    for every tensor are never touched."""
    import lora_adapter_execution_b200 as lora
    from lora_adapter_execution_b200 import abi
    T, d_in, d_out, r = 1 << 16, 4096, 4096, 64
    assert lora.bwd_workspace_size(T, d_in, d_out, r) > (8 << 20)
    t = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = abi._ptr(t)
    L = lora.load_library()
    rc = L.lora_linear_bwd_static(p, p, p, p, 1.0, 0.0, 0, p, p, p, p, p, T, d_in, d_out, r, None,
                                  abi._stream(None))
    assert rc == -8  # LORA_ERR_WORKSPACE, nothing launched
    assert lora.device_status() == 0
