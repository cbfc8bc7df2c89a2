"""C-ABI library checks that need no GPU: it loads, exports every function the
header declares, maps status codes to strings, and validates arguments on the
host before touching CUDA."""

from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

import lora_adapter_execution_b200 as lora
from lora_adapter_execution_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "lora.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_\s\*]*?\b(lora_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_header_function():
    L = abi.load_library()
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_nm_exports():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (lora_[a-z0-9_]+)", out))
    assert set(header_functions()) <= exported


def test_status_strings():
    L = abi.load_library()
    for code in list(abi.STATUS_NAMES) + [-99]:
        s = L.lora_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0


def _host_plan(ids, ranks, d_in=64, d_out=64):
    L = abi.load_library()
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    ranks = np.ascontiguousarray(ranks, dtype=np.int32)
    h = ctypes.c_void_p()
    rc = L.lora_plan_build_host(ids.ctypes.data_as(ctypes.c_void_p), ids.shape[0],
                                ranks.ctypes.data_as(ctypes.c_void_p), ranks.shape[0], d_in, d_out,
                                ctypes.byref(h))
    if rc == 0:
        L.lora_plan_destroy(h)
    return rc


def test_plan_argument_errors():
    assert _host_plan([0, 1, 2], [4, 4, 4]) == 0
    assert _host_plan([0, 3], [4, 4, 4]) == -2           # id out of range
    assert _host_plan([-1], [4]) == -2
    assert _host_plan([0] * 300 + [3], [4, 4, 4]) == -2   # last id of a long run of valid ones
    assert _host_plan([], [4]) == -1                      # an empty batch (T = 0)
    assert _host_plan([0], []) == -1                      # no adapters
    assert _host_plan([1] * 50 + [-2**31] + [1] * 50, [4, 4]) == -2
    assert _host_plan([0], [0]) == -3                     # rank 0
    assert _host_plan([0], [257]) == -3                   # rank above the maximum
    assert _host_plan([0], [4], d_in=12) == -1            # not a multiple of 8
    assert _host_plan([0], [4], d_out=0) == -1
    L = abi.load_library()
    assert L.lora_plan_build_host(None, 1, None, 1, 64, 64, ctypes.byref(ctypes.c_void_p())) == -1


def test_null_plan_calls():
    L = abi.load_library()
    assert L.lora_plan_get(None, None, None, None) == -1
    assert L.lora_plan_info(None, None) == -1
    L.lora_plan_destroy(None)  # ignored
    assert L.lora_linear_fwd(None, None, None, None, None, None, 0.0, 0, None, None, None, None) == -1
    assert L.lora_linear_fwd_host(None, None, 0, None, 0, None, None, None, None, None, None, 0.0, 0, None, None,
                                  None, None, None) == -1


def test_fwd_host_step_rejects_a_host_only_plan_before_cuda():
    """lora_linear_fwd_host checks its plan and buffers before it queues
    anything: a host-only plan (no device tables) and null buffers are argument
    errors, with no CUDA call made."""
    L = abi.load_library()
    ids = np.zeros(4, dtype=np.int32)
    ranks = np.array([4], dtype=np.int32)
    h = ctypes.c_void_p()
    assert L.lora_plan_build_host(ids.ctypes.data_as(ctypes.c_void_p), 4, ranks.ctypes.data_as(ctypes.c_void_p), 1,
                                  64, 64, ctypes.byref(h)) == 0
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    idp, rp = ids.ctypes.data_as(ctypes.c_void_p), ranks.ctypes.data_as(ctypes.c_void_p)
    assert L.lora_linear_fwd_host(h, idp, 4, rp, 1, p, p, p, p, p, p, 0.0, 0, p, p, None, None, None) == -1
    assert L.lora_linear_fwd_host(h, idp, 4, rp, 1, None, p, p, p, p, p, 0.0, 0, p, p, None, None, None) == -1
    L.lora_plan_destroy(h)


def test_bwd_workspace_size_monotone():
    a = lora.bwd_workspace_size(4096, 4096, 4096, 16)
    b = lora.bwd_workspace_size(16384, 4096, 4096, 16)
    assert 0 < a < b
    assert lora.bwd_workspace_size(0, 4096, 4096, 16) == 0


def test_bwd_rejects_bad_rank_before_cuda():
    L = abi.load_library()
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    for bad_rank in (0, -1, 257):
        rc = L.lora_linear_bwd(p, p, p, p, 1.0, 0.0, 0, p, p, p, p, p, 64, 64, 64, bad_rank, p, 1 << 20, None, None)
        assert rc == -3
    rc = L.lora_linear_bwd(p, p, p, p, 1.0, 0.0, 0, p, p, p, p, p, 64, 64, 64, 16, None, 0, None, None)
    assert rc == -8
    rc = L.lora_linear_bwd(p, p, p, p, 1.0, 0.0, 0, p, p, p, p, p, 64, 64, 64, 5, p, 64, None, None)
    assert rc == -8  # a workspace smaller than the rank-5 layout needs


def test_binding_checks_tensor_metadata_before_the_call():
    """The binding rejects a tensor whose shape, dtype, layout or device does not
    match the sizes the library will read, before any library call (a host-only
    plan and CPU tensors: nothing reaches CUDA)."""
    import torch
    T, d_in, d_out = 40, 64, 48
    ids = np.arange(T, dtype=np.int32) % 3
    ranks = np.array([4, 8, 16], dtype=np.int32)
    plan = lora.Plan(ids, ranks, d_in, d_out, host_only=True)
    assert plan.pool_rows == 28 and plan.r_max == 16
    bf = torch.bfloat16
    good = dict(X=torch.zeros(T, d_in, dtype=bf), W=torch.zeros(d_in, d_out, dtype=bf),
                A_pool=torch.zeros(28, d_in, dtype=bf), B_pool=torch.zeros(28, d_out, dtype=bf),
                scale=torch.ones(3, dtype=torch.float32), Y=torch.zeros(T, d_out, dtype=bf))

    def fwd(**over):
        a = dict(good, **over)
        with pytest.raises(lora.LoraError) as e:
            lora.linear_fwd(plan, a["X"], a["W"], a["A_pool"], a["B_pool"], a["scale"], a["Y"],
                            U_save=a.get("U_save"), keep_bits=a.get("keep_bits"))
        assert e.value.code == -1
        return str(e.value)

    assert "X has shape" in fwd(X=torch.zeros(T - 1, d_in, dtype=bf))
    assert "A_pool has shape" in fwd(A_pool=torch.zeros(16, d_in, dtype=bf))
    assert "scale has shape" in fwd(scale=torch.ones(2, dtype=torch.float32))
    assert "U_save has shape" in fwd(U_save=torch.zeros(T, 8, dtype=torch.float32))
    assert "keep_bits has shape" in fwd(keep_bits=torch.zeros(T, 1, dtype=torch.int32))
    assert "W has dtype" in fwd(W=torch.zeros(d_in, d_out, dtype=torch.float16))
    assert "Y is not contiguous" in fwd(Y=torch.zeros(d_out, T, dtype=bf).t())
    assert "X is not a CUDA tensor" in fwd()
    with pytest.raises(lora.LoraError, match="dB has shape"):
        r = 8
        lora.linear_bwd(good["X"], good["W"], torch.zeros(r, d_in, dtype=bf), torch.zeros(r, d_out, dtype=bf), 1.0,
                        torch.zeros(T, r, dtype=torch.float32), torch.zeros(T, d_out, dtype=bf),
                        torch.zeros(T, d_in, dtype=bf), torch.zeros(r, d_in, dtype=torch.float32),
                        torch.zeros(r, d_in, dtype=torch.float32), torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(lora.LoraError, match="bits has shape"):
        lora.dropout_keep_bits(0, 0.1, torch.zeros(T, 3, dtype=torch.int32), d_in)
    plan.destroy()


def test_qr_and_compression_reject_bad_arguments_before_cuda():
    """The tall-skinny QR and the compression calls validate their sizes and
    pointers on the host first (LORA_ERR_ARG = -1), with no CUDA call; their
    workspace-size queries return 0 for sizes out of range."""
    L = abi.load_library()
    vp = ctypes.c_void_p
    fake = vp(0x1000)  # never dereferenced: every call below fails its checks first
    # workspace sizes: n out of range, m < n
    assert L.lora_tsqr_workspace_size(4, 100, 65, 1) == 0
    assert L.lora_tsqr_workspace_size(4, 10, 16, 1) == 0
    assert L.lora_tsqr_workspace_size(4, 4096, 16, 1) > L.lora_tsqr_workspace_size(4, 4096, 16, 0) > 0
    assert L.lora_compress_workspace_size(8, 4096, 4096, 0) == 0
    assert L.lora_compress_workspace_size(8, 4096, 4096, 65) == 0
    assert L.lora_compress_workspace_size(8, 12, 4096, 16) == 0   # r > d_in
    assert L.lora_compress_allocate_workspace_size(0, 16) == 0
    # lora_tsqr: null F or R, n > 64, m < n, ld < m
    assert L.lora_tsqr(None, 4096, 0, 1, 4096, 16, fake, None, None, 0, None) == -1
    assert L.lora_tsqr(fake, 4096, 0, 1, 4096, 16, None, None, None, 0, None) == -1
    assert L.lora_tsqr(fake, 4096, 0, 1, 4096, 65, fake, None, None, 0, None) == -1
    assert L.lora_tsqr(fake, 4096, 0, 1, 8, 16, fake, None, None, 0, None) == -1
    assert L.lora_tsqr(fake, 100, 0, 1, 4096, 16, fake, None, None, 0, None) == -1
    # lora_compress_spectra: null factors or sigma, rank 0
    assert L.lora_compress_spectra(None, 0, fake, 0, 2, 256, 256, 8, fake, fake, 1 << 30, None) == -1
    assert L.lora_compress_spectra(fake, 0, fake, 0, 2, 256, 256, 8, None, fake, 1 << 30, None) == -1
    assert L.lora_compress_spectra(fake, 0, fake, 0, 2, 256, 256, 0, fake, fake, 1 << 30, None) == -1
    # lora_compress_allocate: policy, keep outside [0, 1], negative floor, r_max > 64
    assert L.lora_compress_allocate(fake, fake, fake, 4, 16, 2, 0.5, 1, fake, fake, fake, 1024, None) == -1
    assert L.lora_compress_allocate(fake, fake, fake, 4, 16, 1, 1.5, 1, fake, fake, fake, 1024, None) == -1
    assert L.lora_compress_allocate(fake, fake, fake, 4, 16, 1, 0.5, -1, fake, fake, fake, 1024, None) == -1
    assert L.lora_compress_allocate(fake, fake, fake, 4, 65, 1, 0.5, 1, fake, fake, fake, 1024, None) == -1
    # lora_compress_export: null pools
    assert L.lora_compress_export(fake, fake, fake, 2, 256, 256, 8, None, fake, fake, 1 << 30, None) == -1
    assert L.lora_compress_export(fake, fake, fake, 2, 256, 256, 8, fake, None, fake, 1 << 30, None) == -1
