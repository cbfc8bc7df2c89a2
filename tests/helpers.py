"""Shared test utilities: device transfer of bf16 bit arrays and the parity check."""

from __future__ import annotations

import numpy as np

from lora_adapter_execution_b200 import workloads as wl

# Tolerance for bf16 I/O with fp32 accumulation, against the fp64 oracle.
REL_FRO = 5e-3
ELEM = 3e-2


def check_close(got, ref, what="", rel_fro=REL_FRO, elem=ELEM):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = got - ref
    nref = np.linalg.norm(ref)
    fro = np.linalg.norm(err) / (nref if nref > 0 else 1.0)
    bad = np.abs(err) > elem * np.maximum(1.0, np.abs(ref))
    assert fro <= rel_fro, f"{what}: rel-Frobenius {fro:.3e} > {rel_fro}"
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements off, first {idx.tolist()} "
                             f"got {got[tuple(idx[0])]} ref {ref[tuple(idx[0])]}")
    return fro


def dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_f64(t):
    import torch
    if t.dtype == torch.bfloat16:
        return wl.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.double().cpu().numpy()


def host_bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)
