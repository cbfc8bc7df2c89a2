"""ctypes binding of include/lora.h (argument marshalling only).

Tensors are torch CUDA tensors (bf16 where the ABI says bf16); each call passes
their raw device pointers and the current torch stream to the library. Nothing
here computes any part of the layer. The ABI takes every size from the plan or
from other arguments, so before a pointer crosses it the tensor's metadata is
checked against those sizes (exact shape, dtype, contiguous, on the current
CUDA device); a mismatch raises LoraError with LORA_ERR_ARG and calls nothing.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblora_b200.so")

LORA_OK = 0
STATUS_NAMES = {0: "LORA_OK", -1: "LORA_ERR_ARG", -2: "LORA_ERR_ID", -3: "LORA_ERR_RANK",
                -4: "LORA_ERR_CUDA", -5: "LORA_ERR_DEVICE", -6: "LORA_ERR_UNSUPPORTED",
                -7: "LORA_ERR_NOMEM", -8: "LORA_ERR_WORKSPACE"}

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_u64 = ctypes.c_uint64
_dbl = ctypes.c_double
_f32 = ctypes.c_float
_sz = ctypes.c_size_t


class LoraError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({_lib_or_none_str(code)})")


class _Info(ctypes.Structure):
    _fields_ = [("T", _i64), ("d_in", _i64), ("d_out", _i64), ("n_adapters", _i32),
                ("n_segments", _i32), ("n_tiles", _i32), ("r_max", _i32), ("sum_r_used", _i64),
                ("sum_r_tokens", _i64), ("aug_k_total", _i64), ("scratch_bytes", _i64),
                ("gathers_x", _i32)]


_lib = None


def _lib_or_none_str(code):
    try:
        return load_library().lora_status_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


def load_library():
    """Load liblora_b200.so; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run python -m lora_adapter_execution_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "lora_plan_build": (ctypes.c_int, [_vp, _i64, _vp, _i32, _i64, _i64, _vp, ctypes.POINTER(_vp)]),
        "lora_plan_rebuild": (ctypes.c_int, [_vp, _vp, _i64, _vp, _i32, _i64, _i64, _vp]),
        "lora_plan_build_host": (ctypes.c_int, [_vp, _i64, _vp, _i32, _i64, _i64, ctypes.POINTER(_vp)]),
        "lora_plan_get": (ctypes.c_int, [_vp, _vp, _vp, _vp]),
        "lora_plan_info": (ctypes.c_int, [_vp, ctypes.POINTER(_Info)]),
        "lora_plan_destroy": (None, [_vp]),
        "lora_linear_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _dbl, _u64, _vp, _vp, _vp, _vp]),
        "lora_linear_fwd_fused": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _dbl, _u64, _vp, _vp, _vp, _vp]),
        "lora_linear_fwd_host": (ctypes.c_int, [_vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dbl, _u64,
                                                _vp, _vp, _vp, _vp, _vp]),
        "lora_linear_shrink": (ctypes.c_int, [_vp, _vp, _vp, _vp, _dbl, _u64, _vp, _vp, _vp]),
        "lora_fused_gemm": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp]),
        "lora_base_gemm": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i64, _i64, _vp]),
        "lora_linear_bwd_workspace_size": (_sz, [_i64, _i64, _i64, _i32]),
        "lora_linear_bwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _f32, _dbl, _u64, _vp, _vp, _vp, _vp, _vp,
                                           _i64, _i64, _i64, _i32, _vp, _sz, _vp, _vp]),
        "lora_linear_bwd_static": (ctypes.c_int, [_vp, _vp, _vp, _vp, _f32, _dbl, _u64, _vp, _vp, _vp, _vp, _vp,
                                                  _i64, _i64, _i64, _i32, _vp, _vp]),
        "lora_dropout_mask": (ctypes.c_int, [_u64, _dbl, _i64, _i64, _vp, _vp]),
        "lora_dropout_keep_bits": (ctypes.c_int, [_u64, _dbl, _i64, _i64, _vp, _vp]),
        "lora_device_status": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
        "lora_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, _vp, _vp]),
        "lora_dropout_seed_for_rows": (_u64, [_u64, _i64, _i64]),
        "lora_linear_bwd_multi_workspace_size": (_sz, [_vp]),
        "lora_linear_bwd_multi": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _dbl, _u64, _vp, _vp, _vp, _vp, _vp,
                                                 _vp, _sz, _vp, _vp]),
        "lora_switch_create": (ctypes.c_int, [_vp, _i32, _i64, _i64, _i64, _i32, ctypes.POINTER(_vp)]),
        "lora_switch_apply": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp]),
        "lora_switch_destroy": (None, [_vp]),
        "lora_tsqr_workspace_size": (_sz, [_i64, _i64, _i32, ctypes.c_int]),
        "lora_tsqr": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _sz, _vp]),
        "lora_compress_workspace_size": (_sz, [_i64, _i64, _i64, _i32]),
        "lora_compress_spectra": (ctypes.c_int, [_vp, _i64, _vp, _i64, _i64, _i64, _i64, _i32, _vp, _vp, _sz, _vp]),
        "lora_compress_allocate_workspace_size": (_sz, [_i64, _i32]),
        "lora_compress_allocate": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i32, _i32, _dbl, _i32, _vp, _vp, _vp, _sz,
                                                  _vp]),
        "lora_compress_export": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _sz, _vp]),
        "lora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != LORA_OK:
        raise LoraError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_BF16 = ("bfloat16",)
_F32 = ("float32",)
_I32 = ("int32", "uint32")


_DTYPE_NAME = {}  # torch dtype -> its short name ("bfloat16", ...), filled as dtypes are seen


def _dtype_name(dt):
    n = _DTYPE_NAME.get(dt)
    if n is None:
        n = _DTYPE_NAME[dt] = str(dt).rsplit(".", 1)[-1]
    return n


def _args(what, *specs):
    """Check (name, tensor, shape, dtype names, optional) for each tensor handed
    to the library call `what`: first every tensor's shape, dtype and layout,
    then every tensor's device. (Called on every launch: the checks use the
    cheapest accessors, a cached dtype name and the device index as an int.)"""
    given = []
    for name, t, shape, dtypes, optional in specs:
        if t is None:
            if optional:
                continue
            raise LoraError(-1, f"{what}: {name} is required")
        if t.shape != tuple(shape):
            raise LoraError(-1, f"{what}: {name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if _dtype_name(t.dtype) not in dtypes:
            raise LoraError(-1, f"{what}: {name} has dtype {t.dtype}, expected {' or '.join(dtypes)}")
        if not t.is_contiguous():
            raise LoraError(-1, f"{what}: {name} is not contiguous")
        given.append((name, t))
    dev = None
    for name, t in given:
        idx = t.get_device()  # -1 for a host tensor
        if idx < 0:
            raise LoraError(-1, f"{what}: {name} is not a CUDA tensor")
        if dev is None:
            import torch
            dev = torch.cuda.current_device()
        if idx != dev:
            raise LoraError(-1, f"{what}: {name} is on {t.device}, the current device is cuda:{dev}")


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _host_i32(a):
    a = a.cpu().numpy() if hasattr(a, "cpu") else a
    return np.ascontiguousarray(a, dtype=np.int32)


class Plan:
    """A batch's token-by-adapter grouping (lora_plan_build / lora_plan_build_host)."""

    def __init__(self, ids, ranks, d_in: int, d_out: int, *, stream=None, host_only: bool = False):
        L = load_library()
        self._ids = _host_i32(ids)
        self._ranks = _host_i32(ranks)
        h = _vp()
        T, n = self._ids.shape[0], self._ranks.shape[0]
        if host_only:
            rc = L.lora_plan_build_host(self._ids.ctypes.data_as(_vp), T, self._ranks.ctypes.data_as(_vp), n,
                                        d_in, d_out, ctypes.byref(h))
        else:
            rc = L.lora_plan_build(self._ids.ctypes.data_as(_vp), T, self._ranks.ctypes.data_as(_vp), n,
                                   d_in, d_out, _stream(stream), ctypes.byref(h))
        _check(rc, "lora_plan_build")
        self._h = h
        self.T, self.d_in, self.d_out, self.n_adapters = T, d_in, d_out, n
        self._sizes(True)

    def _sizes(self, ranks_changed):
        # pool rows (all adapters' ranks) and U_save's row length (the largest
        # rank among adapters with tokens), as the library reads them
        if ranks_changed:
            self.pool_rows = int(self._ranks.astype(np.int64).sum())
        inf = _Info()
        _check(load_library().lora_plan_info(self._h, ctypes.byref(inf)), "lora_plan_info")
        self.r_max = int(inf.r_max)

    def rebuild(self, ids, *, ranks=None, stream=None):
        """lora_plan_rebuild: the same plan object for a new batch (device buffers
        reused when they fit). Stream-ordered on `stream` (default: the current
        torch stream): run the plan's work there or after it; work on other
        streams that still uses the old tables must be ordered first."""
        self._ids = _host_i32(ids)
        if ranks is not None:
            self._ranks = _host_i32(ranks)
        T, n = self._ids.shape[0], self._ranks.shape[0]
        _check(load_library().lora_plan_rebuild(self._h, self._ids.ctypes.data_as(_vp), T,
                                                self._ranks.ctypes.data_as(_vp), n, self.d_in, self.d_out,
                                                _stream(stream)), "lora_plan_rebuild")
        self.T, self.n_adapters = T, n
        self._sizes(ranks is not None)

    @property
    def handle(self):
        return self._h

    def info(self) -> dict:
        inf = _Info()
        _check(load_library().lora_plan_info(self._h, ctypes.byref(inf)), "lora_plan_info")
        return {f: getattr(inf, f) for f, _ in _Info._fields_}

    def grouping(self):
        L = load_library()
        ns = _i32(0)
        _check(L.lora_plan_get(self._h, None, None, ctypes.byref(ns)), "lora_plan_get")
        perm = np.empty(self.T, dtype=np.int32)
        seg = np.empty((max(ns.value, 1), 3), dtype=np.int32)
        _check(L.lora_plan_get(self._h, perm.ctypes.data_as(_vp), seg.ctypes.data_as(_vp), None), "lora_plan_get")
        return perm, seg[: ns.value].copy()

    def destroy(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load_library().lora_plan_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def _fwd_args(plan, X, A_pool, scale, U_save, keep_bits):
    T, di, R = plan.T, plan.d_in, plan.pool_rows
    return (("X", X, (T, di), _BF16, False), ("A_pool", A_pool, (R, di), _BF16, False),
            ("scale", scale, (plan.n_adapters,), _F32, False), ("U_save", U_save, (T, plan.r_max), _F32, True),
            ("keep_bits", keep_bits, (T, -(-di // 32)), _I32, True))


def linear_fwd(plan: Plan, X, W, A_pool, B_pool, scale, Y, *, p_drop: float = 0.0, seed: int = 0,
               U_save=None, keep_bits=None, stream=None):
    di, do, R = plan.d_in, plan.d_out, plan.pool_rows
    _args("lora_linear_fwd", *_fwd_args(plan, X, A_pool, scale, U_save, keep_bits),
          ("W", W, (di, do), _BF16, False), ("B_pool", B_pool, (R, do), _BF16, False),
          ("Y", Y, (plan.T, do), _BF16, False))
    _check(load_library().lora_linear_fwd(plan.handle, _ptr(X), _ptr(W), _ptr(A_pool), _ptr(B_pool), _ptr(scale),
                                          float(p_drop), int(seed) & (2**64 - 1), _ptr(Y), _ptr(U_save),
                                          _ptr(keep_bits), _stream(stream)), "lora_linear_fwd")


def linear_fwd_host(plan: Plan, ids, X_host, X_dev, W, A_pool, B_pool, scale, Y_dev, Y_host, *,
                    p_drop: float = 0.0, seed: int = 0, U_save=None, keep_bits=None, stream=None):
    """lora_linear_fwd_host: one step from host memory (the plan rebuilt from the
    host ids with its current ranks, X_host copied into X_dev, the forward into
    Y_dev, Y_dev copied into Y_host), queued on `stream` (default: the current
    torch stream); Y_host holds the result once the stream has passed the call.
    X_host and Y_host are host tensors (pinned for the copies to overlap)."""
    ids = _host_i32(ids)
    T = ids.shape[0]
    di, do, R = plan.d_in, plan.d_out, plan.pool_rows
    for name, t, shape in (("X_host", X_host, (T, di)), ("Y_host", Y_host, (T, do))):
        if t.shape != shape or _dtype_name(t.dtype) not in _BF16 or not t.is_contiguous():
            raise LoraError(-1, f"lora_linear_fwd_host: {name} must be a contiguous bfloat16 tensor of shape {shape}")
        if t.get_device() >= 0:
            raise LoraError(-1, f"lora_linear_fwd_host: {name} must be in host memory")
    # U_save's rows are as long as the largest rank among the batch's adapters
    # (ids out of range: the library reports them before anything is queued)
    rmax = 0
    if U_save is not None:
        valid = T > 0 and ids.min() >= 0 and ids.max() < plan._ranks.shape[0]
        rmax = int(plan._ranks[ids].max()) if valid else (U_save.shape[1] if U_save.dim() == 2 else 0)
    _args("lora_linear_fwd_host", ("X_dev", X_dev, (T, di), _BF16, False), ("W", W, (di, do), _BF16, False),
          ("A_pool", A_pool, (R, di), _BF16, False), ("B_pool", B_pool, (R, do), _BF16, False),
          ("scale", scale, (plan.n_adapters,), _F32, False), ("Y_dev", Y_dev, (T, do), _BF16, False),
          ("U_save", U_save, (T, rmax), _F32, True), ("keep_bits", keep_bits, (T, -(-di // 32)), _I32, True))
    _check(load_library().lora_linear_fwd_host(plan.handle, ids.ctypes.data_as(_vp), T,
                                               plan._ranks.ctypes.data_as(_vp), plan._ranks.shape[0],
                                               _ptr(X_host), _ptr(X_dev), _ptr(W), _ptr(A_pool), _ptr(B_pool),
                                               _ptr(scale), float(p_drop), int(seed) & (2**64 - 1), _ptr(Y_dev),
                                               _ptr(Y_host), _ptr(U_save), _ptr(keep_bits), _stream(stream)),
           "lora_linear_fwd_host")
    plan._ids = ids
    plan.T = T
    plan._sizes(False)


def linear_fwd_fused(plan: Plan, X, W, A_pool, B_pool, scale, Y, *, p_drop: float = 0.0, seed: int = 0,
                     U_save=None, keep_bits=None, stream=None):
    """lora_linear_fwd_fused: the forward (row gather, shrink and fused GEMM) in one launch."""
    di, do, R = plan.d_in, plan.d_out, plan.pool_rows
    _args("lora_linear_fwd_fused", *_fwd_args(plan, X, A_pool, scale, U_save, keep_bits),
          ("W", W, (di, do), _BF16, False), ("B_pool", B_pool, (R, do), _BF16, False),
          ("Y", Y, (plan.T, do), _BF16, False))
    _check(load_library().lora_linear_fwd_fused(plan.handle, _ptr(X), _ptr(W), _ptr(A_pool), _ptr(B_pool),
                                                _ptr(scale), float(p_drop), int(seed) & (2**64 - 1), _ptr(Y),
                                                _ptr(U_save), _ptr(keep_bits), _stream(stream)),
           "lora_linear_fwd_fused")


def linear_shrink(plan: Plan, X, A_pool, scale, *, p_drop: float = 0.0, seed: int = 0, U_save=None,
                  keep_bits=None, stream=None):
    _args("lora_linear_shrink", *_fwd_args(plan, X, A_pool, scale, U_save, keep_bits))
    _check(load_library().lora_linear_shrink(plan.handle, _ptr(X), _ptr(A_pool), _ptr(scale), float(p_drop),
                                             int(seed) & (2**64 - 1), _ptr(U_save), _ptr(keep_bits),
                                             _stream(stream)),
           "lora_linear_shrink")


def fused_gemm(plan: Plan, X, W, B_pool, Y, *, stream=None):
    T, di, do = plan.T, plan.d_in, plan.d_out
    _args("lora_fused_gemm", ("X", X, (T, di), _BF16, False), ("W", W, (di, do), _BF16, False),
          ("B_pool", B_pool, (plan.pool_rows, do), _BF16, False), ("Y", Y, (T, do), _BF16, False))
    _check(load_library().lora_fused_gemm(plan.handle, _ptr(X), _ptr(W), _ptr(B_pool), _ptr(Y), _stream(stream)),
           "lora_fused_gemm")


def base_gemm(X, W, Y, *, stream=None):
    T, d_in = X.shape
    d_out = W.shape[1]
    _args("lora_base_gemm", ("X", X, (T, d_in), _BF16, False), ("W", W, (d_in, d_out), _BF16, False),
          ("Y", Y, (T, d_out), _BF16, False))
    _check(load_library().lora_base_gemm(_ptr(X), _ptr(W), _ptr(Y), T, d_in, d_out, _stream(stream)),
           "lora_base_gemm")


def bwd_workspace_size(T: int, d_in: int, d_out: int, r: int) -> int:
    return int(load_library().lora_linear_bwd_workspace_size(T, d_in, d_out, r))


def _bwd_args(X, W, A, B, U_save, dY, dX, dA, dB, keep_bits):
    T, di = X.shape
    do = W.shape[1]
    r = A.shape[0]
    return (("X", X, (T, di), _BF16, False), ("W", W, (di, do), _BF16, False), ("A", A, (r, di), _BF16, False),
            ("B", B, (r, do), _BF16, False), ("U_save", U_save, (T, r), _F32, False),
            ("dY", dY, (T, do), _BF16, False), ("dX", dX, (T, di), _BF16, False),
            ("dA", dA, (r, di), _F32, False), ("dB", dB, (r, do), _F32, False),
            ("keep_bits", keep_bits, (T, -(-di // 32)), _I32, True))


def linear_bwd(X, W, A, B, scale: float, U_save, dY, dX, dA, dB, workspace, *, p_drop: float = 0.0,
               seed: int = 0, keep_bits=None, stream=None):
    T, d_in = X.shape
    d_out = W.shape[1]
    r = A.shape[0]
    _args("lora_linear_bwd", *_bwd_args(X, W, A, B, U_save, dY, dX, dA, dB, keep_bits))
    _args("lora_linear_bwd", ("workspace", workspace, tuple(workspace.shape), (str(workspace.dtype)[6:],), False))
    nbytes = workspace.numel() * workspace.element_size()
    _check(load_library().lora_linear_bwd(_ptr(X), _ptr(W), _ptr(A), _ptr(B), float(scale), float(p_drop),
                                          int(seed) & (2**64 - 1), _ptr(U_save), _ptr(dY), _ptr(dX), _ptr(dA),
                                          _ptr(dB), T, d_in, d_out, r, _ptr(workspace), nbytes, _ptr(keep_bits),
                                          _stream(stream)),
           "lora_linear_bwd")


def bwd_multi_workspace_size(plan: Plan) -> int:
    return int(load_library().lora_linear_bwd_multi_workspace_size(plan.handle))


def linear_bwd_multi(plan: Plan, X, W, A_pool, B_pool, scale, U_save, dY, dX, dA_pool, dB_pool, workspace, *,
                     p_drop: float = 0.0, seed: int = 0, keep_bits=None, stream=None):
    """lora_linear_bwd_multi: the backward of a mixed-adapter batch over its plan
    (dX, and the gradient rows of every adapter with tokens in dA_pool, dB_pool)."""
    T, di, do, R = plan.T, plan.d_in, plan.d_out, plan.pool_rows
    _args("lora_linear_bwd_multi", *_fwd_args(plan, X, A_pool, scale, U_save, keep_bits),
          ("W", W, (di, do), _BF16, False), ("B_pool", B_pool, (R, do), _BF16, False),
          ("dY", dY, (T, do), _BF16, False), ("dX", dX, (T, di), _BF16, False),
          ("dA_pool", dA_pool, (R, di), _F32, False), ("dB_pool", dB_pool, (R, do), _F32, False),
          ("workspace", workspace, tuple(workspace.shape), (str(workspace.dtype)[6:],), False))
    if U_save is None:
        raise LoraError(-1, "lora_linear_bwd_multi: U_save is required")
    nbytes = workspace.numel() * workspace.element_size()
    _check(load_library().lora_linear_bwd_multi(plan.handle, _ptr(X), _ptr(W), _ptr(A_pool), _ptr(B_pool), _ptr(scale),
                                                float(p_drop), int(seed) & (2**64 - 1), _ptr(U_save), _ptr(dY),
                                                _ptr(dX), _ptr(dA_pool), _ptr(dB_pool), _ptr(workspace), nbytes,
                                                _ptr(keep_bits), _stream(stream)),
           "lora_linear_bwd_multi")


def linear_bwd_static(X, W, A, B, scale: float, U_save, dY, dX, dA, dB, *, p_drop: float = 0.0,
                      seed: int = 0, keep_bits=None, stream=None):
    """lora_linear_bwd_static: the backward without a caller workspace (for callers
    that cannot allocate device memory); see include/lora.h for its limit and
    sharing rules."""
    T, d_in = X.shape
    d_out = W.shape[1]
    r = A.shape[0]
    _args("lora_linear_bwd_static", *_bwd_args(X, W, A, B, U_save, dY, dX, dA, dB, keep_bits))
    _check(load_library().lora_linear_bwd_static(_ptr(X), _ptr(W), _ptr(A), _ptr(B), float(scale), float(p_drop),
                                                 int(seed) & (2**64 - 1), _ptr(U_save), _ptr(dY), _ptr(dX),
                                                 _ptr(dA), _ptr(dB), T, d_in, d_out, r, _ptr(keep_bits),
                                                 _stream(stream)),
           "lora_linear_bwd_static")


def dropout_mask(seed: int, p_drop: float, mask, *, stream=None):
    T, d_in = mask.shape
    _args("lora_dropout_mask", ("mask", mask, (T, d_in), ("uint8",), False))
    _check(load_library().lora_dropout_mask(int(seed) & (2**64 - 1), float(p_drop), T, d_in, _ptr(mask),
                                            _stream(stream)), "lora_dropout_mask")


def dropout_keep_bits(seed: int, p_drop: float, bits, d_in: int, *, stream=None):
    """Write the dropout keep bits of a [T, d_in] input into `bits` (int32 device
    tensor [T, ceil(d_in / 32)]), for linear_fwd / linear_bwd's keep_bits."""
    T = bits.shape[0]
    _args("lora_dropout_keep_bits", ("bits", bits, (T, -(-d_in // 32)), _I32, False))
    _check(load_library().lora_dropout_keep_bits(int(seed) & (2**64 - 1), float(p_drop), T, d_in, _ptr(bits),
                                                 _stream(stream)), "lora_dropout_keep_bits")


def dropout_seed_for_rows(seed: int, t0: int, d_in: int) -> int:
    """lora_dropout_seed_for_rows: the seed that gives local rows 0.. the dropout
    mask of global rows t0.. (host only)."""
    return int(load_library().lora_dropout_seed_for_rows(int(seed) & (2**64 - 1), int(t0), int(d_in)))


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    v = ctypes.c_uint32(0)
    rc = load_library().lora_device_status(_stream(stream), ctypes.byref(v))
    if rc not in (LORA_OK, -5):
        raise LoraError(rc, "lora_device_status")
    return int(v.value)


def selftest_bounded_wait(limit_us: int, waited_ok, *, stream=None):
    """Run the bounded-wait self-test (see include/lora.h)."""
    _check(load_library().lora_selftest_bounded_wait(int(limit_us), _ptr(waited_ok), _stream(stream)),
           "lora_selftest_bounded_wait")


class Switch:
    """A fused adapter switch context for a stack of layers (lora_switch_create)."""

    def __init__(self, ranks, L: int, d_in: int, d_out: int, max_terms: int):
        self._ranks = _host_i32(ranks)
        self.L, self.d_in, self.d_out, self.max_terms = L, d_in, d_out, max_terms
        self.pool_rows = int(self._ranks.astype(np.int64).sum())
        h = _vp()
        _check(load_library().lora_switch_create(self._ranks.ctypes.data_as(_vp), self._ranks.shape[0], L, d_in, d_out,
                                                 max_terms, ctypes.byref(h)), "lora_switch_create")
        self._h = h

    def apply(self, W, A_pool, B_pool, term_adapters, term_coefs, *, stream=None):
        """W[l] += sum_j coef_j · A_a·B_a (a = term_adapters[j]) for every layer, in place."""
        L, di, do, R = self.L, self.d_in, self.d_out, self.pool_rows
        _args("lora_switch_apply", ("W", W, (L, di, do), _BF16, False), ("A_pool", A_pool, (L, R, di), _BF16, False),
              ("B_pool", B_pool, (L, R, do), _BF16, False))
        ta = _host_i32(term_adapters)
        tc = np.ascontiguousarray(term_coefs, dtype=np.float32)
        if ta.shape != tc.shape or ta.ndim != 1:
            raise LoraError(-1, "lora_switch_apply: term_adapters and term_coefs differ in shape")
        _check(load_library().lora_switch_apply(self._h, _ptr(W), _ptr(A_pool), _ptr(B_pool), ta.ctypes.data_as(_vp),
                                                tc.ctypes.data_as(_vp), ta.shape[0], _stream(stream)),
               "lora_switch_apply")

    def destroy(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load_library().lora_switch_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def tsqr_workspace_size(batch: int, m: int, n: int, want_q: bool) -> int:
    return int(load_library().lora_tsqr_workspace_size(int(batch), int(m), int(n), 1 if want_q else 0))


def tsqr(F, R, Q=None, workspace=None, *, stream=None):
    """lora_tsqr: A_b = Q_b·R_b for the matrices A_b[i, j] = F[b, j, i] (F bf16
    [batch, n, m], unit stride along m, any strides along b and j: e.g. one
    adapter's rows of a stack of pools, A_pool[:, off:off + r, :]). R fp32
    [batch, n, n]; Q fp32 [batch, n, m] (Q[b, j] is column j) or None. The
    workspace is allocated when not given."""
    if F is None or F.dim() != 3:
        raise LoraError(-1, "lora_tsqr: F must be a [batch, n, m] tensor")
    batch, n, m = (int(v) for v in F.shape)
    if str(F.dtype).rsplit(".", 1)[-1] not in _BF16 or F.stride(2) != 1:
        raise LoraError(-1, "lora_tsqr: F must be bfloat16 with unit stride along m")
    if not F.is_cuda:
        raise LoraError(-1, "lora_tsqr: F is not a CUDA tensor")
    _args("lora_tsqr", ("R", R, (batch, n, n), _F32, False), ("Q", Q, (batch, n, m), _F32, True))
    need = tsqr_workspace_size(batch, m, n, Q is not None)
    if workspace is None and need > 0:
        import torch
        workspace = torch.empty(need, dtype=torch.uint8, device=F.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    ptr = ctypes.c_void_p(F.data_ptr())
    _check(load_library().lora_tsqr(ptr, F.stride(1), F.stride(0), batch, m, n, _ptr(R), _ptr(Q), _ptr(workspace),
                                    nbytes, _stream(stream)), "lora_tsqr")


def _pool_rows(name, t):
    """A [n, r, d] bf16 view of module rows (unit stride along d, rows of d
    consecutive, any stride between modules)."""
    if t is None or t.dim() != 3 or str(t.dtype).rsplit(".", 1)[-1] not in _BF16 or t.stride(2) != 1 \
            or t.stride(1) != t.shape[2] or not t.is_cuda:
        raise LoraError(-1, f"{name}: a CUDA bfloat16 [n, r, d] tensor with rows of d consecutive is required")
    return int(t.shape[0]), int(t.shape[1]), int(t.shape[2])


class Compressor:
    """Post-hoc compression of a group of modules sharing d_in, d_out and r
    (lora_compress_spectra / lora_compress_export); the workspace holds the
    factorisation between the two calls."""

    def __init__(self, A_rows, B_rows, *, stream=None):
        import torch
        n, r, d_in = _pool_rows("A_rows", A_rows)
        n2, r2, d_out = _pool_rows("B_rows", B_rows)
        if (n2, r2) != (n, r):
            raise LoraError(-1, "lora_compress_spectra: A_rows and B_rows differ in modules or rank")
        self.n, self.r, self.d_in, self.d_out = n, r, d_in, d_out
        need = int(load_library().lora_compress_workspace_size(n, d_in, d_out, r))
        if need == 0:
            raise LoraError(-1, "lora_compress_spectra: sizes out of range")
        self.workspace = torch.empty(need, dtype=torch.uint8, device=A_rows.device)
        self.sigma = torch.empty(n, r, dtype=torch.float32, device=A_rows.device)
        _check(load_library().lora_compress_spectra(_ptr(A_rows), A_rows.stride(0), _ptr(B_rows), B_rows.stride(0), n,
                                                    d_in, d_out, r, _ptr(self.sigma), _ptr(self.workspace), need,
                                                    _stream(stream)), "lora_compress_spectra")

    def export(self, k, offsets, A_new, B_new, *, stream=None):
        """Write this group's truncated factors: k int32 [n], offsets int64 [n]
        (device; each module's first row), A_new bf16 [rows, d_in], B_new [rows, d_out]."""
        _args("lora_compress_export", ("k", k, (self.n,), _I32, False), ("offsets", offsets, (offsets.shape[0],),
                                                                         ("int64",), False),
              ("A_new", A_new, (A_new.shape[0], self.d_in), _BF16, False),
              ("B_new", B_new, (B_new.shape[0], self.d_out), _BF16, False))
        if offsets.shape[0] < self.n:
            raise LoraError(-1, "lora_compress_export: offsets has fewer entries than modules")
        _check(load_library().lora_compress_export(_ptr(self.sigma), _ptr(k), _ptr(offsets), self.n, self.d_in,
                                                   self.d_out, self.r, _ptr(A_new), _ptr(B_new),
                                                   _ptr(self.workspace), self.workspace.numel(), _stream(stream)),
               "lora_compress_export")


def compress_allocate(sigma, ranks, costs, policy: str, keep: float, k_floor: int, *, stream=None):
    """lora_compress_allocate: sigma fp32 [n, r_max], ranks int32 [n], costs int64 [n]
    (device). Returns (k int32 [n], offsets int64 [n + 1]) on the device."""
    import torch
    n, r_max = int(sigma.shape[0]), int(sigma.shape[1])
    _args("lora_compress_allocate", ("sigma", sigma, (n, r_max), _F32, False), ("ranks", ranks, (n,), _I32, False),
          ("costs", costs, (n,), ("int64",), False))
    k = torch.empty(n, dtype=torch.int32, device=sigma.device)
    off = torch.empty(n + 1, dtype=torch.int64, device=sigma.device)
    need = int(load_library().lora_compress_allocate_workspace_size(n, r_max))
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=sigma.device)
    pol = {"U": 0, "S": 1}[policy]
    _check(load_library().lora_compress_allocate(_ptr(sigma), _ptr(ranks), _ptr(costs), n, r_max, pol, float(keep),
                                                 int(k_floor), _ptr(k), _ptr(off), _ptr(ws), need, _stream(stream)),
           "lora_compress_allocate")
    return k, off
