"""Python binding of ``libtpmlp.so`` (ctypes). Argument marshalling only.

Every step of the block runs in the library's CUDA kernels; torch supplies
device memory (the output and workspace tensors) and the current stream.
There is no other implementation behind these functions: if the library is
missing or the tensors are not on a CUDA device, they raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from .build import LIB as _LIB_PATH

OK, ERR_INVALID, ERR_ALIGN, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(7)
BF16, FP32 = 0, 1
ACTIVATIONS = {"gelu": 0, "gelu_tanh": 1}

# The entry points include/tpmlp.h declares, in declaration order.
EXPORTS = (
    "tpmlp_workspace_size", "tp_mlp_fwd", "tp_mlp_bwd", "tp_mlp_fwd_ex", "tp_mlp_bwd_ex",
    "tpmlp_linear_workspace_size", "tp_linear_fwd", "tp_linear_bwd",
    "tp_mlp_recompute_activation", "tp_mlp_recompute_hidden", "tpmlp_strerror",
    "tpmlp_last_device_status", "tpmlp_set_split_policy", "tpmlp_get_split_policy",
    "tpmlp_set_launch_overlap", "tpmlp_get_launch_overlap", "tpmlp_set_dynamic_schedule",
    "tpmlp_get_dynamic_schedule",
    "tpmlp_set_wait_limit_ns", "tpmlp_wait_selftest", "tpmlp_launch_count", "tpmlp_eval_activation",
    "tpmlp_profile_enable", "tpmlp_profile_collect", "tpmlp_profile_kinds", "tpmlp_profile_name",
    "tpmlp_profile_read", "tpmlp_profile_reset", "tp_mlp_bwd_noalloc",
    "tpmlp_noalloc_scratch_bytes", "tpmlp_schedule_units", "tpmlp_plan_schedules", "tpmlp_plan_dynamic",
    "tpmlp_version",
)

_lib = None
_lock = threading.Lock()


class TPMLPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {strerror(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libtpmlp.so (once). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"CUDA library {_LIB_PATH} is missing; build it with "
                    "`python -m tensor_transformer_mlp_block_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
            L.tpmlp_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int]
            L.tpmlp_workspace_size.restype = sz
            ci = ctypes.c_int
            L.tpmlp_schedule_units.argtypes = [ci, ci, ci, ci, ci, ci, ctypes.POINTER(i64), i64]
            L.tpmlp_schedule_units.restype = i64
            L.tpmlp_plan_schedules.argtypes = [i64, i64, i64, ci, ci, ctypes.POINTER(ci)]
            L.tpmlp_plan_schedules.restype = ci
            L.tpmlp_plan_dynamic.argtypes = [i64, i64, i64, ci, ci, ctypes.POINTER(ci)]
            L.tpmlp_plan_dynamic.restype = ci
            L.tp_mlp_fwd.argtypes = [vp] * 8 + [i64, i64, i64, ctypes.c_int, ctypes.c_int, vp, sz, vp]
            L.tp_mlp_fwd.restype = ctypes.c_int
            L.tp_mlp_bwd.argtypes = [vp] * 12 + [i64, i64, i64, ctypes.c_int, ctypes.c_int, vp, sz, vp]
            L.tp_mlp_bwd.restype = ctypes.c_int
            L.tp_mlp_fwd_ex.argtypes = [vp] * 8 + [i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, vp, sz, vp]
            L.tp_mlp_fwd_ex.restype = ctypes.c_int
            L.tp_mlp_bwd_ex.argtypes = [vp] * 12 + [i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, vp, sz, vp]
            L.tp_mlp_bwd_ex.restype = ctypes.c_int
            L.tpmlp_linear_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int]
            L.tpmlp_linear_workspace_size.restype = sz
            L.tp_linear_fwd.argtypes = [vp] * 4 + [i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, vp, sz, vp]
            L.tp_linear_fwd.restype = ctypes.c_int
            L.tp_linear_bwd.argtypes = [vp] * 6 + [i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, vp, sz, vp]
            L.tp_linear_bwd.restype = ctypes.c_int
            L.tp_mlp_recompute_activation.argtypes = [vp, vp, i64, ctypes.c_int, ctypes.c_int, vp]
            L.tp_mlp_recompute_activation.restype = ctypes.c_int
            L.tp_mlp_recompute_hidden.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, vp]
            L.tp_mlp_recompute_hidden.restype = ctypes.c_int
            L.tpmlp_strerror.argtypes = [ctypes.c_int]
            L.tpmlp_strerror.restype = ctypes.c_char_p
            L.tpmlp_last_device_status.argtypes = [vp]
            L.tpmlp_last_device_status.restype = ctypes.c_int
            L.tpmlp_set_split_policy.argtypes = [ctypes.c_int]
            L.tpmlp_set_split_policy.restype = ctypes.c_int
            L.tpmlp_get_split_policy.restype = ctypes.c_int
            L.tpmlp_set_launch_overlap.argtypes = [ctypes.c_int]
            L.tpmlp_set_launch_overlap.restype = None
            L.tpmlp_get_launch_overlap.restype = ctypes.c_int
            L.tpmlp_set_dynamic_schedule.argtypes = [ctypes.c_int]
            L.tpmlp_set_dynamic_schedule.restype = None
            L.tpmlp_get_dynamic_schedule.restype = ctypes.c_int
            L.tpmlp_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.tpmlp_set_wait_limit_ns.restype = None
            L.tpmlp_wait_selftest.argtypes = [ctypes.c_uint64, vp]
            L.tpmlp_wait_selftest.restype = ctypes.c_int
            L.tpmlp_launch_count.restype = ctypes.c_uint64
            L.tpmlp_eval_activation.argtypes = [vp, vp, vp, i64, ctypes.c_int, vp]
            L.tpmlp_eval_activation.restype = ctypes.c_int
            L.tpmlp_version.restype = ctypes.c_int
            L.tpmlp_profile_enable.argtypes = [ctypes.c_int]
            L.tpmlp_profile_enable.restype = None
            L.tpmlp_profile_collect.restype = ctypes.c_int
            L.tpmlp_profile_kinds.restype = ctypes.c_int
            L.tpmlp_profile_name.argtypes = [ctypes.c_int]
            L.tpmlp_profile_name.restype = ctypes.c_char_p
            L.tpmlp_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint64)] + \
                [ctypes.POINTER(ctypes.c_double)] * 3
            L.tpmlp_profile_read.restype = ctypes.c_int
            L.tpmlp_profile_reset.restype = None
            L.tp_mlp_bwd_noalloc.argtypes = [vp] * 12 + [i64, i64, i64, ctypes.c_int, ctypes.c_int, vp]
            L.tp_mlp_bwd_noalloc.restype = ctypes.c_int
            L.tpmlp_noalloc_scratch_bytes.restype = sz
            _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().tpmlp_strerror(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise TPMLPError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _stream_ptr(device: torch.device, stream) -> int:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, shape, dtype, device) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def workspace_size(T: int, h: int, F: int, p: int, dtype: torch.dtype = torch.bfloat16) -> int:
    code = BF16 if dtype == torch.bfloat16 else FP32
    return int(lib().tpmlp_workspace_size(T, h, F, p, code))


def _workspace(T, h, F, p, dtype, device, workspace):
    n = workspace_size(T, h, F, p, dtype)
    if workspace is None:
        return torch.empty(max(n, 1), dtype=torch.uint8, device=device), n
    if workspace.numel() * workspace.element_size() < n:
        raise ValueError(f"workspace has {workspace.nbytes} bytes, needs {n}")
    return workspace, workspace.numel() * workspace.element_size()


def _act_code(activation: str) -> int:
    try:
        return ACTIVATIONS[activation]
    except KeyError:
        raise ValueError(f"activation must be one of {sorted(ACTIVATIONS)}") from None


def forward(X, A, a, B, b, p: int, *, out=None, workspace=None, stream=None,
            activation: str = "gelu"):
    """H, Y, Z of Z = GeLU(X·A + a)·B + b with A, B split into p shards.

    X: T×h, A: h×F, a: F or None, B: F×h, b: h or None, all bf16 (or all
    fp32) CUDA tensors. Returns (H, Y, Z); `out` may supply them.
    activation: "gelu" (exact, x·Φ(x)) or "gelu_tanh" (tanh approximation)."""
    T, h = X.shape
    F = A.shape[1]
    dt, dev = X.dtype, X.device
    _need(X, "X", (T, h), dt, dev)
    _need(A, "A", (h, F), dt, dev)
    _need(B, "B", (F, h), dt, dev)
    if a is not None:
        _need(a, "a", (F,), dt, dev)
    if b is not None:
        _need(b, "b", (h,), dt, dev)
    if out is None:
        H = torch.empty((T, F), dtype=dt, device=dev)
        Y = torch.empty((T, F), dtype=dt, device=dev)
        Z = torch.empty((T, h), dtype=dt, device=dev)
    else:
        H, Y, Z = out
        _need(H, "H", (T, F), dt, dev)
        _need(Y, "Y", (T, F), dt, dev)
        _need(Z, "Z", (T, h), dt, dev)
    with torch.cuda.device(dev):
        ws, ws_bytes = _workspace(T, h, F, p, dt, dev, workspace)
        st = lib().tp_mlp_fwd_ex(_ptr(X), _ptr(A), _ptr(a), _ptr(B), _ptr(b), _ptr(H), _ptr(Y),
                                 _ptr(Z), T, h, F, int(p), _dtype_code(X), _act_code(activation),
                                 _ptr(ws), ws_bytes, _stream_ptr(dev, stream))
    _check(st, "tp_mlp_fwd_ex")
    return H, Y, Z


def backward(dZ, X, A, B, H, Y, p: int, *, out=None, workspace=None, stream=None,
             activation: str = "gelu"):
    """Gradients of the block for upstream gradient dZ (T×h); `activation`
    must be the forward's.

    Returns a dict: dX (T×h, input dtype), dA (h×F, fp32), da (F, fp32),
    dB (F×h, fp32), db (h, fp32), dH (T×F, input dtype)."""
    T, h = X.shape
    F = A.shape[1]
    dt, dev = X.dtype, X.device
    for name, t, shp in (("dZ", dZ, (T, h)), ("X", X, (T, h)), ("A", A, (h, F)), ("B", B, (F, h)),
                         ("H", H, (T, F)), ("Y", Y, (T, F))):
        _need(t, name, shp, dt, dev)
    f32 = torch.float32
    if out is None:
        out = dict(dX=torch.empty((T, h), dtype=dt, device=dev),
                   dA=torch.empty((h, F), dtype=f32, device=dev),
                   da=torch.empty((F,), dtype=f32, device=dev),
                   dB=torch.empty((F, h), dtype=f32, device=dev),
                   db=torch.empty((h,), dtype=f32, device=dev),
                   dH=torch.empty((T, F), dtype=dt, device=dev))
    for name, shp, d in (("dX", (T, h), dt), ("dA", (h, F), f32), ("da", (F,), f32),
                         ("dB", (F, h), f32), ("db", (h,), f32), ("dH", (T, F), dt)):
        _need(out[name], name, shp, d, dev)
    with torch.cuda.device(dev):
        ws, ws_bytes = _workspace(T, h, F, p, dt, dev, workspace)
        st = lib().tp_mlp_bwd_ex(_ptr(dZ), _ptr(X), _ptr(A), _ptr(B), _ptr(H), _ptr(Y),
                                 _ptr(out["dX"]), _ptr(out["dA"]), _ptr(out["da"]),
                                 _ptr(out["dB"]), _ptr(out["db"]), _ptr(out["dH"]), T, h, F,
                                 int(p), _dtype_code(X), _act_code(activation), _ptr(ws), ws_bytes,
                                 _stream_ptr(dev, stream))
    _check(st, "tp_mlp_bwd_ex")
    return out


def set_split_policy(policy: int) -> None:
    _check(lib().tpmlp_set_split_policy(int(policy)), "tpmlp_set_split_policy")


def get_split_policy() -> int:
    return int(lib().tpmlp_get_split_policy())


def set_dynamic_schedule(on: bool) -> None:
    lib().tpmlp_set_dynamic_schedule(1 if on else 0)


def get_dynamic_schedule() -> bool:
    return bool(lib().tpmlp_get_dynamic_schedule())


def set_launch_overlap(on: bool) -> None:
    """Programmatic dependent launches between the library's kernels (default on)."""
    lib().tpmlp_set_launch_overlap(1 if on else 0)


def get_launch_overlap() -> bool:
    return bool(lib().tpmlp_get_launch_overlap())


def set_wait_limit_ns(ns: int) -> None:
    lib().tpmlp_set_wait_limit_ns(int(ns))


def last_device_status(stream=None, device=None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib().tpmlp_last_device_status(_stream_ptr(dev, stream)))


def wait_selftest(limit_ns: int, stream=None) -> None:
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib().tpmlp_wait_selftest(int(limit_ns), _stream_ptr(dev, stream)), "tpmlp_wait_selftest")


def launch_count() -> int:
    return int(lib().tpmlp_launch_count())


def version() -> int:
    return int(lib().tpmlp_version())


def profile_enable(on: bool = True) -> None:
    """Bracket every library launch with CUDA events on its stream."""
    lib().tpmlp_profile_enable(1 if on else 0)


def profile_reset() -> None:
    lib().tpmlp_profile_reset()


def profile_collect() -> dict:
    """Wait for the recorded events; return {kind: dict(launches, ms, flops,
    bytes)} accumulated since the last reset (kinds with launches only)."""
    L = lib()
    n = L.tpmlp_profile_collect()
    if n < 0:
        raise TPMLPError(ERR_CUDA, "tpmlp_profile_collect")
    out = {}
    for k in range(L.tpmlp_profile_kinds()):
        cnt = ctypes.c_uint64()
        ms, fl, by = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
        _check(L.tpmlp_profile_read(k, ctypes.byref(cnt), ctypes.byref(ms), ctypes.byref(fl),
                                    ctypes.byref(by)), "tpmlp_profile_read")
        if cnt.value:
            out[L.tpmlp_profile_name(k).decode()] = dict(launches=int(cnt.value), ms=ms.value,
                                                         flops=fl.value, bytes=by.value)
    return out


def eval_activation(x: torch.Tensor, form: int):
    """(GeLU(x), GeLU′(x)) of a CUDA fp32 tensor with one of the kernels'
    forms: 0 exact GeLU as the tensor-core epilogues compute it (Hastings
    erf), 1 exact GeLU through CUDA's erff, 2 tanh form as the tensor-core
    epilogues compute it, 3 tanh form through CUDA's tanhf."""
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    dy = torch.empty_like(x)
    with torch.cuda.device(x.device):
        _check(lib().tpmlp_eval_activation(x.data_ptr(), y.data_ptr(), dy.data_ptr(), x.numel(),
                                           int(form), _stream_ptr(x.device, None)),
               "tpmlp_eval_activation")
    return y, dy


SPLITS = {"columns": 0, "rows": 1}


def _split_code(split: str) -> int:
    try:
        return SPLITS[split]
    except KeyError:
        raise ValueError(f"split must be one of {sorted(SPLITS)}") from None


def linear_workspace_size(T: int, K: int, N: int, p: int, split: str,
                          dtype: torch.dtype = torch.bfloat16) -> int:
    code = BF16 if dtype == torch.bfloat16 else FP32
    return int(lib().tpmlp_linear_workspace_size(T, K, N, p, _split_code(split), code))


def linear_forward(X, W, bias, p: int, split: str, *, out=None, workspace=None, stream=None):
    """Y = X·W + bias with W split into p shards by "columns" (QKV-style) or
    "rows" (output-projection style). X: T×K, W: K×N, bias: N or None."""
    T, K = X.shape
    N = W.shape[1]
    dt, dev = X.dtype, X.device
    _need(X, "X", (T, K), dt, dev)
    _need(W, "W", (K, N), dt, dev)
    if bias is not None:
        _need(bias, "bias", (N,), dt, dev)
    Y = torch.empty((T, N), dtype=dt, device=dev) if out is None else out
    _need(Y, "Y", (T, N), dt, dev)
    with torch.cuda.device(dev):
        n = linear_workspace_size(T, K, N, p, split, dt)
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev) if workspace is None else workspace
        st = lib().tp_linear_fwd(_ptr(X), _ptr(W), _ptr(bias), _ptr(Y), T, K, N, int(p),
                                 _split_code(split), _dtype_code(X), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream_ptr(dev, stream))
    _check(st, "tp_linear_fwd")
    return Y


def linear_backward(dY, X, W, p: int, split: str, *, out=None, workspace=None, stream=None):
    """(dX, dW, dbias) of linear_forward for upstream dY (T×N); dW and dbias fp32."""
    T, K = X.shape
    N = W.shape[1]
    dt, dev = X.dtype, X.device
    for name, t, shp in (("dY", dY, (T, N)), ("X", X, (T, K)), ("W", W, (K, N))):
        _need(t, name, shp, dt, dev)
    if out is None:
        out = (torch.empty((T, K), dtype=dt, device=dev),
               torch.empty((K, N), dtype=torch.float32, device=dev),
               torch.empty((N,), dtype=torch.float32, device=dev))
    dX, dW, db = out
    _need(dX, "dX", (T, K), dt, dev)
    _need(dW, "dW", (K, N), torch.float32, dev)
    _need(db, "dbias", (N,), torch.float32, dev)
    with torch.cuda.device(dev):
        n = linear_workspace_size(T, K, N, p, split, dt)
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev) if workspace is None else workspace
        st = lib().tp_linear_bwd(_ptr(dY), _ptr(X), _ptr(W), _ptr(dX), _ptr(dW), _ptr(db), T, K,
                                 N, int(p), _split_code(split), _dtype_code(X), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream_ptr(dev, stream))
    _check(st, "tp_linear_bwd")
    return dX, dW, db


def recompute_hidden(X, A, a, p: int, *, out=None, activation: str = "gelu", stream=None):
    """H = X·A + a and Y = act(H) (the forward's first product alone), for
    a caller that keeps only X. Returns (H, Y); `out` may supply them."""
    T, h = X.shape
    F = A.shape[1]
    dt, dev = X.dtype, X.device
    _need(X, "X", (T, h), dt, dev)
    _need(A, "A", (h, F), dt, dev)
    if a is not None:
        _need(a, "a", (F,), dt, dev)
    if out is None:
        H = torch.empty((T, F), dtype=dt, device=dev)
        Y = torch.empty((T, F), dtype=dt, device=dev)
    else:
        H, Y = out
        _need(H, "H", (T, F), dt, dev)
        _need(Y, "Y", (T, F), dt, dev)
    with torch.cuda.device(dev):
        _check(lib().tp_mlp_recompute_hidden(_ptr(X), _ptr(A), _ptr(a), _ptr(H), _ptr(Y), T, h, F,
                                             int(p), _dtype_code(X), _act_code(activation),
                                             _stream_ptr(dev, stream)),
               "tp_mlp_recompute_hidden")
    return H, Y


def recompute_activation(H, *, out=None, activation: str = "gelu", stream=None):
    """Y = act(H) elementwise (activation recompute before the backward)."""
    if not H.is_cuda or not H.is_contiguous():
        raise ValueError("H must be a contiguous CUDA tensor")
    Y = torch.empty_like(H) if out is None else out
    _need(Y, "Y", tuple(H.shape), H.dtype, H.device)
    with torch.cuda.device(H.device):
        _check(lib().tp_mlp_recompute_activation(_ptr(H), _ptr(Y), H.numel(), _dtype_code(H),
                                                 _act_code(activation),
                                                 _stream_ptr(H.device, stream)),
               "tp_mlp_recompute_activation")
    return Y


# Work-unit schedules of the tensor-core products (tpmlp_schedule_units).
SCHED_TILES, SCHED_GROUPS, SCHED_STREAMK = 0, 1, 2
SCHEDULE_FIELDS = ("worker", "local", "mb", "nb", "kb0", "kb1", "pieces", "piece", "key", "slot")


def schedule_units(sched: int, m_blocks: int, n_blocks: int, k_blocks: int, workers: int,
                   groups: int = 1):
    """The units the GEMM kernels run for this tile grid (host only), as a
    list of dicts with SCHEDULE_FIELDS; None if the kernels would not run
    this schedule."""
    L = lib()
    n = int(L.tpmlp_schedule_units(sched, m_blocks, n_blocks, k_blocks, groups, workers, None, 0))
    if n < 0:
        return None
    buf = (ctypes.c_int64 * (10 * max(n, 1)))()
    got = int(L.tpmlp_schedule_units(sched, m_blocks, n_blocks, k_blocks, groups, workers, buf, n))
    assert got == n
    return [dict(zip(SCHEDULE_FIELDS, buf[10 * i:10 * i + 10])) for i in range(n)]


def plan_schedules(T: int, h: int, F: int, p: int, dtype: torch.dtype = torch.bfloat16):
    """The schedule planned for F1, F2, B2, B3, B4, B5 at these sizes under
    the current split policy (host only)."""
    kinds = (ctypes.c_int * 6)()
    code = BF16 if dtype == torch.bfloat16 else FP32
    _check(lib().tpmlp_plan_schedules(T, h, F, p, code, kinds), "tpmlp_plan_schedules")
    return dict(zip(("F1", "F2", "B2", "B3", "B4", "B5"), list(kinds)))


def plan_dynamic(T: int, h: int, F: int, p: int, dtype: torch.dtype = torch.bfloat16):
    """Which of F1, F2, B2, B3, B4, B5 run the dynamic tile schedule at these
    sizes under the current settings (host only)."""
    dyn = (ctypes.c_int * 6)()
    code = BF16 if dtype == torch.bfloat16 else FP32
    _check(lib().tpmlp_plan_dynamic(T, h, F, p, code, dyn), "tpmlp_plan_dynamic")
    return dict(zip(("F1", "F2", "B2", "B3", "B4", "B5"), [bool(x) for x in dyn]))
