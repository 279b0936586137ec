"""ctypes front end of the fp64 C oracle (``tpmlp_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline call this; the product path never does.

Every function takes numpy arrays (any float dtype; they are promoted to
float64, row-major) and returns float64 arrays. The formulas are stated in
``tpmlp_oracle.c``; they follow page "Megatron" (zzmblog.top), section
"张量并行 / 数学原理": column split Y = [X·A_1, …, X·A_p], row split
Z = Σ_i Y_i·B_i, with GeLU from the training script's ``activation_func``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tpmlp_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_tpmlp.so")
_lib = None
_lock = threading.Lock()

# -ffp-contract=off: no fused multiply-add contraction, so each sum is the
# plain sequence of double multiplies and adds the C source states.
CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``liboracle_tpmlp.so`` beside its source."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64
_P64 = ctypes.POINTER(ctypes.c_int64)


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.tpo_set_threads.argtypes = [ctypes.c_int]
    lib.tpo_get_threads.restype = ctypes.c_int
    for name in ("tpo_normal_cdf", "tpo_normal_pdf", "tpo_gelu", "tpo_gelu_grad", "tpo_gelu_tanh",
                 "tpo_gelu_tanh_grad"):
        fn = getattr(lib, name)
        fn.argtypes = [ctypes.c_double]
        fn.restype = ctypes.c_double
    lib.tpo_colsum.argtypes = [_I64, _I64, _D, _D]
    _c = ctypes.c_int
    lib.tpo_forward_act.argtypes = [_I64, _I64, _I64] + [_D] * 8 + [_c]
    lib.tpo_backward_act.argtypes = [_I64, _I64, _I64] + [_D] * 12 + [_c]
    lib.tpo_forward_sharded_act.argtypes = [_I64, _I64, _I64, _c] + [_D] * 8 + [_c]
    lib.tpo_forward_sharded_act.restype = _c
    lib.tpo_backward_sharded_act.argtypes = [_I64, _I64, _I64, _c] + [_D] * 12 + [_c]
    lib.tpo_backward_sharded_act.restype = _c
    lib.tpo_rows_act.argtypes = [_I64, _I64, _I64] + [_D] * 6 + [_I64, _P64] + [_D] * 5 + [_c]
    lib.tpo_cols_act.argtypes = [_I64, _I64, _I64] + [_D] * 5 + [_I64, _P64] + [_D] * 6 + [_c]
    lib.tpo_linear_forward.argtypes = [_I64, _I64, _I64] + [_D] * 4
    lib.tpo_linear_backward.argtypes = [_I64, _I64, _I64] + [_D] * 6
    lib.tpo_linear_forward_sharded.argtypes = [_I64, _I64, _I64, _c, _c] + [_D] * 4
    lib.tpo_linear_forward_sharded.restype = _c
    lib.tpo_linear_backward_sharded.argtypes = [_I64, _I64, _I64, _c, _c] + [_D] * 6
    lib.tpo_linear_backward_sharded.restype = _c
    return lib


def _in(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x: np.ndarray):
    return x.ctypes.data_as(_D)


class Oracle:
    """The oracle's functions bound to one build of ``tpmlp_oracle.c``."""

    def __init__(self, path: str):
        self.path = path
        self._lib = _bind(path)

    def set_threads(self, n: int) -> None:
        self._lib.tpo_set_threads(int(n))

    def get_threads(self) -> int:
        return int(self._lib.tpo_get_threads())

    def normal_cdf(self, x: float) -> float:
        return float(self._lib.tpo_normal_cdf(float(x)))

    def normal_pdf(self, x: float) -> float:
        return float(self._lib.tpo_normal_pdf(float(x)))

    def gelu(self, x: float) -> float:
        return float(self._lib.tpo_gelu(float(x)))

    def gelu_grad(self, x: float) -> float:
        return float(self._lib.tpo_gelu_grad(float(x)))

    def gelu_tanh(self, x: float) -> float:
        return float(self._lib.tpo_gelu_tanh(float(x)))

    def gelu_tanh_grad(self, x: float) -> float:
        return float(self._lib.tpo_gelu_tanh_grad(float(x)))

    def colsum(self, M) -> np.ndarray:
        M = _in(M)
        T, N = M.shape
        out = np.empty(N)
        self._lib.tpo_colsum(T, N, _ptr(M), _ptr(out))
        return out

    def forward(self, X, A, a, B, b, act: int = 0):
        """Unsplit forward. Returns (H, Y, Z) in float64. act: 0 = exact GeLU,
        1 = tanh approximation."""
        X, A, a, B, b = map(_in, (X, A, a, B, b))
        T, h = X.shape
        F = A.shape[1]
        assert A.shape == (h, F) and a.shape == (F,) and B.shape == (F, h) and b.shape == (h,)
        H, Y, Z = np.empty((T, F)), np.empty((T, F)), np.empty((T, h))
        self._lib.tpo_forward_act(T, h, F, *map(_ptr, (X, A, a, B, b, H, Y, Z)), int(act))
        return H, Y, Z

    @staticmethod
    def _grads(T, h, F):
        return dict(dH=np.empty((T, F)), dX=np.empty((T, h)), dA=np.empty((h, F)),
                    da=np.empty(F), dB=np.empty((F, h)), db=np.empty(h))

    def backward(self, X, A, B, H, Y, dZ, act: int = 0):
        """Unsplit backward. Returns dict with dH, dX, dA, da, dB, db (float64)."""
        X, A, B, H, Y, dZ = map(_in, (X, A, B, H, Y, dZ))
        T, h = X.shape
        F = A.shape[1]
        out = self._grads(T, h, F)
        self._lib.tpo_backward_act(T, h, F, *map(_ptr, (X, A, B, H, Y, dZ)),
                                   *map(_ptr, (out[k] for k in ("dH", "dX", "dA", "da", "dB", "db"))),
                                   int(act))
        return out

    def forward_sharded(self, X, A, a, B, b, p: int, act: int = 0):
        """Forward through the p-way column/row partition. Returns (H, Y, Z)."""
        X, A, a, B, b = map(_in, (X, A, a, B, b))
        T, h = X.shape
        F = A.shape[1]
        H, Y, Z = np.empty((T, F)), np.empty((T, F)), np.empty((T, h))
        rc = self._lib.tpo_forward_sharded_act(T, h, F, int(p), *map(_ptr, (X, A, a, B, b, H, Y, Z)),
                                               int(act))
        if rc != 0:
            raise ValueError(f"p={p} does not divide F={F}")
        return H, Y, Z

    def backward_sharded(self, X, A, B, H, Y, dZ, p: int, act: int = 0):
        """Backward through the p-way partition (dX summed over shards in order)."""
        X, A, B, H, Y, dZ = map(_in, (X, A, B, H, Y, dZ))
        T, h = X.shape
        F = A.shape[1]
        out = self._grads(T, h, F)
        rc = self._lib.tpo_backward_sharded_act(
            T, h, F, int(p), *map(_ptr, (X, A, B, H, Y, dZ)),
            *map(_ptr, (out[k] for k in ("dH", "dX", "dA", "da", "dB", "db"))), int(act))
        if rc != 0:
            raise ValueError(f"p={p} does not divide F={F}")
        return out

    def rows(self, X, A, a, B, b, dZ, R, act: int = 0):
        """Outputs restricted to token rows R: dict with H, Y, Z, dH, dX."""
        X, A, a, B, b, dZ = map(_in, (X, A, a, B, b, dZ))
        R = np.ascontiguousarray(np.asarray(R, dtype=np.int64))
        T, h = X.shape
        F = A.shape[1]
        assert R.min() >= 0 and R.max() < T
        n = len(R)
        out = dict(H=np.empty((n, F)), Y=np.empty((n, F)), Z=np.empty((n, h)),
                   dH=np.empty((n, F)), dX=np.empty((n, h)))
        self._lib.tpo_rows_act(T, h, F, *map(_ptr, (X, A, a, B, b, dZ)), n, R.ctypes.data_as(_P64),
                               *map(_ptr, (out[k] for k in ("H", "Y", "Z", "dH", "dX"))), int(act))
        return out

    def cols(self, X, A, a, B, dZ, J, act: int = 0):
        """Outputs restricted to hidden columns J: dict with H, Y, dH (T × |J|),
        dA (h × |J|), da (|J|), dB (|J| × h)."""
        X, A, a, B, dZ = map(_in, (X, A, a, B, dZ))
        J = np.ascontiguousarray(np.asarray(J, dtype=np.int64))
        T, h = X.shape
        F = A.shape[1]
        assert J.min() >= 0 and J.max() < F
        n = len(J)
        out = dict(H=np.empty((T, n)), Y=np.empty((T, n)), dH=np.empty((T, n)),
                   dA=np.empty((h, n)), da=np.empty(n), dB=np.empty((n, h)))
        self._lib.tpo_cols_act(T, h, F, *map(_ptr, (X, A, a, B, dZ)), n, J.ctypes.data_as(_P64),
                               *map(_ptr, (out[k] for k in ("H", "Y", "dH", "dA", "da", "dB"))),
                               int(act))
        return out


    # ------------------------------------------------ tensor-parallel linear
    def linear_forward(self, X, W, bias):
        """Y = X·W + bias (unsplit). X: T×K, W: K×N, bias: N."""
        X, W, bias = map(_in, (X, W, bias))
        T, K = X.shape
        N = W.shape[1]
        assert W.shape == (K, N) and bias.shape == (N,)
        Y = np.empty((T, N))
        self._lib.tpo_linear_forward(T, K, N, *map(_ptr, (X, W, bias, Y)))
        return Y

    def linear_backward(self, X, W, dY):
        """(dX, dW, dbias) of Y = X·W + bias (unsplit)."""
        X, W, dY = map(_in, (X, W, dY))
        T, K = X.shape
        N = W.shape[1]
        dX, dW, db = np.empty((T, K)), np.empty((K, N)), np.empty(N)
        self._lib.tpo_linear_backward(T, K, N, *map(_ptr, (X, W, dY, dX, dW, db)))
        return dX, dW, db

    def linear_forward_sharded(self, X, W, bias, p: int, split: str):
        """Y through the p-way partition; split = "columns" or "rows"."""
        X, W, bias = map(_in, (X, W, bias))
        T, K = X.shape
        N = W.shape[1]
        Y = np.empty((T, N))
        rc = self._lib.tpo_linear_forward_sharded(T, K, N, int(p), {"columns": 0, "rows": 1}[split],
                                                  *map(_ptr, (X, W, bias, Y)))
        if rc != 0:
            raise ValueError(f"p={p} does not divide the {split} dimension")
        return Y

    def linear_backward_sharded(self, X, W, dY, p: int, split: str):
        X, W, dY = map(_in, (X, W, dY))
        T, K = X.shape
        N = W.shape[1]
        dX, dW, db = np.empty((T, K)), np.empty((K, N)), np.empty(N)
        rc = self._lib.tpo_linear_backward_sharded(T, K, N, int(p),
                                                   {"columns": 0, "rows": 1}[split],
                                                   *map(_ptr, (X, W, dY, dX, dW, db)))
        if rc != 0:
            raise ValueError(f"p={p} does not divide the {split} dimension")
        return dX, dW, db


def compile_variant(source_text: str, out_path: str) -> Oracle:
    """Compile a (possibly edited) copy of the oracle source and bind it.
    Used by the tests to plant mistakes in a throw-away build and check that
    the pins catch them; the committed source is never changed."""
    src_path = out_path + ".c"
    with open(src_path, "w") as f:
        f.write(source_text)
    subprocess.check_call(["gcc", *CFLAGS, "-o", out_path, src_path, "-lm"])
    return Oracle(out_path)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def default() -> Oracle:
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def set_threads(n: int) -> None:
    default().set_threads(n)


def get_threads() -> int:
    return default().get_threads()


def normal_cdf(x):
    return default().normal_cdf(x)


def normal_pdf(x):
    return default().normal_pdf(x)


def gelu(x):
    return default().gelu(x)


def gelu_grad(x):
    return default().gelu_grad(x)


def colsum(M):
    return default().colsum(M)


def gelu_tanh(x):
    return default().gelu_tanh(x)


def gelu_tanh_grad(x):
    return default().gelu_tanh_grad(x)


def forward(X, A, a, B, b, act=0):
    return default().forward(X, A, a, B, b, act)


def backward(X, A, B, H, Y, dZ, act=0):
    return default().backward(X, A, B, H, Y, dZ, act)


def forward_sharded(X, A, a, B, b, p, act=0):
    return default().forward_sharded(X, A, a, B, b, p, act)


def backward_sharded(X, A, B, H, Y, dZ, p, act=0):
    return default().backward_sharded(X, A, B, H, Y, dZ, p, act)


def rows(X, A, a, B, b, dZ, R, act=0):
    return default().rows(X, A, a, B, b, dZ, R, act)


def cols(X, A, a, B, dZ, J, act=0):
    return default().cols(X, A, a, B, dZ, J, act)


def linear_forward(X, W, bias):
    return default().linear_forward(X, W, bias)


def linear_backward(X, W, dY):
    return default().linear_backward(X, W, dY)


def linear_forward_sharded(X, W, bias, p, split):
    return default().linear_forward_sharded(X, W, bias, p, split)


def linear_backward_sharded(X, W, dY, p, split):
    return default().linear_backward_sharded(X, W, dY, p, split)
