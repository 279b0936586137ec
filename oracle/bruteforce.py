"""Pure-Python brute-force evaluation of the MLP block, for tiny shapes only.

TEST INFRASTRUCTURE ONLY. It shares nothing with the C oracle: each entry is
an explicit dot product summed with ``math.fsum`` (correctly rounded sum) and
GeLU uses ``math.erf``. It exists to pin the C oracle on shapes up to about
T = 8, h = 6, F = 24.

Definitions (page "Megatron", zzmblog.top, section "张量并行 / 数学原理";
activation "gelu" from the training script's TransformerConfig):
H = X·A + a, Y = GeLU(H), Z = Y·B + b; the gradients follow the chain rule.
"""
from __future__ import annotations

import math


def _phi_cdf(x: float) -> float:
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def _gelu(x: float) -> float:
    return x * _phi_cdf(x)


def _gelu_grad(x: float) -> float:
    return _phi_cdf(x) + x * math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _gelu_tanh(x: float) -> float:
    return 0.5 * x * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def _gelu_tanh_grad(x: float) -> float:
    u = math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)
    du = math.sqrt(2.0 / math.pi) * (1.0 + 3 * 0.044715 * x * x)
    return 0.5 * (1.0 + math.tanh(u)) + 0.5 * x * (1.0 - math.tanh(u) ** 2) * du


def mlp(X, A, a, B, b, dZ, act: int = 0):
    """X: T×h, A: h×F, a: F, B: F×h, b: h, dZ: T×h, as nested lists of floats.
    act: 0 = exact GeLU, 1 = tanh approximation.

    Returns a dict of nested lists: H, Y, Z, dH, dX, dA, da, dB, db.
    """
    g, dg = (_gelu_tanh, _gelu_tanh_grad) if act else (_gelu, _gelu_grad)
    T, h, F = len(X), len(X[0]), len(A[0])
    H = [[math.fsum([X[t][k] * A[k][f] for k in range(h)] + [a[f]]) for f in range(F)]
         for t in range(T)]
    Y = [[g(H[t][f]) for f in range(F)] for t in range(T)]
    Z = [[math.fsum([Y[t][f] * B[f][j] for f in range(F)] + [b[j]]) for j in range(h)]
         for t in range(T)]
    db = [math.fsum(dZ[t][j] for t in range(T)) for j in range(h)]
    dB = [[math.fsum(Y[t][f] * dZ[t][j] for t in range(T)) for j in range(h)] for f in range(F)]
    dY = [[math.fsum(dZ[t][j] * B[f][j] for j in range(h)) for f in range(F)] for t in range(T)]
    dH = [[dY[t][f] * dg(H[t][f]) for f in range(F)] for t in range(T)]
    da = [math.fsum(dH[t][f] for t in range(T)) for f in range(F)]
    dA = [[math.fsum(X[t][k] * dH[t][f] for t in range(T)) for f in range(F)] for k in range(h)]
    dX = [[math.fsum(dH[t][f] * A[k][f] for f in range(F)) for k in range(h)] for t in range(T)]
    return dict(H=H, Y=Y, Z=Z, dH=dH, dX=dX, dA=dA, da=da, dB=dB, db=db)


def linear(X, W, bias, dY):
    """Y = X·W + bias and its gradients (dX, dW, dbias) for upstream dY,
    as nested lists; X: T×K, W: K×N, bias: N, dY: T×N."""
    T, K, N = len(X), len(X[0]), len(W[0])
    Y = [[math.fsum([X[t][k] * W[k][n] for k in range(K)] + [bias[n]]) for n in range(N)]
         for t in range(T)]
    db = [math.fsum(dY[t][n] for t in range(T)) for n in range(N)]
    dW = [[math.fsum(X[t][k] * dY[t][n] for t in range(T)) for n in range(N)] for k in range(K)]
    dX = [[math.fsum(dY[t][n] * W[k][n] for n in range(N)) for k in range(K)] for t in range(T)]
    return dict(Y=Y, dX=dX, dW=dW, db=db)
