"""Shared helpers of the GPU parity tests: run the CUDA path, run the oracle
on the same rounded inputs, compare with the block's tolerance.

Tolerance (per output tensor O): max|O_gpu − O_ref| ≤ tol · rms(O_ref),
tol = 2e-2 for bf16 inputs with fp32 accumulation and 1e-5 for fp32.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"bf16": 2e-2, "fp32": 1e-5}

# H, Y and dH are activations the block stores (in the input dtype) for the
# backward, not outputs or gradients of the block. Their storage rounding
# alone reaches u·|value| (u = 2^-8, the bf16 unit roundoff), which for the
# skewed GeLU output exceeds 2e-2·rms at its largest values; their bound adds
# that rounding: |got − ref| ≤ tol·rms(ref) + u·|ref|, element by element.
STORED = ("H", "Y", "dH")
UNIT_ROUNDOFF = {"bf16": 2.0 ** -8, "fp32": 2.0 ** -24}

# The products that consume a stored bf16 activation (Z = Y·B, dX = dH·Aᵀ,
# dA = Xᵀ·dH, dB = Yᵀ·dZ, da = 1ᵀ·dH) inherit its rounding: an element
# Σ_k a_k·b_k whose a_k each carry a relative error ≤ 2⁻⁹ is off by at most
# 2⁻⁹·Σ_k |a_k·b_k| ≤ u·(Σ_k (a_k·b_k)²)^½ for up to 4 terms (Cauchy–Schwarz),
# and for more terms that is still above 3σ of the random rounding errors.
# With many terms it is far below tol·rms; with 1–2 tokens an element of dA
# or dB is a single product, where the rms-relative bound alone does not hold.
# That allowance is added element by element, as for the stored activations.


class OracleResult(dict):
    """The oracle's outputs, with the rounded inputs they were computed from."""

    inputs: dict


def product_allowance(key: str, ref: OracleResult, dtype: str):
    """u·(Σ_k (a_k·b_k)²)^½ for the products that read a stored bf16
    activation, element by element (None for the others, or for fp32)."""
    if dtype != "bf16" or not hasattr(ref, "inputs"):
        return None
    n = ref.inputs
    u = UNIT_ROUNDOFF["bf16"]
    Y, dH = ref["Y"], ref["dH"]
    if key == "Z":
        return u * np.sqrt((Y * Y) @ (n["B"] * n["B"]))
    if key == "dX":
        return u * np.sqrt((dH * dH) @ (n["A"] * n["A"]).T)
    if key == "dA":
        return u * np.sqrt((n["X"] * n["X"]).T @ (dH * dH))
    if key == "dB":
        return u * np.sqrt((Y * Y).T @ (n["dZ"] * n["dZ"]))
    if key == "da":
        return u * np.sqrt((dH * dH).sum(axis=0))
    return None


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(got, ref, u: float = 0.0, allow=None) -> float:
    """max over elements of (|got − ref| − u·|ref| − allow), divided by rms(ref)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    slack = u * np.abs(ref) + (0.0 if allow is None else np.asarray(allow, dtype=np.float64))
    err = float(np.max(np.abs(got - ref) - slack))
    if rms == 0.0:
        return max(err, 0.0)
    return err / rms


def _u(key: str, dtype: str) -> float:
    return UNIT_ROUNDOFF[dtype] if key.split("[")[0] in STORED else 0.0


def run_gpu(inp: dict, p: int, device="cuda:0", activation: str = "gelu", keep_on_device=False):
    """Forward + backward on the GPU through the binding. Returns CPU tensors
    (or the device tensors with keep_on_device)."""
    from tensor_transformer_mlp_block_b200 import binding
    d = {k: v.to(device) for k, v in inp.items()}
    H, Y, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p, activation=activation)
    g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, p, activation=activation)
    torch.cuda.synchronize(device)
    st = binding.last_device_status(device=device)
    assert st == 0, f"device status {st}"
    out = dict(H=H, Y=Y, Z=Z, **g)
    if keep_on_device:
        return out
    return {k: v.cpu() for k, v in out.items()}


def oracle_full(inp: dict, act: int = 0):
    """Full fp64 oracle on the rounded inputs (act: 0 exact GeLU, 1 tanh form)."""
    n = {k: to_np(v) for k, v in inp.items()}
    H, Y, Z = oracle.forward(n["X"], n["A"], n["a"], n["B"], n["b"], act)
    g = oracle.backward(n["X"], n["A"], n["B"], H, Y, n["dZ"], act)
    out = OracleResult(H=H, Y=Y, Z=Z, **g)
    out.inputs = n
    return out


def compare_full(gpu: dict, ref: dict, dtype: str, keys=None) -> dict:
    tol = TOL[dtype]
    errs = {}
    for k in keys or ref:
        errs[k] = rel_err(to_np(gpu[k]), ref[k], _u(k, dtype), product_allowance(k, ref, dtype))
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"outside {tol}·rms: {bad} (all: {errs})"
    print("parity", {k: round(v, 5) for k, v in errs.items()})
    return errs


def oracle_sampled(inp: dict, R, J, act: int = 0) -> dict:
    """The oracle's exact values on token rows R (H, Y, Z, dH, dX) and hidden
    columns J (H, Y, dH, dA, da, dB), plus db in full."""
    n = {k: to_np(v) for k, v in inp.items()}
    R = np.asarray(R)
    J = np.asarray(J)
    r = oracle.rows(n["X"], n["A"], n["a"], n["B"], n["b"], n["dZ"], R, act)
    # the column subset needs only A[:, J], a[J], B[J, :]
    c = oracle.cols(n["X"], n["A"][:, J], n["a"][J], n["B"][J, :], n["dZ"], np.arange(len(J)), act)
    return {"R": R, "J": J, "rows": r, "cols": c, "db": oracle.colsum(n["dZ"])}


def compare_to_sampled(gpu: dict, ref: dict, dtype: str) -> dict:
    """Compare GPU outputs (CPU or CUDA tensors) with oracle_sampled's values."""
    R, J, r, c = ref["R"], ref["J"], ref["rows"], ref["cols"]
    tol = TOL[dtype]
    errs = {}
    for k in ("H", "Y", "Z", "dH", "dX"):
        errs[f"{k}[R]"] = rel_err(to_np(gpu[k][R]), r[k], _u(k, dtype))
    for k in ("H", "Y", "dH"):
        errs[f"{k}[:,J]"] = rel_err(to_np(gpu[k][:, J]), c[k], _u(k, dtype))
    errs["dA[:,J]"] = rel_err(to_np(gpu["dA"][:, J]), c["dA"])
    errs["da[J]"] = rel_err(to_np(gpu["da"][J]), c["da"])
    errs["dB[J]"] = rel_err(to_np(gpu["dB"][J]), c["dB"])
    errs["db"] = rel_err(to_np(gpu["db"]), ref["db"])
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"outside {tol}·rms: {bad} (all: {errs})"
    print("parity", {k: round(v, 5) for k, v in errs.items()})
    return errs


def compare_sampled(gpu: dict, inp: dict, R, J, dtype: str, act: int = 0) -> dict:
    """Compare on token rows R and hidden columns J, each computed exactly by
    the oracle (rows: H, Y, Z, dH, dX; columns: H, Y, dH, dA, da, dB), plus
    db in full."""
    return compare_to_sampled(gpu, oracle_sampled(inp, R, J, act), dtype)
