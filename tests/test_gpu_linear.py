"""GPU parity of the tensor-parallel linear layers (the attention side of the
tensor-parallel Transformer layer: QKV projection split by columns, output
projection split by rows) against the fp64 oracle.

Tolerances as for the MLP block: max|err| ≤ 2e-2·rms(ref) for bf16 inputs
with fp32 accumulation (Y, dX bf16; dW, dbias fp32), 1e-5·rms for fp32.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import TOL, rel_err, to_np
from tensor_transformer_mlp_block_b200 import binding
from tensor_transformer_mlp_block_b200.inputs import sample_indices

pytestmark = pytest.mark.gpu


def _inputs(T, K, N, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    X = torch.randn((T, K), generator=g).to(dt)
    W = (torch.randn((K, N), generator=g) * (1.0 / np.sqrt(K))).to(dt)
    bias = (torch.randn((N,), generator=g) * 0.1).to(dt)
    dY = torch.randn((T, N), generator=g).to(dt)
    return dict(X=X, W=W, bias=bias, dY=dY)


def _run(inp, p, split):
    d = {k: v.cuda() for k, v in inp.items()}
    Y = binding.linear_forward(d["X"], d["W"], d["bias"], p, split)
    dX, dW, db = binding.linear_backward(d["dY"], d["X"], d["W"], p, split)
    torch.cuda.synchronize()
    assert binding.last_device_status() == binding.OK
    return dict(Y=Y.cpu(), dX=dX.cpu(), dW=dW.cpu(), db=db.cpu())


def _check(got, ref, dtype):
    errs = {k: rel_err(to_np(got[k]), ref[k]) for k in ref}
    bad = {k: e for k, e in errs.items() if not e <= TOL[dtype]}
    assert not bad, (bad, errs)
    return errs


def _oracle(inp):
    n = {k: to_np(v) for k, v in inp.items()}
    Y = oracle.linear_forward(n["X"], n["W"], n["bias"])
    dX, dW, db = oracle.linear_backward(n["X"], n["W"], n["dY"])
    return dict(Y=Y, dX=dX, dW=dW, db=db)


@pytest.fixture(autouse=True)
def _auto_policy():
    binding.set_split_policy(0)
    yield
    binding.set_split_policy(0)


@pytest.mark.parametrize("T,K,N,p,split", [
    (256, 768, 2304, 2, "columns"),  # GPT-2-small QKV projection (h -> 3h), TP 2
    (256, 768, 768, 2, "rows"),      # GPT-2-small output projection, TP 2
    (300, 200, 520, 2, "columns"),   # ragged rows, K and N
    (300, 200, 520, 4, "rows"),
    (129, 64, 264, 3, "columns"),
    (1, 8, 8, 1, "rows"),
    (64, 32, 48, 48, "columns"),     # p = N: one output column per shard
    (64, 48, 32, 48, "rows"),        # p = K: one input row of W per shard
])
def test_linear_bf16_full_oracle(T, K, N, p, split):
    inp = _inputs(T, K, N, "bf16", seed=T + K + N)
    _check(_run(inp, p, split), _oracle(inp), "bf16")


@pytest.mark.parametrize("split", ["columns", "rows"])
def test_linear_plain_path_and_fp32(split):
    inp = _inputs(37, 12, 44, "bf16", seed=5)
    _check(_run(inp, 2, split), _oracle(inp), "bf16")
    inp = _inputs(512, 12, 48, "fp32", seed=6)
    _check(_run(inp, 2, split), _oracle(inp), "fp32")


@pytest.mark.parametrize("policy", [1, 2, 3])
@pytest.mark.parametrize("split", ["columns", "rows"])
def test_linear_shard_sum_schedules(policy, split):
    """Both schedules of the product that carries the shard sum (the forward
    of the row split, dX of the column split) match the oracle."""
    binding.set_split_policy(policy)
    inp = _inputs(256, 512, 1024, "bf16", seed=7)
    _check(_run(inp, 4, split), _oracle(inp), "bf16")


@pytest.mark.parametrize("split,K,N", [("columns", 4096, 12288), ("rows", 4096, 4096)])
def test_linear_7b_attention_projections_sampled(split, K, N):
    """7B-class attention projections (T = 8192, TP 2) on exact subsets: token
    rows R of Y and dX, columns J of dW and dbias."""
    T, p = 8192, 2
    inp = _inputs(T, K, N, "bf16", seed=8)
    got = _run(inp, p, split)
    n = {k: to_np(v) for k, v in inp.items()}
    R = sample_indices(T, 24, seed=1234).numpy()
    J = sample_indices(N, 48, seed=1235).numpy()
    Y_R = oracle.linear_forward(n["X"][R], n["W"], n["bias"])
    dX_R, _, _ = oracle.linear_backward(n["X"][R], n["W"], n["dY"][R])
    _, dW_J, db_J = oracle.linear_backward(n["X"], n["W"][:, J], n["dY"][:, J])
    errs = {"Y[R]": rel_err(to_np(got["Y"][R]), Y_R), "dX[R]": rel_err(to_np(got["dX"][R]), dX_R),
            "dW[:,J]": rel_err(to_np(got["dW"][:, J]), dW_J), "db[J]": rel_err(to_np(got["db"][J]), db_J)}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_linear_errors():
    d = {k: v.cuda() for k, v in _inputs(64, 64, 96, "bf16", seed=9).items()}
    with pytest.raises(binding.TPMLPError) as e:
        binding.linear_forward(d["X"], d["W"], d["bias"], 5, "columns")  # 96 % 5 != 0
    assert e.value.status == binding.ERR_INVALID
    with pytest.raises(ValueError):
        binding.linear_forward(d["X"], d["W"], d["bias"], 2, "diagonal")
