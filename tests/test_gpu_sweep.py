"""A seeded sweep of random shapes through the whole block against the full
oracle: token counts from 1 to ~700 (ragged against every tile size),
hidden and shard sizes on both sides of the tensor-core path's 16-byte rule,
p from 1 to 8, both split policies, both activations, launch overlap on and
off. The shapes come from a fixed seed, so the sweep is the same every run."""
import random

import pytest

from parity_util import compare_full, oracle_full, run_gpu
from tensor_transformer_mlp_block_b200 import binding
from tensor_transformer_mlp_block_b200.inputs import make_shape

pytestmark = pytest.mark.gpu


def _cases(n=48, seed=2024):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        p = rng.choice([1, 2, 3, 4, 8])
        if i % 6 == 5:  # plain path: h or F not a multiple of 8
            h = rng.choice([4, 12, 20, 36])
            Fp = rng.choice([3, 5, 6, 10])
        else:           # tensor-core path
            h = 8 * rng.randint(1, 48)
            Fp = 8 * rng.randint(1, 40)
        T = rng.choice([1, 2, 17, 64, 127, 128, 129, 255, 256, 257]) if i % 3 == 0 else rng.randint(1, 700)
        out.append(dict(T=T, h=h, F=Fp * p, p=p, policy=rng.choice([0, 1, 2, 3]),
                        act=rng.choice(["gelu", "gelu_tanh"]), overlap=rng.random() < 0.7, seed=i))
    return out


@pytest.fixture(autouse=True)
def _restore():
    yield
    binding.set_split_policy(0)
    binding.set_launch_overlap(True)


@pytest.mark.parametrize("c", _cases(), ids=lambda c: "T{T}-h{h}-F{F}-p{p}-s{policy}-{act}-o{overlap:d}".format(**c))
def test_random_shape_against_oracle(c):
    binding.set_split_policy(c["policy"])
    binding.set_launch_overlap(c["overlap"])
    inp = make_shape(c["T"], c["h"], c["F"], "bf16", seed_offset=1000 + c["seed"])
    gpu = run_gpu(inp, c["p"], activation=c["act"])
    compare_full(gpu, oracle_full(inp, act=1 if c["act"] == "gelu_tanh" else 0), "bf16")


def _linear_cases(n=24, seed=77):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        p = rng.choice([1, 2, 3, 4, 8])
        split = rng.choice(["columns", "rows"])
        if i % 6 == 5:  # plain path
            K = rng.choice([4, 12, 20]) * (p if split == "rows" else 1)
            N = rng.choice([6, 10, 14]) * (p if split == "columns" else 1)
        else:
            K = 8 * rng.randint(1, 40) * (p if split == "rows" else 1)
            N = 8 * rng.randint(1, 40) * (p if split == "columns" else 1)
        T = rng.choice([1, 2, 127, 128, 129, 256, 257]) if i % 3 == 0 else rng.randint(1, 600)
        out.append(dict(T=T, K=K, N=N, p=p, split=split, policy=rng.choice([0, 1, 2, 3]),
                        overlap=rng.random() < 0.7, seed=i))
    return out


@pytest.mark.parametrize("c", _linear_cases(),
                         ids=lambda c: "T{T}-K{K}-N{N}-p{p}-{split}-s{policy}-o{overlap:d}".format(**c))
def test_random_linear_against_oracle(c):
    import numpy as np
    import torch

    import oracle
    from parity_util import TOL, rel_err, to_np
    binding.set_split_policy(c["policy"])
    binding.set_launch_overlap(c["overlap"])
    g = torch.Generator().manual_seed(500 + c["seed"])
    T, K, N = c["T"], c["K"], c["N"]
    X = torch.randn((T, K), generator=g).to(torch.bfloat16)
    W = (torch.randn((K, N), generator=g) / np.sqrt(K)).to(torch.bfloat16)
    bias = (torch.randn((N,), generator=g) * 0.1).to(torch.bfloat16)
    dY = torch.randn((T, N), generator=g).to(torch.bfloat16)
    Y = binding.linear_forward(X.cuda(), W.cuda(), bias.cuda(), c["p"], c["split"])
    dX, dW, db = binding.linear_backward(dY.cuda(), X.cuda(), W.cuda(), c["p"], c["split"])
    torch.cuda.synchronize()
    assert binding.last_device_status() == binding.OK
    n = dict(X=to_np(X), W=to_np(W), bias=to_np(bias), dY=to_np(dY))
    ref_Y = oracle.linear_forward(n["X"], n["W"], n["bias"])
    ref_dX, ref_dW, ref_db = oracle.linear_backward(n["X"], n["W"], n["dY"])
    errs = {"Y": rel_err(to_np(Y.cpu()), ref_Y), "dX": rel_err(to_np(dX.cpu()), ref_dX),
            "dW": rel_err(to_np(dW.cpu()), ref_dW), "db": rel_err(to_np(db.cpu()), ref_db)}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def _fp32_cases(n=12, seed=5):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        p = rng.choice([1, 2, 3, 4])
        out.append(dict(T=rng.choice([1, 2, 15, 16, 17, 100, 257, 513]), h=rng.randint(1, 40),
                        F=rng.randint(1, 24) * p, p=p, act=rng.choice(["gelu", "gelu_tanh"]),
                        overlap=rng.random() < 0.7, seed=i))
    return out


@pytest.mark.parametrize("c", _fp32_cases(),
                         ids=lambda c: "T{T}-h{h}-F{F}-p{p}-{act}-o{overlap:d}".format(**c))
def test_random_fp32_shape_against_oracle(c):
    """fp32 (plain FFMA kernels, no TF32): within 1e-5·rms of the oracle."""
    binding.set_launch_overlap(c["overlap"])
    inp = make_shape(c["T"], c["h"], c["F"], "fp32", seed_offset=3000 + c["seed"])
    gpu = run_gpu(inp, c["p"], activation=c["act"])
    compare_full(gpu, oracle_full(inp, act=1 if c["act"] == "gelu_tanh" else 0), "fp32")
