"""The tensor-core epilogues compute Φ from the Hastings rational
approximation of erf (Abramowitz & Stegun eq. 7.1.26, |error| ≤ 1.5e−7)
instead of CUDA's erff. Checked here against CUDA's erff/expf form on the
GPU and against the fp64 oracle's GeLU and GeLU′."""
import numpy as np
import pytest
import torch

import oracle
from tensor_transformer_mlp_block_b200 import binding

pytestmark = pytest.mark.gpu


def _grid():
    x = np.concatenate([np.linspace(-12.0, 12.0, 200001), [0.0, -0.0, 1e-30, -1e-30, 88.0, -88.0]])
    return torch.tensor(x, dtype=torch.float32)


def test_fast_form_matches_cuda_erff_form():
    x = _grid().cuda()
    y0, d0 = binding.eval_activation(x, 0)
    y1, d1 = binding.eval_activation(x, 1)
    xa = x.abs().double()
    # Φ differs by at most ~3e-7 (approximation + fast exp/reciprocal)
    assert torch.all((y0.double() - y1.double()).abs() <= 4e-7 * xa + 1e-30)
    assert torch.all((d0.double() - d1.double()).abs() <= 4e-7 * (1 + xa))


def test_fast_form_against_fp64_oracle():
    x = _grid()
    y0, d0 = binding.eval_activation(x.cuda(), 0)
    y0, d0 = y0.cpu().double().numpy(), d0.cpu().double().numpy()
    xs = x.double().numpy()
    idx = np.linspace(0, len(xs) - 1, 4001).astype(int)
    for i in idx:
        g, dg = oracle.gelu(xs[i]), oracle.gelu_grad(xs[i])
        assert abs(y0[i] - g) <= 4e-7 * abs(xs[i]) + 1e-7 * abs(g) + 1e-37, (xs[i], y0[i], g)
        assert abs(d0[i] - dg) <= 4e-7 * (1 + abs(xs[i])), (xs[i], d0[i], dg)
    # exact special values of the form
    assert y0[np.where(xs == 0.0)[0][0]] == 0.0
    assert abs(d0[np.where(xs == 0.0)[0][0]] - 0.5) < 1e-7


def test_tanh_forms_match_each_other_and_the_oracle():
    """The tanh approximation as the tensor-core epilogues compute it (tanh
    from one exponential) against CUDA's tanhf form and the fp64 oracle."""
    x = _grid()
    y2, d2 = binding.eval_activation(x.cuda(), 2)
    y3, d3 = binding.eval_activation(x.cuda(), 3)
    xa = x.abs().double().cuda()
    assert torch.all((y2.double() - y3.double()).abs() <= 1e-6 * xa + 1e-30)
    assert torch.all((d2.double() - d3.double()).abs() <= 2e-6 * (1 + xa))
    y2, d2 = y2.cpu().double().numpy(), d2.cpu().double().numpy()
    xs = x.double().numpy()
    for i in np.linspace(0, len(xs) - 1, 4001).astype(int):
        g, dg = oracle.gelu_tanh(xs[i]), oracle.gelu_tanh_grad(xs[i])
        assert abs(y2[i] - g) <= 1e-6 * abs(xs[i]) + 1e-7 * abs(g) + 1e-37, (xs[i], y2[i], g)
        assert abs(d2[i] - dg) <= 2e-6 * (1 + abs(xs[i])), (xs[i], d2[i], dg)
