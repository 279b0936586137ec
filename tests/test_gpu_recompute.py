"""Activation recompute: a caller keeps only H after the forward and
rebuilds Y = act(H) before the backward (tp_mlp_recompute_activation).

The rebuilt Y is compared element by element with the oracle's activation
of the same stored H (only the output rounding and the kernels' activation
form separate them), and a backward run on the rebuilt Y must still match
the oracle's gradients within the block's tolerance."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import compare_full, oracle_full, to_np
from tensor_transformer_mlp_block_b200 import binding, configs
from tensor_transformer_mlp_block_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,act", [("bf16", "gelu"), ("bf16", "gelu_tanh"),
                                       ("fp32", "gelu"), ("fp32", "gelu_tanh")])
@pytest.mark.parametrize("n", [4096 * 8, 1001])
def test_recomputed_activation_matches_oracle(dtype, act, n):
    g = torch.Generator().manual_seed(n)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    H = (torch.randn(n, generator=g) * 2.0).to(dt)
    Y = binding.recompute_activation(H.cuda(), activation=act).cpu()
    f = oracle.gelu if act == "gelu" else oracle.gelu_tanh
    h = to_np(H)
    ref = np.array([f(x) for x in h])
    u = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -23
    err = np.abs(to_np(Y) - ref) - u * np.abs(ref) - 1e-6 * np.abs(h)
    assert float(err.max()) <= 1e-30


def test_backward_on_recomputed_activation():
    """fwd -> drop Y -> rebuild Y from H -> bwd: gradients match the oracle."""
    for name in ("gpt2-small",):
        cfg = configs.get(name)
        inp = make_inputs(cfg)
        d = {k: v.cuda() for k, v in inp.items()}
        H, Y, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], cfg.p)
        Y_fwd = Y.clone()
        Y.zero_()
        binding.recompute_activation(H, out=Y)
        # The forward's Y is act(H) before H is rounded, the rebuilt one
        # act(round(H)): besides each side's own output rounding (2^-8
        # relative, bf16), they differ by |act'| <= 1.13 times the rounding of
        # H (2^-8·|H|).
        y, y0, h = to_np(Y), to_np(Y_fwd), to_np(H)
        bound = 2.0 ** -8 * (np.abs(y) + np.abs(y0)) + 1.13 * 2.0 ** -8 * np.abs(h) + 1e-6
        assert float((np.abs(y - y0) - bound).max()) <= 0.0
        g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, cfg.p)
        torch.cuda.synchronize()
        got = dict(H=H.cpu(), Y=Y.cpu(), Z=Z.cpu(), **{k: v.cpu() for k, v in g.items()})
        ref = oracle_full(inp)
        compare_full(got, ref, "bf16", keys=["dH", "dX", "dA", "da", "dB", "db"])


def test_recompute_errors_and_empty():
    H = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    assert binding.recompute_activation(H[:0]).numel() == 0
    with pytest.raises(ValueError):
        binding.recompute_activation(H, activation="relu")
    L = binding.lib()
    assert L.tp_mlp_recompute_activation(H.data_ptr(), H.data_ptr(), -1, 0, 0, None) == binding.ERR_INVALID


@pytest.mark.parametrize("T,h,F,p,dtype,act", [
    (300, 200, 520, 2, "bf16", "gelu"),        # tensor-core path, ragged tails
    (256, 128, 512, 4, "bf16", "gelu_tanh"),
    (37, 12, 44, 2, "bf16", "gelu"),           # plain path (h, F not multiples of 8)
    (512, 12, 48, 2, "fp32", "gelu"),          # fp32 toy shape
])
def test_recompute_hidden_is_the_forward_first_product(T, h, F, p, dtype, act):
    """H and Y rebuilt from X are bitwise those of the forward."""
    from tensor_transformer_mlp_block_b200.inputs import make_shape
    inp = make_shape(T, h, F, dtype, seed_offset=T + F)
    d = {k: v.cuda() for k, v in inp.items()}
    H, Y, _ = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p, activation=act)
    H2, Y2 = binding.recompute_hidden(d["X"], d["A"], d["a"], p, activation=act)
    torch.cuda.synchronize()
    assert torch.equal(H, H2) and torch.equal(Y, Y2)


def test_backward_on_hidden_recomputed_from_x():
    """fwd -> drop H and Y -> rebuild both from X -> bwd: gradients match the oracle."""
    cfg = configs.get("gpt2-small")
    inp = make_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    _, _, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], cfg.p)
    H, Y = binding.recompute_hidden(d["X"], d["A"], d["a"], cfg.p)
    g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, cfg.p)
    torch.cuda.synchronize()
    got = dict(H=H.cpu(), Y=Y.cpu(), Z=Z.cpu(), **{k: v.cpu() for k, v in g.items()})
    compare_full(got, oracle_full(inp), "bf16")


def test_recompute_hidden_errors():
    X = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((64, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.TPMLPError) as e:
        binding.recompute_hidden(X, A, None, 5)  # 96 % 5 != 0
    assert e.value.status == binding.ERR_INVALID
    with pytest.raises(ValueError):
        binding.recompute_hidden(X, A, None, 2, activation="relu")
    L = binding.lib()
    assert L.tp_mlp_recompute_hidden(None, A.data_ptr(), None, X.data_ptr(), X.data_ptr(),
                                     64, 64, 96, 2, 0, 0, None) == binding.ERR_INVALID
    H, Y = binding.recompute_hidden(X[:0], A, None, 2)
    assert H.shape == (0, 96) and Y.shape == (0, 96)
