"""Launch overlap (programmatic dependent launches between the library's
kernels) changes when kernels start, never what they compute: results are
bit-identical with it on or off, for single calls and for steps issued back
to back on shared buffers without host synchronisation."""
import pytest
import torch

from parity_util import compare_full, oracle_full
from tensor_transformer_mlp_block_b200 import binding, configs
from tensor_transformer_mlp_block_b200.inputs import make_inputs, make_shape

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _restore():
    yield
    binding.set_launch_overlap(True)
    binding.set_split_policy(0)


def _step(d, p, act="gelu", out=None):
    H, Y, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p, activation=act,
                              out=None if out is None else out[0])
    g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, p, activation=act,
                         out=None if out is None else out[1])
    return dict(H=H, Y=Y, Z=Z, **g)


def _both(inp, p, act="gelu"):
    d = {k: v.cuda() for k, v in inp.items()}
    res = {}
    for on in (False, True):
        binding.set_launch_overlap(on)
        r = _step(d, p, act)
        torch.cuda.synchronize()
        assert binding.last_device_status() == binding.OK
        res[on] = {k: v.cpu() for k, v in r.items()}
    return res


@pytest.mark.parametrize("T,h,F,p,policy,act", [
    (300, 200, 520, 2, 0, "gelu"),       # ragged, one-CTA and pair kernels
    (384, 320, 1024, 4, 2, "gelu"),      # row products split by shard + ordered reduction
    (256, 128, 512, 4, 1, "gelu_tanh"),
    (37, 12, 44, 2, 0, "gelu"),          # plain kernels (ordinary launches)
    (600, 3072, 1536, 2, 3, "gelu"),     # stream-K tail in every product
])
def test_overlap_on_off_bit_identical(T, h, F, p, policy, act):
    binding.set_split_policy(policy)
    res = _both(make_shape(T, h, F, "bf16", seed_offset=T + h), p, act)
    for k in res[False]:
        assert torch.equal(res[False][k], res[True][k]), k


def test_overlap_gpt2_full_oracle():
    cfg = configs.get("gpt2-small")
    inp = make_inputs(cfg)
    res = _both(inp, cfg.p)
    for k in res[False]:
        assert torch.equal(res[False][k], res[True][k]), k
    compare_full(res[True], oracle_full(inp), "bf16")


@pytest.mark.parametrize("policy", [0, 2, 3])
def test_back_to_back_steps_on_shared_buffers(policy):
    """Five steps with new X and dZ each, all writing the same H, Y, Z and
    gradient buffers, queued without synchronising: each step's results
    (copied out on the stream right after it) match the same steps run with
    overlap off."""
    binding.set_split_policy(policy)
    T, h, F, p = 512, 256, 1024, 2
    steps = [make_shape(T, h, F, "bf16", seed_offset=100 + i) for i in range(5)]
    base = {k: v.cuda() for k, v in steps[0].items()}
    dt = torch.bfloat16
    out = ((torch.empty(T, F, dtype=dt, device="cuda"), torch.empty(T, F, dtype=dt, device="cuda"),
            torch.empty(T, h, dtype=dt, device="cuda")),
           dict(dX=torch.empty(T, h, dtype=dt, device="cuda"),
                dA=torch.empty(h, F, device="cuda"), da=torch.empty(F, device="cuda"),
                dB=torch.empty(F, h, device="cuda"), db=torch.empty(h, device="cuda"),
                dH=torch.empty(T, F, dtype=dt, device="cuda")))
    results = {}
    for on in (False, True):
        binding.set_launch_overlap(on)
        copies = []
        for s in steps:
            d = dict(base, X=s["X"].cuda(), dZ=s["dZ"].cuda())
            r = _step(d, p, out=out)
            copies.append({k: v.clone() for k, v in r.items()})
        torch.cuda.synchronize()
        assert binding.last_device_status() == binding.OK
        results[on] = copies
    for i in range(len(steps)):
        for k in results[False][i]:
            assert torch.equal(results[False][i][k], results[True][i][k]), (i, k)
    # and the steps really differ from each other
    assert not torch.equal(results[True][0]["dA"], results[True][1]["dA"])


def test_overlap_switch_roundtrip():
    binding.set_launch_overlap(False)
    assert binding.get_launch_overlap() is False
    binding.set_launch_overlap(True)
    assert binding.get_launch_overlap() is True
