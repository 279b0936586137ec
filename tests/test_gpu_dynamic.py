"""The dynamic tile schedule: tiles (and stream-K segments) handed out in
order from a counter in the workspace, so that faster CTA pairs take more of
them. Which pair computes a tile does not change its arithmetic, so results
must be bit-identical to the static round-robin; the counters must reset
themselves between launches, in eager calls and in CUDA-graph replays."""
import numpy as np
import pytest
import torch

from parity_util import compare_sampled, run_gpu
from tensor_transformer_mlp_block_b200 import binding
from tensor_transformer_mlp_block_b200.inputs import make_shape, sample_indices

pytestmark = pytest.mark.gpu

# the dynamic schedule runs bf16-output products of ≥ 4 waves of 74 CTA
# pairs, ≥ 192 k-blocks per tile and ≥ 3072 per pair: here X·A and dZ·Bᵀ
# (K = h = 24584, ragged; 8 × 96 pair tiles), Y·B and dH·Aᵀ (K = F = 24576;
# 8 × 97 tiles, ragged N), ~4000 k-blocks per pair each, at a ragged token
# count; the weight gradients (fp32, K = T) stay static.
# F/p = 6144 lets policy 2 cut the row products into shard units.
SHAPE = (2000, 24584, 24576, 4)


@pytest.fixture(autouse=True)
def _restore():
    binding.set_dynamic_schedule(True)
    yield
    binding.set_dynamic_schedule(True)
    binding.set_split_policy(0)


@pytest.mark.parametrize("policy", [0, 2, 3])
def test_dynamic_matches_static_bitwise(policy):
    T, h, F, p = SHAPE
    binding.set_split_policy(policy)
    inp = make_shape(T, h, F, "bf16", seed_offset=61 + policy)
    binding.set_dynamic_schedule(False)
    ref = run_gpu(inp, p, keep_on_device=True)
    binding.set_dynamic_schedule(True)
    got = run_gpu(inp, p, keep_on_device=True)
    for k in ref:
        assert torch.equal(ref[k], got[k]), k
    R = sample_indices(T, 12, seed=1234).numpy()
    J = sample_indices(F, 16, seed=1235).numpy()
    compare_sampled(got, inp, R, J, "bf16")


def test_dynamic_back_to_back_calls_on_one_workspace():
    """The last pair of each launch puts the counters back to zero: calls in a
    row on the same workspace give the same results."""
    T, h, F, p = SHAPE
    inp = make_shape(T, h, F, "bf16", seed_offset=67)
    d = {k: v.cuda() for k, v in inp.items()}
    ws = torch.empty(binding.workspace_size(T, h, F, p), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        H, Y, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p, workspace=ws)
        g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, p, workspace=ws)
        torch.cuda.synchronize()
        assert binding.last_device_status() == binding.OK
        outs.append(dict(H=H, Y=Y, Z=Z, **g))
    for o in outs[1:]:
        for k in o:
            assert torch.equal(o[k], outs[0][k]), k


def test_dynamic_graph_replay():
    T, h, F, p = SHAPE
    inp = make_shape(T, h, F, "bf16", seed_offset=71)
    d = {k: v.cuda() for k, v in inp.items()}
    bf, f32 = torch.bfloat16, torch.float32
    H = torch.empty((T, F), dtype=bf, device="cuda")
    Y = torch.empty_like(H)
    Z = torch.empty((T, h), dtype=bf, device="cuda")
    g = dict(dX=torch.empty((T, h), dtype=bf, device="cuda"), dA=torch.empty((h, F), dtype=f32, device="cuda"),
             da=torch.empty((F,), dtype=f32, device="cuda"), dB=torch.empty((F, h), dtype=f32, device="cuda"),
             db=torch.empty((h,), dtype=f32, device="cuda"), dH=torch.empty((T, F), dtype=bf, device="cuda"))
    ws = torch.empty(binding.workspace_size(T, h, F, p), dtype=torch.uint8, device="cuda")

    def step():
        binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p, out=(H, Y, Z), workspace=ws)
        binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, p, out=g, workspace=ws)

    step()
    torch.cuda.synchronize()
    eager = {"H": H.clone(), "Y": Y.clone(), "Z": Z.clone(), **{k: v.clone() for k, v in g.items()}}
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        for t in [H, Y, Z, *g.values()]:
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert binding.last_device_status() == binding.OK
        got = {"H": H, "Y": Y, "Z": Z, **g}
        for k, v in eager.items():
            assert torch.equal(got[k], v), k


def test_dynamic_plan_reserves_its_counters():
    binding.set_split_policy(0)
    T, h, F, p = SHAPE
    assert binding.get_dynamic_schedule()
    ws_dyn = binding.workspace_size(T, h, F, p)
    binding.set_dynamic_schedule(False)
    # the dynamic counters share a 256-byte block with the split counters
    assert 0 <= ws_dyn - binding.workspace_size(T, h, F, p) <= 256
