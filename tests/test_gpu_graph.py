"""Forward + backward captured in one CUDA graph and replayed: the library's
launches are stream-ordered and capture-safe once the first (eager) call on
the device has set the kernels' attributes. Replays reproduce the eager
results bit for bit, and the replayed outputs match the fp64 oracle."""
import pytest
import torch

from parity_util import compare_full, oracle_full
from tensor_transformer_mlp_block_b200 import binding
from tensor_transformer_mlp_block_b200.inputs import make_shape

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,h,F,p", [(512, 256, 1024, 2), (4096, 768, 3072, 2)])
def test_graph_replay_matches_eager(T, h, F, p):
    inp = make_shape(T, h, F, "bf16", seed_offset=41)
    d = {k: v.cuda() for k, v in inp.items()}
    bf, f32 = torch.bfloat16, torch.float32
    H = torch.empty((T, F), dtype=bf, device="cuda")
    Y = torch.empty_like(H)
    Z = torch.empty((T, h), dtype=bf, device="cuda")
    g = dict(dX=torch.empty((T, h), dtype=bf, device="cuda"), dA=torch.empty((h, F), dtype=f32, device="cuda"),
             da=torch.empty((F,), dtype=f32, device="cuda"), dB=torch.empty((F, h), dtype=f32, device="cuda"),
             db=torch.empty((h,), dtype=f32, device="cuda"), dH=torch.empty((T, F), dtype=bf, device="cuda"))
    ws = torch.empty(max(binding.workspace_size(T, h, F, p), 1), dtype=torch.uint8, device="cuda")

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
    for t in [H, Y, Z, *g.values()]:
        t.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert binding.last_device_status() == binding.OK
    got = {"H": H, "Y": Y, "Z": Z, **g}
    for k, v in eager.items():
        assert torch.equal(got[k], v), k
    # the replayed results themselves against the oracle on the same inputs
    compare_full({k: v.cpu() for k, v in got.items()}, oracle_full(inp), "bf16")
