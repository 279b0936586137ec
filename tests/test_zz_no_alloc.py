"""tp_mlp_bwd_noalloc: the backward for callers that cannot allocate device
memory when they run it, such as a plugin inside another framework that owns
every device allocation, or a runtime with a fixed memory budget after
start-up. It keeps its only scratch (the bias gradients' partial column
sums) in a fixed array inside the library and takes no workspace.

Each case calls it twice in a row through the C ABI, on outputs pre-filled
with NaN, and checks every gradient against the regular tp_mlp_bwd within
the tests' tolerance. This file is collected last on purpose.
"""
import pytest
import torch

from parity_util import TOL, rel_err, to_np
from tensor_transformer_mlp_block_b200 import binding
from tensor_transformer_mlp_block_b200.inputs import make_shape

pytestmark = pytest.mark.gpu


def _fresh(T, h, F, dt):
    nan = float("nan")
    f32 = torch.float32
    return dict(dX=torch.full((T, h), nan, dtype=dt, device="cuda"),
                dA=torch.full((h, F), nan, dtype=f32, device="cuda"),
                da=torch.full((F,), nan, dtype=f32, device="cuda"),
                dB=torch.full((F, h), nan, dtype=f32, device="cuda"),
                db=torch.full((h,), nan, dtype=f32, device="cuda"),
                dH=torch.full((T, F), nan, dtype=dt, device="cuda"))


def _noalloc(d, H, Y, out, T, h, F, p):
    L = binding.lib()
    code = binding.BF16 if d["X"].dtype == torch.bfloat16 else binding.FP32
    return L.tp_mlp_bwd_noalloc(
        d["dZ"].data_ptr(), d["X"].data_ptr(), d["A"].data_ptr(), d["B"].data_ptr(),
        H.data_ptr(), Y.data_ptr(), out["dX"].data_ptr(), out["dA"].data_ptr(),
        out["da"].data_ptr(), out["dB"].data_ptr(), out["db"].data_ptr(), out["dH"].data_ptr(),
        T, h, F, p, code, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("T,h,F,p,dtype", [
    (256, 768, 3072, 2, "bf16"),  # tp_mlp_bwd splits dX by shard here; this one never does
    (300, 4096, 1024, 2, "bf16"), # h ≥ 3072: the relaying GeLU′ epilogue without da partials
    (300, 200, 520, 2, "bf16"),   # ragged tiles
    (37, 12, 44, 2, "bf16"),      # plain CUDA-core path
    (512, 12, 48, 2, "fp32"),     # the fp32 workload
])
def test_noalloc_backward_matches_backward_twice(T, h, F, p, dtype):
    binding.set_split_policy(0)
    inp = make_shape(T, h, F, dtype, seed_offset=31 + T)
    d = {k: v.cuda() for k, v in inp.items()}
    H, Y, _ = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p)
    ref = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, p)
    torch.cuda.synchronize()
    ref = {k: to_np(v) for k, v in ref.items()}
    for call in range(2):
        out = _fresh(T, h, F, d["X"].dtype)
        assert _noalloc(d, H, Y, out, T, h, F, p) == binding.OK
        torch.cuda.synchronize()
        assert binding.last_device_status() == binding.OK
        for k, r in ref.items():
            # dX and dH are stored in bf16 by both calls, each rounding once;
            # where the two sum in different orders they may round the same
            # value to neighbouring bf16 numbers (up to u·|value| each)
            u = 2 * 2.0 ** -8 if out[k].dtype == torch.bfloat16 else 0.0
            err = rel_err(to_np(out[k]), r, u)
            assert err <= TOL[dtype], (call, k, err)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = binding.lib()
    cap = L.tpmlp_noalloc_scratch_bytes()
    assert cap == 8 << 20
    T, h, F = 65536, 4096, 16384  # needs 4·512·(h + F) bytes ≫ 8 MiB
    assert 4 * (T // 128) * (h + F) > cap
    before = binding.launch_count()
    dummy = 256  # never dereferenced: the size check comes first
    st = L.tp_mlp_bwd_noalloc(*([dummy] * 12), T, h, F, 2, binding.BF16, None)
    assert st == binding.ERR_WORKSPACE
    assert binding.launch_count() == before
