"""GPU-side error behaviour: argument errors return before any launch, the
bounded-wait path reports a timeout and leaves the context usable."""
import pytest
import torch

from parity_util import compare_full, oracle_full, run_gpu
from tensor_transformer_mlp_block_b200 import binding
from tensor_transformer_mlp_block_b200.inputs import make_shape

pytestmark = pytest.mark.gpu


def _dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def test_misaligned_pointer_is_rejected():
    d = _dev(make_shape(128, 64, 256, "bf16"))
    X_big = torch.zeros(128 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    X_off = X_big[1:].view(128, 64)  # 2-byte offset
    before = binding.launch_count()
    with pytest.raises(binding.TPMLPError) as e:
        binding.forward(X_off, d["A"], d["a"], d["B"], d["b"], 2)
    assert e.value.status == binding.ERR_ALIGN
    assert binding.launch_count() == before


def test_small_workspace_is_rejected():
    binding.set_split_policy(2)
    try:
        d = _dev(make_shape(128, 256, 1024, "bf16"))
        need = binding.workspace_size(128, 256, 1024, 4)
        assert need > 0
        ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
        with pytest.raises(ValueError):
            binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], 4, workspace=ws)
        L = binding.lib()
        H = torch.empty((128, 1024), dtype=torch.bfloat16, device="cuda")
        st = L.tp_mlp_fwd(d["X"].data_ptr(), d["A"].data_ptr(), None, d["B"].data_ptr(), None,
                          H.data_ptr(), H.data_ptr(), d["X"].data_ptr(), 128, 256, 1024, 4,
                          binding.BF16, ws.data_ptr(), need - 256, None)
        assert st == binding.ERR_WORKSPACE
    finally:
        binding.set_split_policy(0)


def test_invalid_shard_count():
    d = _dev(make_shape(128, 64, 256, "bf16"))
    for p in (0, 3, -1):
        with pytest.raises(binding.TPMLPError) as e:
            binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p)
        assert e.value.status == binding.ERR_INVALID


def test_bounded_wait_times_out_and_context_survives():
    binding.wait_selftest(2_000_000)  # 2 ms on a barrier nothing completes
    assert binding.last_device_status() == binding.ERR_TIMEOUT
    assert binding.last_device_status() == binding.OK  # read clears it
    inp = make_shape(256, 128, 512, "bf16", seed_offset=23)
    compare_full(run_gpu(inp, 2), oracle_full(inp), "bf16")
