"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs, element by element.

Small cases use the full oracle and span several 128×256 output tiles, a
ragged K and ragged tails; the named workloads (GPT-2-small, 350M, 7B, 175B
MLPs) are checked on seeded token rows and hidden columns that the oracle
computes exactly, in the same launch configuration the bench times.
"""
import numpy as np
import pytest
import torch

from parity_util import (TOL, compare_full, compare_sampled, compare_to_sampled, oracle_full,
                         oracle_sampled, rel_err, run_gpu, to_np)
from tensor_transformer_mlp_block_b200 import configs
from tensor_transformer_mlp_block_b200.inputs import make_inputs, make_shape, sample_indices

pytestmark = pytest.mark.gpu


# shard-sum schedules of tpmlp_set_split_policy: 0 automatic, 1 whole tiles
# only, 2 every shard its own work unit, 3 stream-K tail wherever valid
POLICIES = (0, 1, 2, 3)


@pytest.fixture(autouse=True)
def _auto_policy():
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(0)
    yield
    binding.set_split_policy(0)


def test_tiny_fp32_full():
    cfg = configs.get("tiny")
    inp = make_inputs(cfg)
    gpu = run_gpu(inp, cfg.p)
    compare_full(gpu, oracle_full(inp), "fp32")


@pytest.mark.parametrize("T,h,F,p", [
    (300, 200, 520, 2),    # ragged M (2 tiles + 44 rows), ragged K (200), ragged N (520)
    (256, 128, 512, 4),    # whole tiles, Fp = 128 (two k-blocks per shard)
    (129, 64, 264, 3),     # one row past a tile, single k-block, Fp = 88
    (1, 8, 8, 1),          # single token, smallest aligned shape
    (640, 96, 776, 1),     # p = 1: the unsplit MLP
    (300, 3072, 520, 2),   # h ≥ 3072: relaying epilogues, da summed in the GeLU′ epilogue
    (100, 3072, 264, 3),   # the same on the one-CTA kernel (T ≤ 128), ragged F
])
def test_bf16_full_oracle(T, h, F, p):
    inp = make_shape(T, h, F, "bf16", seed_offset=T + h + F)
    gpu = run_gpu(inp, p)
    compare_full(gpu, oracle_full(inp), "bf16")


def test_bf16_unaligned_shape_plain_path():
    """h and F not multiples of 8: the plain CUDA-core kernels serve bf16."""
    inp = make_shape(37, 12, 44, "bf16", seed_offset=9)
    gpu = run_gpu(inp, 2)
    compare_full(gpu, oracle_full(inp), "bf16")


@pytest.mark.parametrize("policy", [1, 2, 3])
def test_row_parallel_split_policies(policy):
    """Every schedule of the row-parallel products (shard K-loop in tensor
    memory; per-shard fp32 partials summed in order; a stream-K tail) matches
    the oracle."""
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(policy)
    inp = make_shape(384, 320, 1024, "bf16", seed_offset=11)
    gpu = run_gpu(inp, 4)
    compare_full(gpu, oracle_full(inp), "bf16")


def test_shard_count_invariance():
    """p changes the partition, not the math: every p gives the oracle's
    result, and any two p agree within the same bound."""
    from tensor_transformer_mlp_block_b200 import binding
    inp = make_shape(256, 256, 2048, "bf16", seed_offset=13)
    ref = oracle_full(inp)
    outs = {}
    for policy in (1, 2):
        binding.set_split_policy(policy)
        for p in (1, 2, 4, 8):
            outs[(policy, p)] = run_gpu(inp, p)
            compare_full(outs[(policy, p)], ref, "bf16")
    base = outs[(1, 1)]
    for key, o in outs.items():
        for k in ref:
            rms = float(np.sqrt(np.mean(ref[k] ** 2)))
            diff = float(np.max(np.abs(to_np(o[k]) - to_np(base[k]))))
            assert diff <= TOL["bf16"] * rms, (key, k, diff / rms)


def test_deterministic_bitwise():
    inp = make_shape(300, 200, 520, "bf16", seed_offset=17)
    a = run_gpu(inp, 2)
    b = run_gpu(inp, 2)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_empty_tokens():
    from tensor_transformer_mlp_block_b200 import binding
    inp = make_shape(0, 64, 256, "bf16")
    d = {k: v.cuda() for k, v in inp.items()}
    H, Y, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], 2)
    assert H.shape == (0, 256) and Z.shape == (0, 64)
    out = dict(dX=torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"),
               dA=torch.full((64, 256), 7.0, device="cuda"), da=torch.full((256,), 7.0, device="cuda"),
               dB=torch.full((256, 64), 7.0, device="cuda"), db=torch.full((64,), 7.0, device="cuda"),
               dH=torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"))
    g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, 2, out=out)
    for k in ("dA", "da", "dB", "db"):
        assert torch.count_nonzero(g[k]).item() == 0, k


def test_nan_propagates_without_fault():
    from tensor_transformer_mlp_block_b200 import binding
    inp = make_shape(256, 128, 512, "bf16", seed_offset=19)
    inp["X"][5, 3] = float("nan")
    gpu = run_gpu(inp, 2)
    assert torch.isnan(gpu["Z"][5]).all()
    assert not torch.isnan(gpu["Z"][6]).any()
    assert binding.last_device_status() == 0


@pytest.mark.parametrize("name", ["gpt2-small", "350m", "7b", "175b"])
def test_named_config_sampled(name):
    cfg = configs.get(name)
    inp = make_inputs(cfg)
    gpu = run_gpu(inp, cfg.p, keep_on_device=True)
    R = sample_indices(cfg.T, 48, seed=1234).numpy()
    J = sample_indices(cfg.F, 64, seed=1235).numpy()
    errs = compare_sampled(gpu, inp, R, J, cfg.dtype)
    assert all(np.isfinite(list(errs.values())))


@pytest.mark.parametrize("name", ["gpt2-small", "350m"])
def test_named_config_full(name):
    """The GPT-2-small and 350M-class MLPs against the full oracle (every
    element of every output and gradient)."""
    cfg = configs.get(name)
    inp = make_inputs(cfg)
    gpu = run_gpu(inp, cfg.p)
    compare_full(gpu, oracle_full(inp), "bf16")


def test_shard_count_invariance_7b_sampled():
    """The 7B-class workload with p = 1, 2, 4, 8 under every shard-sum
    schedule: each matches the oracle on seeded rows and columns, and any two
    agree element by element (every output, in full) within the same bound."""
    from tensor_transformer_mlp_block_b200 import binding
    cfg = configs.get("7b")
    inp = make_inputs(cfg)
    R = sample_indices(cfg.T, 16, seed=1234).numpy()
    J = sample_indices(cfg.F, 32, seed=1235).numpy()
    ref = oracle_sampled(inp, R, J)
    base, rms = None, None
    for policy in POLICIES:
        binding.set_split_policy(policy)
        for p in (1, 2, 4, 8):
            out = run_gpu(inp, p, keep_on_device=True)
            compare_to_sampled(out, ref, "bf16")
            if base is None:
                base = out
                rms = {k: float(v.double().pow(2).mean().sqrt()) for k, v in base.items()}
                continue
            for k, v in out.items():
                # outputs stored in bf16 are each rounded once: two results
                # with different summation orders may round the same exact
                # value to neighbouring bf16 numbers, up to u·|value| each
                u = 2.0 ** -8 if v.dtype == torch.bfloat16 else 0.0
                excess = (v.double() - base[k].double()).abs() - 2.0 * u * base[k].double().abs()
                diff = float(excess.max())
                assert diff <= TOL["bf16"] * rms[k], (policy, p, k, diff / rms[k])
            del out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,h,F,p", [(300, 200, 520, 2), (256, 128, 512, 4), (37, 12, 44, 2)])
def test_gelu_tanh_variant(T, h, F, p):
    """The tanh approximation (activation="gelu_tanh") against the oracle's
    tanh form, on the tensor-core and the plain paths."""
    inp = make_shape(T, h, F, "bf16", seed_offset=T + 7)
    gpu = run_gpu(inp, p, activation="gelu_tanh")
    compare_full(gpu, oracle_full(inp, act=1), "bf16")


def test_gelu_tanh_variant_fp32():
    cfg = configs.get("tiny")
    inp = make_inputs(cfg)
    gpu = run_gpu(inp, cfg.p, activation="gelu_tanh")
    compare_full(gpu, oracle_full(inp, act=1), "fp32")


def test_gelu_tanh_variant_7b_sampled():
    """The tanh variant on the 7B-class workload, where the GeLU epilogues use
    the relaying warps (K = 4096)."""
    cfg = configs.get("7b")
    inp = make_inputs(cfg)
    gpu = run_gpu(inp, cfg.p, activation="gelu_tanh")
    R = sample_indices(cfg.T, 32, seed=1234).numpy()
    J = sample_indices(cfg.F, 48, seed=1235).numpy()
    compare_sampled(gpu, inp, R, J, cfg.dtype, act=1)


def test_activation_forms_differ_where_they_should():
    """Exact and tanh forms give different Y (by up to ~5e-4·|x| scale), the
    same shapes, and the backward refuses an unknown activation name."""
    from tensor_transformer_mlp_block_b200 import binding
    inp = make_shape(256, 128, 512, "bf16", seed_offset=3)
    a = run_gpu(inp, 2)
    b = run_gpu(inp, 2, activation="gelu_tanh")
    assert torch.equal(a["H"], b["H"])
    assert not torch.equal(a["Y"], b["Y"])
    d = {k: v.cuda() for k, v in inp.items()}
    with pytest.raises(ValueError):
        binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], 2, activation="relu")


def test_index_space_beyond_2_31_sampled():
    """T·F > 2^31 elements (H, Y, dH of 4.3 GB each): every kernel's row,
    column and tile offsets must be 64-bit. Ragged T and F; checked on seeded
    token rows and hidden columns the oracle computes exactly."""
    from tensor_transformer_mlp_block_b200 import binding
    T, h, F, p = 65576, 64, 33032, 2
    assert T * F > 2 ** 31
    inp = make_shape(T, h, F, "bf16", seed_offset=23)
    d = {k: v.cuda() for k, v in inp.items()}
    H, Y, Z = binding.forward(d["X"], d["A"], d["a"], d["B"], d["b"], p)
    g = binding.backward(d["dZ"], d["X"], d["A"], d["B"], H, Y, p)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    got = dict(H=H, Y=Y, Z=Z, **g)  # stays on the GPU; only sampled slices are copied back
    R = np.concatenate([sample_indices(T, 20, seed=1234).numpy(), [T - 1]])
    J = np.concatenate([sample_indices(F, 40, seed=1235).numpy(), [F - 1]])
    compare_sampled(got, inp, R, J, "bf16")
    del H, Y, Z, g, got
    torch.cuda.empty_cache()


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two GPUs")
def test_tensors_on_a_device_other_than_the_current_one():
    """The binding makes the tensors' device current around each call: a
    block on cuda:1 while cuda:0 is current gives cuda:0's result."""
    inp = make_shape(300, 200, 520, "bf16", seed_offset=31)
    ref = run_gpu(inp, 2, device="cuda:0")
    with torch.cuda.device(0):
        got = run_gpu(inp, 2, device="cuda:1")
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


@pytest.mark.parametrize("policy", [0, 2, 3])
@pytest.mark.parametrize("T,h,F,p", [
    (200, 64, 64, 64),     # p = F: every shard is one hidden column
    (200, 64, 128, 16),    # Fp = 8: shards narrower than one 64-deep k-block
    (130, 16, 24, 24),     # tensor-core path, p = F with a ragged 24-column hidden
    (130, 12, 20, 20),     # plain path (h, F not multiples of 8), p = F
])
def test_degenerate_one_column_shards(T, h, F, p, policy):
    """The finest partitions the method allows give the unsplit result."""
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(policy)
    inp = make_shape(T, h, F, "bf16", seed_offset=T + F + p)
    gpu = run_gpu(inp, p)
    compare_full(gpu, oracle_full(inp), "bf16")


@pytest.mark.parametrize("T", [64, 129, 257, 385])
def test_fused_da_partials_at_tile_edges(T):
    """da summed in the relaying GeLU′ epilogue (h ≥ 3072) when CTA tiles are
    partly or wholly past the last token row: T = 64 (one CTA, the computing
    warps' own rows all past T), 129 and 385 (the pair's second CTA holds one
    valid row), 257."""
    inp = make_shape(T, 3072, 264, "bf16", seed_offset=T + 71)
    gpu = run_gpu(inp, 2)
    compare_full(gpu, oracle_full(inp), "bf16")


@pytest.mark.parametrize("T,h,F,p", [
    (600, 3072, 1536, 2),  # every product takes the tail; relaying GeLU / GeLU′ epilogues, da partials
    (600, 512, 4096, 4),   # row products with the relaying bias epilogue (K = 4096)
    (100, 3072, 8192, 2),  # one-CTA kernel (T ≤ 128): 148 workers, ragged rows
    (1000, 1000, 2000, 2), # ragged M, N and K in the split tiles
])
def test_streamk_tail_full_oracle(T, h, F, p):
    """Policy 3 (stream-K tail wherever valid): tiles split over CTA pairs at
    arbitrary k-blocks, partials summed by the last unit to finish, against
    the full oracle; two runs are bit-identical."""
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(3)
    kinds = binding.plan_schedules(T, h, F, p)
    assert binding.SCHED_STREAMK in kinds.values(), kinds
    inp = make_shape(T, h, F, "bf16", seed_offset=T + h + 5)
    a = run_gpu(inp, p)
    compare_full(a, oracle_full(inp), "bf16")
    b = run_gpu(inp, p)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_streamk_tail_175b_row_products_sampled():
    """The 175B-class workload as the automatic plan runs it (row-parallel
    products on the stream-K tail) against the oracle on 48 seeded rows and
    64 columns."""
    from tensor_transformer_mlp_block_b200 import binding
    cfg = configs.get("175b")
    kinds = binding.plan_schedules(cfg.T, cfg.h, cfg.F, cfg.p)
    assert kinds["F2"] == kinds["B5"] == binding.SCHED_STREAMK, kinds
    inp = make_inputs(cfg)
    gpu = run_gpu(inp, cfg.p, keep_on_device=True)
    R = sample_indices(cfg.T, 48, seed=4321).numpy()
    J = sample_indices(cfg.F, 64, seed=4322).numpy()
    compare_sampled(gpu, inp, R, J, cfg.dtype)
