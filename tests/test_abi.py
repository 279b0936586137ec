"""The C ABI on the host: the library builds, loads and exports every entry
point include/tpmlp.h declares; argument errors are reported before any
launch (no GPU needed for these)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tpmlp.h")


@pytest.fixture(scope="module")
def lib():
    from tensor_transformer_mlp_block_b200 import binding, build
    build.build()
    return binding.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)
    return sorted({n for n in names if n.startswith(("tp_", "tpmlp_"))})


def test_header_declares_expected_entry_points():
    from tensor_transformer_mlp_block_b200 import binding
    assert _declared_functions() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    from tensor_transformer_mlp_block_b200 import build
    for name in _declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "tpmlp.h"\nint main(void){ return (int)TPMLP_OK; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-c", str(src), "-o", str(tmp_path / "t.o")], check=True)


def test_strerror_covers_every_status(lib):
    from tensor_transformer_mlp_block_b200 import binding
    seen = set()
    for s in range(7):
        msg = binding.strerror(s)
        assert msg and msg != "unknown status"
        seen.add(msg)
    assert len(seen) == 7
    assert binding.strerror(99) == "unknown status"


def test_version(lib):
    assert lib.tpmlp_version() >= 100


def test_invalid_arguments_fail_before_any_launch(lib):
    from tensor_transformer_mlp_block_b200 import binding
    before = binding.launch_count()
    vp = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    cases = [
        dict(T=8, h=8, F=16, p=0, dt=binding.BF16),   # p < 1
        dict(T=8, h=8, F=16, p=3, dt=binding.BF16),   # F % p != 0
        dict(T=-1, h=8, F=16, p=2, dt=binding.BF16),  # negative T
        dict(T=8, h=0, F=16, p=2, dt=binding.BF16),   # h < 1
        dict(T=8, h=8, F=16, p=2, dt=7),              # dtype code
    ]
    for c in cases:
        st = lib.tp_mlp_fwd(vp, vp, None, vp, None, vp, vp, vp, c["T"], c["h"], c["F"], c["p"],
                            c["dt"], None, 0, None)
        assert st == binding.ERR_INVALID, c
        st = lib.tp_mlp_bwd(vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, c["T"], c["h"], c["F"],
                            c["p"], c["dt"], None, 0, None)
        assert st == binding.ERR_INVALID, c
    assert binding.launch_count() == before


def test_workspace_size_host_logic(lib):
    from tensor_transformer_mlp_block_b200 import binding
    assert binding.workspace_size(8, 8, 16, 3) == 0  # invalid -> 0
    binding.set_split_policy(1)
    base = binding.workspace_size(1024, 512, 2048, 4)
    binding.set_split_policy(2)
    split = binding.workspace_size(1024, 512, 2048, 4)
    binding.set_split_policy(0)
    # one unit per shard and tile adds p fp32 partial tiles per output tile
    assert split - base >= 4 * 1024 * 512 * 4
    assert base % 256 == 0 and split % 256 == 0
    with pytest.raises(binding.TPMLPError):
        binding.set_split_policy(4)


def _r256(x):
    return (x + 255) // 256 * 256


# column sums of the bias gradients: ⌈T/128⌉·h for db; 2·⌈T/128⌉·F for da on
# the tensor-core path (two partial rows per 128-row tile), ⌈T/128⌉·F on the
# plain path
def _colsums(T, h, F, tc=True):
    c = -(-T // 128) if T > 0 else 1
    return _r256(4 * c * h) + _r256(4 * (2 * c if tc else c) * F)


def test_workspace_size_formula(lib):
    """The workspace holds, each part rounded up to 256 bytes: the fp32 partial
    tiles and the arrival counters of split tiles (none with whole tiles
    only), then the bias gradients' column-sum partials."""
    import torch
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(1)
    binding.set_dynamic_schedule(False)
    try:
        for T, h, F, p in [(8192, 4096, 16384, 2), (300, 200, 520, 2), (1, 8, 8, 1), (129, 64, 264, 3)]:
            assert binding.workspace_size(T, h, F, p) == _colsums(T, h, F), (T, h, F)
        assert binding.workspace_size(37, 12, 44, 2) == _colsums(37, 12, 44, tc=False)  # plain path
        assert binding.workspace_size(512, 12, 48, 2, torch.float32) == _r256(16 * 12) + _r256(16 * 48)
        assert binding.workspace_size(0, 12, 44, 2) == _r256(4 * 12) + _r256(4 * 44)
        # the 7B-class step: 9 MiB
        assert binding.workspace_size(8192, 4096, 16384, 2) == 9 * 2 ** 20
        # one unit per shard and tile: 2 × 2 pair tiles of 256 × 256 fp32, p of
        # each; 16 int counters per tile
        binding.set_split_policy(2)
        T, h, F, p = 384, 320, 1024, 4
        tiles = 2 * 2
        assert binding.workspace_size(T, h, F, p) == (_r256(tiles * p * 256 * 256 * 4)
                                                      + _r256(tiles * 16 * 4) + _colsums(T, h, F))
        # stream-K tail everywhere valid: two partial tiles and 16 counters per
        # worker (74 CTA pairs of a 148-SM GPU); at 384 × 320 × 1024 no product
        # has the 4 k-blocks per pair a tail needs
        binding.set_split_policy(3)
        assert binding.workspace_size(T, h, F, p) == _colsums(T, h, F)
        T, h, F, p = 2048, 1024, 4096, 4
        assert binding.plan_schedules(T, h, F, p)["F1"] == binding.SCHED_STREAMK
        assert binding.workspace_size(T, h, F, p) == (_r256(2 * 74 * 256 * 256 * 4)
                                                      + _r256(74 * 16 * 4) + _colsums(T, h, F))
        # the dynamic schedule, when on, adds its two int counters after the
        # split counters for bf16-output products of ≥ 4 waves on CTA pairs,
        # ≥ 192 k-blocks per tile and ≥ 3072 per pair (here Y·B and dH·Aᵀ,
        # K = F = 32768: 512 tiles × 512 k-blocks over 74 pairs)
        binding.set_split_policy(1)
        binding.set_dynamic_schedule(True)
        assert binding.workspace_size(8192, 4096, 32768, 2) == _colsums(8192, 4096, 32768) + 256
        assert binding.workspace_size(8192, 4096, 16384, 2) == 9 * 2 ** 20  # 1771 per pair
        assert binding.workspace_size(4096, 768, 3072, 2) == _colsums(4096, 768, 3072)  # < 4 waves
        # only the weight gradients (fp32 outputs; K = T = 24576, 18 × 18
        # tiles each) would qualify here: they always run statically
        assert binding.workspace_size(24576, 4608, 4608, 1) == _colsums(24576, 4608, 4608)
        # X·A and dZ·Bᵀ with 192 k-blocks per tile and 32 × 16 tiles (6.9
        # waves), but 1328 k-blocks per pair: static
        assert binding.workspace_size(8192, 12288, 4096, 2) == _colsums(8192, 12288, 4096)
    finally:
        binding.set_split_policy(0)
        binding.set_dynamic_schedule(True)


def test_dynamic_schedule_default(lib):
    """On by default, for the longest products only: the 7B-class step (~1770
    k-blocks per CTA pair) reserves no dynamic counters, a step with K = F =
    32768 (~3540 per pair) does, and switching it off drops them."""
    from tensor_transformer_mlp_block_b200 import binding
    assert binding.get_dynamic_schedule()
    binding.set_split_policy(1)
    try:
        on_7b = binding.workspace_size(8192, 4096, 16384, 2)
        on_long = binding.workspace_size(8192, 4096, 32768, 2)
        binding.set_dynamic_schedule(False)
        assert not binding.get_dynamic_schedule()
        assert binding.workspace_size(8192, 4096, 16384, 2) == on_7b
        assert on_long - binding.workspace_size(8192, 4096, 32768, 2) == 256
    finally:
        binding.set_dynamic_schedule(True)
        binding.set_split_policy(0)


def test_automatic_schedules_for_the_named_workloads(lib):
    """The automatic policy keeps whole tiles where the last wave of 74 CTA
    pairs is nearly full (every 7B-class product) or the tail would save less
    than its own cost (GPT-2-small, 350M), and takes the stream-K tail for the
    175B-class row-parallel products (8 × 48 pair tiles = 5.19 waves of
    768 k-blocks). (Without a GPU the planner assumes 148 SMs.)"""
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(0)
    TILES, SK = binding.SCHED_TILES, binding.SCHED_STREAMK
    assert set(binding.plan_schedules(8192, 4096, 16384, 2).values()) == {TILES}
    assert binding.plan_schedules(2048, 12288, 49152, 8) == dict(F1=TILES, F2=SK, B2=TILES, B3=TILES,
                                                                 B4=TILES, B5=SK)
    assert set(binding.plan_schedules(4096, 768, 3072, 2).values()) == {TILES}
    assert set(binding.plan_schedules(6144, 1024, 4096, 4).values()) == {TILES}
    # policy 1: whole tiles everywhere; policy 2: shard groups for the row products
    binding.set_split_policy(1)
    assert set(binding.plan_schedules(2048, 12288, 49152, 8).values()) == {TILES}
    binding.set_split_policy(2)
    k = binding.plan_schedules(2048, 12288, 49152, 8)
    assert k["F2"] == k["B5"] == binding.SCHED_GROUPS and k["F1"] == TILES
    binding.set_split_policy(0)


def test_dynamic_products_of_the_named_workloads(lib):
    """The dynamic schedule (on by default) takes the four 175B-class row
    products (~3990 k-blocks per CTA pair each: 1536 tiles of 192 k-blocks,
    or 384 tiles of 768) and nothing of the smaller workloads (7B-class Y·B
    and dH·Aᵀ: 512 tiles of 256 k-blocks, ~1770 per pair); never the fp32
    weight gradients; nothing with it switched off."""
    import torch
    from tensor_transformer_mlp_block_b200 import binding
    binding.set_split_policy(0)
    assert binding.plan_dynamic(2048, 12288, 49152, 8) == dict(F1=True, F2=True, B2=True, B3=False,
                                                               B4=False, B5=True)
    for T, h, F, p in [(8192, 4096, 16384, 2), (4096, 768, 3072, 2), (6144, 1024, 4096, 4)]:
        assert not any(binding.plan_dynamic(T, h, F, p).values()), (T, h, F, p)
    assert not any(binding.plan_dynamic(512, 12, 48, 2, torch.float32).values())
    binding.set_split_policy(2)  # shard groups: the same work per pair, cut finer
    assert binding.plan_dynamic(2048, 12288, 49152, 8)["F2"]
    binding.set_split_policy(0)
    binding.set_dynamic_schedule(False)
    try:
        assert not any(binding.plan_dynamic(2048, 12288, 49152, 8).values())
    finally:
        binding.set_dynamic_schedule(True)


def test_product_path_refuses_cpu_tensors():
    import torch
    from tensor_transformer_mlp_block_b200 import binding
    X = torch.zeros(4, 8, dtype=torch.bfloat16)
    A = torch.zeros(8, 16, dtype=torch.bfloat16)
    B = torch.zeros(16, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.forward(X, A, None, B, None, 2)
