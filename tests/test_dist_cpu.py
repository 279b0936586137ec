"""The bench's N > 1 host logic on CPU: two gloo ranks, spawned processes.

With N GPUs the bench runs N independent replicas of the block (no data-path
collective); the process group carries only the barrier and the reductions
of the timings. Here two CPU ranks check those reductions, the whole-job
aggregation (all ranks' flops ÷ the slowest rank's time) and that only rank 0
runs the reference arm.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    try:
        w, r, lr = bench.dist_env()
        bench.dist_init(w, "gloo")
        seconds = 1.0 + rank  # rank 1 is the slowest
        mx = bench.max_over_ranks(seconds)
        sm = bench.sum_over_ranks(seconds)
        bench.barrier()
        agg = bench.aggregate(2.0e12, 10, mx, w)
        args = bench.parse_args(["--impl", "reference", "--steps", "3", "--warmup", "3"])
        from tensor_transformer_mlp_block_b200 import configs
        ref = bench.bench_reference(args, configs.get("tiny"), w, r) if r != 0 else "skip"
        q.put((rank, (w, r, lr), mx, sm, agg, ref))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_timing_reductions_and_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(2):
        rank, env, mx, sm, agg, ref = q.get(timeout=120)
        results[rank] = (env, mx, sm, agg, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (env, mx, sm, agg, ref) in results.items():
        assert env == (2, rank, rank)
        assert mx == 2.0 and sm == 3.0
        # 2 ranks × 10 steps × 2 TFLOP in 2 s (the slowest rank) = 20 TFLOP/s
        assert agg["value"] == pytest.approx(20.0)
        assert agg["ms_per_step"] == pytest.approx(200.0)
        if rank != 0:
            assert ref is None  # only rank 0 runs and prints the reference arm


def test_single_process_reductions_are_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.sum_over_ranks(3.5) == 3.5
    assert bench.aggregate(1e12, 4, 2.0, 1) == {"value": 2.0, "ms_per_step": 500.0}


def test_reference_arm_tiny_runs_on_cpu():
    """The reference arm (the fp64 oracle on the host) prints the bench's
    JSON fields for the fp32 toy workload."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from tensor_transformer_mlp_block_b200 import configs
    args = bench.parse_args(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    line = bench.bench_reference(args, configs.get("tiny"), 1, 0)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] >= 1
