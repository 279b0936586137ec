#!/usr/bin/env python
"""Bench of the tensor-parallel MLP block: forward + backward TFLOP/s on B200.

One step = tp_mlp_fwd + tp_mlp_bwd over one batch of seeded synthetic input
(the whole hot path: column GEMM with bias+GeLU, row GEMM with the ordered
shard sum, bias-gradient column sums, dgrad with GeLU′, two weight-gradient
GEMMs, dgrad of X with the ordered shard sum). FLOPs counted = 12·T·h·F per
step (the six T·h·F products); elementwise and reduction work is in the time
but not in the count.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 7b]
  python bench.py --impl reference ...   # the fp64 CPU oracle, bounded sample

With N > 1 (launched by torch.distributed.run) every rank runs an
independent replica of the workload (the block is not sharded across GPUs):
weak scaling, value = all ranks' FLOPs / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TP-MLP fwd+bwd TFLOP/s (bf16, 1 B200) and % of dense BF16 tensor peak"
UNIT = "TFLOP/s"
DATASHEET_BF16_DENSE_TFLOPS = 2250.0  # NVIDIA B200 datasheet (HGX B200), dense BF16
# Used only when the measured peaks of this machine are absent: an earlier
# measurement on the same kind of B200 (copy bandwidth, cuBLAS bf16 burst).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# A timed region at least this long under an active power cap runs in the
# sustained regime; shorter regions run at burst clocks.
SUSTAINED_MIN_SECONDS = 1.0
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="175b",
                    help="workload preset (default: the largest, 175b; also 7b, 350m, gpt2-small, tiny)")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the end-to-end measurement (default: --steps, so that both "
                         "numbers cover the same sustained power-capped interval)")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step in a CUDA graph and time its replays")
    ap.add_argument("--activation", choices=["gelu", "gelu_tanh"], default="gelu",
                    help="MLP activation: exact GeLU (default) or its tanh approximation")
    ap.add_argument("--launch-overlap", choices=["on", "off"], default="on",
                    help="programmatic dependent launches between the library's kernels")
    ap.add_argument("--recompute", choices=["none", "activation", "hidden"], default="none",
                    help="activation recompute before each backward: rebuild Y from H "
                         "(activation) or H and Y from X (hidden)")
    ap.add_argument("--block", choices=["mlp", "attn-proj"], default="mlp",
                    help="mlp: the MLP block (default); attn-proj: the attention layer's "
                         "tensor-parallel projections (QKV split by columns, output by rows)")
    ap.add_argument("--split-policy", type=int, choices=[0, 1, 2, 3], default=0,
                    help="work schedule of the products (tpmlp_set_split_policy): 0 automatic "
                         "(default), 1 whole tiles only, 2 one unit per shard for the row "
                         "products, 3 stream-K tail wherever valid")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle CPU baseline (for profiler runs)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target seconds of oracle work for the CPU baseline sample")
    args = ap.parse_args(argv)
    if args.e2e_steps is None:
        args.e2e_steps = args.steps
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    return args


# ----------------------------------------------------------- distributed glue

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def aggregate(flops_per_step_per_rank: float, steps: int, max_seconds: float, world: int) -> dict:
    """Whole-job throughput of `world` replicas that each ran `steps` steps,
    timed by the slowest rank."""
    total = flops_per_step_per_rank * steps * world
    return {"value": total / max_seconds / 1e12, "ms_per_step": 1e3 * max_seconds / steps}


# ------------------------------------------------------------------- peaks

def load_peaks():
    """This machine's measured peaks (copy bandwidth, bf16 GEMM burst and, if
    recorded, sustained), else the fallback figures (no sustained one)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        out = {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops")}
        if p.get("bf16_tflops_sustained") is not None:
            out["bf16_tflops_sustained"] = float(p["bf16_tflops_sustained"])
        return out, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def pick_tensor_peak(peaks: dict, src: str, region_s: float, clocks: dict):
    """The bf16 peak that matches the regime of the timed region: the
    sustained figure only for a region of SUSTAINED_MIN_SECONDS or more in
    which the power cap was active, the burst figure otherwise."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    if region_s >= SUSTAINED_MIN_SECONDS and capped and "bf16_tflops_sustained" in peaks:
        return peaks["bf16_tflops_sustained"], (
            f"{src} bf16 sustained: timed region {region_s:.2f} s under sw_power_cap")
    if region_s < SUSTAINED_MIN_SECONDS:
        why = "short"
    elif not capped:
        why = "not power-capped"
    else:
        why = "power-capped, but no sustained figure was measured"
    return peaks["bf16_tflops"], f"{src} bf16 burst: timed region {region_s:.2f} s ({why})"


def source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tensor_transformer_mlp_block_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kind: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources for this workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[workload][kind]
        if e.get("source_hash") != source_hash():
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) < 10:
                    continue
                try:
                    stamp, _, frac = r[0].strip().partition(".")
                    ts = time.mktime(time.strptime(stamp, "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + frac) if frac.isdigit() else 0.0
                    rows.append((ts, [c.strip() for c in r]))
                except Exception:
                    continue
        os.unlink(self.path)
        # samples taken while the timed work ran
        inside = [c for ts, c in rows if t0 <= ts <= t1] or [c for _, c in rows]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(c[2]) for c in inside if c[2].replace(".", "").isdigit()]
        smax = [float(c[3]) for c in inside if c[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for c in inside for i in range(4) if c[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(inside),
                "power_w_max": max((float(c[4]) for c in inside if c[4].replace(".", "").isdigit()),
                                   default=None)}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if local_rank < len(parts) and parts[local_rank].isdigit():
            return int(parts[local_rank])
    return local_rank


# ------------------------------------------------------------ CPU baseline

def cpu_baseline(inp: dict, cfg, target_seconds: float) -> dict:
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    token rows R (forward and dX for those rows) and hidden columns J (H, dH,
    dA, dB for those columns). Rate = the sample's algorithmic flops / wall
    time on this host's cores."""
    import numpy as np

    import oracle
    from tensor_transformer_mlp_block_b200.inputs import sample_indices
    n = {k: v.to(dtype=__import__("torch").float64).numpy() for k, v in inp.items()}

    def run(n_r, n_j):
        R = sample_indices(cfg.T, n_r, seed=1234).numpy()[:n_r]
        J = sample_indices(cfg.F, n_j, seed=1235).numpy()[:n_j]
        t0 = time.perf_counter()
        oracle.rows(n["X"], n["A"], n["a"], n["B"], n["b"], n["dZ"], R)
        oracle.cols(n["X"], n["A"][:, J], n["a"][J], n["B"][J, :], n["dZ"], np.arange(len(J)))
        dt = time.perf_counter() - t0
        flops = 8.0 * cfg.h * cfg.F * len(R) + 8.0 * cfg.T * cfg.h * len(J)
        return dt, flops, len(R), len(J)

    dt, fl, _, _ = run(2, 2)
    rate = fl / max(dt, 1e-9)
    per_unit = 8.0 * cfg.h * cfg.F + 8.0 * cfg.T * cfg.h
    k = max(2, int(target_seconds * rate / per_unit))
    k = min(k, cfg.T, cfg.F)
    dt, fl, nr, nj = run(k, k)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
            "sample": f"{nr} token rows + {nj} hidden columns of the {cfg.name} workload "
                      f"({fl / 1e9:.1f} GFLOP fp64 in {dt:.1f} s)",
            "seconds": dt}


# --------------------------------------------------------------- our arm

def bench_ours(args, cfg, world, rank, local):
    import torch

    from tensor_transformer_mlp_block_b200 import binding
    from tensor_transformer_mlp_block_b200.inputs import make_inputs, torch_dtype

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    peaks, peaks_src = load_peaks()

    inp = make_inputs(cfg)
    d = {k: v.to(dev) for k, v in inp.items()}
    dt = torch_dtype(cfg.dtype)
    T, h, F, p = cfg.T, cfg.h, cfg.F, cfg.p
    f32 = torch.float32
    H = torch.empty((T, F), dtype=dt, device=dev)
    Y = torch.empty((T, F), dtype=dt, device=dev)
    Z = torch.empty((T, h), dtype=dt, device=dev)
    gout = dict(dX=torch.empty((T, h), dtype=dt, device=dev), dA=torch.empty((h, F), dtype=f32, device=dev),
                da=torch.empty((F,), dtype=f32, device=dev), dB=torch.empty((F, h), dtype=f32, device=dev),
                db=torch.empty((h,), dtype=f32, device=dev), dH=torch.empty((T, F), dtype=dt, device=dev))
    binding.set_split_policy(args.split_policy)  # the workspace size depends on it
    ws = torch.empty(max(binding.workspace_size(T, h, F, p, dt), 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    binding.set_launch_overlap(args.launch_overlap == "on")

    act = args.activation

    def step(x=None, dz=None):
        x = d["X"] if x is None else x
        dz = d["dZ"] if dz is None else dz
        binding.forward(x, d["A"], d["a"], d["B"], d["b"], p, out=(H, Y, Z), workspace=ws,
                        activation=act)
        if args.recompute == "activation":
            binding.recompute_activation(H, out=Y, activation=act)
        elif args.recompute == "hidden":
            binding.recompute_hidden(x, d["A"], d["a"], p, out=(H, Y), activation=act)
        binding.backward(dz, x, d["A"], d["B"], H, Y, p, out=gout, workspace=ws, activation=act)

    working_set = sum(t.numel() * t.element_size() for t in [*d.values(), H, Y, Z, *gout.values()])
    flops_per_step = cfg.flops_fwd_bwd
    if args.block == "attn-proj":
        # the attention layer's two tensor-parallel projections at this width:
        # QKV = X·W_qkv (h -> 3h, columns), Z = O·W_o (h -> h, rows), fwd + bwd
        del H, Y, gout
        torch.cuda.empty_cache()
        gen = torch.Generator().manual_seed(21)
        Wqkv = (torch.randn((h, 3 * h), generator=gen) * 0.02).to(dt).to(dev)
        bqkv = torch.zeros((3 * h,), dtype=dt, device=dev)
        Wo = (torch.randn((h, h), generator=gen) * 0.02).to(dt).to(dev)
        bo = torch.zeros((h,), dtype=dt, device=dev)
        O = torch.randn((T, h), generator=gen).to(dt).to(dev)
        dQKV = torch.randn((T, 3 * h), generator=gen).to(dt).to(dev)
        QKV = torch.empty((T, 3 * h), dtype=dt, device=dev)
        g_qkv = (torch.empty((T, h), dtype=dt, device=dev), torch.empty((h, 3 * h), dtype=f32, device=dev),
                 torch.empty((3 * h,), dtype=f32, device=dev))
        g_o = (torch.empty((T, h), dtype=dt, device=dev), torch.empty((h, h), dtype=f32, device=dev),
               torch.empty((h,), dtype=f32, device=dev))
        ws_l = torch.empty(max(binding.linear_workspace_size(T, h, 3 * h, p, "columns", dt),
                               binding.linear_workspace_size(T, h, h, p, "rows", dt), 1),
                           dtype=torch.uint8, device=dev)

        def step(x=None, dz=None):
            x = d["X"] if x is None else x
            dz = d["dZ"] if dz is None else dz
            binding.linear_forward(x, Wqkv, bqkv, p, "columns", out=QKV, workspace=ws_l)
            binding.linear_backward(dQKV, x, Wqkv, p, "columns", out=g_qkv, workspace=ws_l)
            binding.linear_forward(O, Wo, bo, p, "rows", out=Z, workspace=ws_l)
            binding.linear_backward(dz, O, Wo, p, "rows", out=g_o, workspace=ws_l)

        flops_per_step = 24.0 * T * h * h
        working_set = sum(t.numel() * t.element_size()
                          for t in [d["X"], d["dZ"], Wqkv, Wo, O, dQKV, QKV, Z, *g_qkv, *g_o])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    n0 = binding.launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = binding.launch_count() - n0

    run_step = step
    if args.graph:
        # one step captured once; replays re-launch the same kernels
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        run_step = graph.replay

    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    time.sleep(1.0)
    # The step time is taken without per-launch events: an event recorded
    # between two of the library's kernels would stop the second from starting
    # while the first drains (programmatic dependent launch). Per-kernel times
    # come from a second pass right after, with an event pair around every
    # launch, inside the same clock-sampled window.
    binding.profile_enable(False)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    launches = launches_per_step * args.steps
    kernel_pass_steps = min(args.steps, 50)
    binding.profile_reset()
    binding.profile_enable(True)
    for _ in range(kernel_pass_steps):
        step()
    torch.cuda.synchronize()
    binding.profile_enable(False)
    kinds = binding.profile_collect()
    t_wall2 = time.time()
    clocks = sampler.stop(t_wall0, t_wall2)
    status = binding.last_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    seconds = e0.elapsed_time(e1) / 1e3
    max_seconds = max_over_ranks(seconds, dev)
    agg = aggregate(flops_per_step, args.steps, max_seconds, world)

    # Per-kernel times inside the step. The event pass brackets every launch
    # with an event pair, which stops the launch overlap between neighbours,
    # so its durations add up to a little more than the step. Each kernel's
    # in-step time is its event time scaled by (step time / sum of the event
    # times of one step): the shares come from the events, the total from the
    # timed region itself, and the in-step times add up to the step.
    step_ms = 1e3 * seconds / args.steps
    event_step_ms = sum(v["ms"] for v in kinds.values()) / kernel_pass_steps
    scale = step_ms / event_step_ms if event_step_ms > 0 else 1.0
    per_kernel = {}
    for k, v in kinds.items():
        ev_ms = v["ms"] / v["launches"]
        in_ms = ev_ms * scale
        per_kernel[k] = {"launches_per_step": v["launches"] / kernel_pass_steps,
                         "ms_per_launch": in_ms, "event_ms_per_launch": ev_ms,
                         "tflops": (v["flops"] / v["launches"] / in_ms / 1e9) if v["flops"] else None,
                         "gbs": v["bytes"] / v["launches"] / in_ms / 1e6}

    # dominant kernel and its roofline (tensor-bound: algorithmic flops / in-step time)
    tensor_peak, peak_source = pick_tensor_peak(peaks, peaks_src, seconds, clocks)
    top_name, top = max(kinds.items(), key=lambda kv: kv[1]["ms"])
    top_ms = per_kernel[top_name]["ms_per_launch"]
    flops_per_launch = top["flops"] / top["launches"]
    achieved = flops_per_launch / (top_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": top_name, "achieved": achieved, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": achieved / tensor_peak,
                "traffic": traffic_for(top_name, cfg.name),
                "peak_source": peak_source,
                "flops_per_launch": flops_per_launch,
                "launches_per_step": top["launches"] / kernel_pass_steps,
                "ms_per_launch": top_ms,
                "event_ms_per_launch": top["ms"] / top["launches"],
                "share_of_step": top["ms"] / sum(k["ms"] for k in kinds.values()),
                "step_frac": agg["value"] / world / tensor_peak,
                "kernel_timing": f"in-step time = event-pair time x (step time {step_ms:.4f} ms / "
                                 f"event times of one step {event_step_ms:.4f} ms); event pairs around "
                                 f"every launch on its stream over {kernel_pass_steps} eager steps right "
                                 "after the timed steps (events between kernels stop their launch "
                                 "overlap, so they are not recorded inside the timed steps)"}

    if args.block != "mlp":
        e2e = None
    else:
        e2e = e2e_measure(args, cfg, inp, d, H, Y, Z, gout, ws, p, T, h, dt, dev, stream, world, act,
                          binding, torch)

    line = _line(args, cfg, world, agg, peaks, peaks_src, roofline, per_kernel, e2e, launches,
                 clocks, working_set, flops_per_step, T, h, F, p, seconds)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.block == "mlp":
        line["cpu_baseline"] = cpu_baseline(inp, cfg, args.cpu_seconds)
    elif rank == 0:
        line["cpu_baseline"] = None
    return line


def e2e_measure(args, cfg, inp, d, H, Y, Z, gout, ws, p, T, h, dt, dev, stream, world, act,
                binding, torch):
    # End to end through the public API with pinned host buffers: every step
    # copies its X and dZ in from pinned host memory and its Z and dX back
    # out. The copies run on two copy streams, double-buffered, so step i's
    # upload and step i-1's download overlap step i-1's / i's compute, as an
    # input pipeline does; the timed region spans the first upload to the
    # last download.
    hX = inp["X"].pin_memory()
    hdZ = inp["dZ"].pin_memory()
    hZ = torch.empty((T, h), dtype=dt).pin_memory()
    hdX = torch.empty((T, h), dtype=dt).pin_memory()
    xin = [torch.empty_like(d["X"]) for _ in range(2)]
    dzin = [torch.empty_like(d["dZ"]) for _ in range(2)]
    zout = [torch.empty((T, h), dtype=dt, device=dev) for _ in range(2)]
    dxout = [torch.empty((T, h), dtype=dt, device=dev) for _ in range(2)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[b])  # step i-2 has finished reading xin[b]
                xin[b].copy_(hX, non_blocking=True)
                dzin[b].copy_(hdZ, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's outputs are on the host
            binding.forward(xin[b], d["A"], d["a"], d["B"], d["b"], p, out=(H, Y, zout[b]),
                            workspace=ws, activation=act)
            gout["dX"] = dxout[b]
            if args.recompute == "activation":
                binding.recompute_activation(H, out=Y, activation=act)
            elif args.recompute == "hidden":
                binding.recompute_hidden(xin[b], d["A"], d["a"], p, out=(H, Y), activation=act)
            binding.backward(dzin[b], xin[b], d["A"], d["B"], H, Y, p, out=gout, workspace=ws,
                             activation=act)
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                hZ.copy_(zout[b], non_blocking=True)
                hdX.copy_(dxout[b], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_event(ev_out[(n - 1) % 2])
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / 1e3

    e2e_run(4)
    barrier()
    torch.cuda.synchronize()
    e2e_max = max_over_ranks(e2e_run(args.e2e_steps), dev)
    e2e_val = aggregate(cfg.flops_fwd_bwd, args.e2e_steps, e2e_max, world)["value"]
    assert torch.equal(hZ, zout[(args.e2e_steps - 1) % 2].cpu())
    bytes_in = hX.numel() * hX.element_size() + hdZ.numel() * hdZ.element_size()
    bytes_out = hZ.numel() * hZ.element_size() + hdX.numel() * hdX.element_size()
    return {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": bytes_in,
            "d2h_bytes_per_step": bytes_out, "steps": args.e2e_steps,
            "what": "per step: X and dZ copied in from pinned host memory, fwd+bwd through the "
                    "public API, Z and dX copied out to pinned host memory; copies pipelined on "
                    "two copy streams with double-buffered device tensors; weights and weight "
                    "gradients stay resident"}


SCHED_NAMES = {0: "whole tiles", 1: "shard groups", 2: "stream-K tail"}


def plan_summary(T, h, F, p, dtype_name):
    """The work schedule the library plans for each of the six products."""
    from tensor_transformer_mlp_block_b200 import binding
    from tensor_transformer_mlp_block_b200.inputs import torch_dtype
    dt = torch_dtype(dtype_name)
    kinds = binding.plan_schedules(T, h, F, p, dt)
    dyn = binding.plan_dynamic(T, h, F, p, dt)
    return {k: SCHED_NAMES[v] + (", dynamic" if dyn[k] else "") for k, v in kinds.items()}


def _line(args, cfg, world, agg, peaks, peaks_src, roofline, per_kernel, e2e, launches, clocks,
          working_set, flops_per_step, T, h, F, p, seconds):
    workload = f"{cfg.name}-class TP-MLP fwd+bwd"
    if args.block == "attn-proj":
        workload = f"{cfg.name}-class attention projections (QKV columns + output rows) fwd+bwd"
    else:
        if args.activation != "gelu":
            workload += f" ({args.activation})"
        if args.recompute == "activation":
            workload += " with activation recompute (Y from H)"
        elif args.recompute == "hidden":
            workload += " with activation recompute (H and Y from X)"
    metric = METRIC if args.block == "mlp" else \
        "TP attention projections fwd+bwd TFLOP/s (bf16, 1 B200) and % of dense BF16 tensor peak"
    return {
        "metric": metric, "value": agg["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": agg["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "fp32",
        "data": "synthetic (seeded Gaussian inputs, random-init weights of the named shapes)",
        "config": {"workload": workload, "T": T, "h": h, "F": F, "p": p,
                   "flops_per_step": flops_per_step, "parallelism": f"replicas x{world}",
                   "cuda_graph": bool(args.graph), "activation": args.activation,
                   "launch_overlap": args.launch_overlap == "on",
                   "split_policy": args.split_policy,
                   "schedules": plan_summary(T, h, F, p, cfg.dtype) if args.block == "mlp" else None,
                   "l2": f"working set {working_set / 2**30:.2f} GiB > L2 {L2_BYTES / 2**20:.0f} MiB "
                         "(inputs larger than L2; no flush)"},
        "frac_of_peak": {"measured_burst": agg["value"] / world / peaks["bf16_tflops"],
                         "measured_sustained": (agg["value"] / world / peaks["bf16_tflops_sustained"]
                                                if "bf16_tflops_sustained" in peaks else None),
                         "datasheet_dense": agg["value"] / world / DATASHEET_BF16_DENSE_TFLOPS,
                         "peaks": peaks_src, "timed_region_s": seconds},
        "roofline": roofline,
        "kernels": per_kernel,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }


# ---------------------------------------------------------- reference arm

def bench_reference(args, cfg, world, rank):
    """The fp64 oracle on the host cores: each step is a bounded sample of the
    workload (token rows + hidden columns), so K + W steps end in minutes."""
    if rank != 0:
        return None
    from tensor_transformer_mlp_block_b200.inputs import make_inputs
    inp = make_inputs(cfg)
    per_step = max(0.2, min(10.0, 120.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(inp, cfg, per_step)
    total_flops, total_s, last = 0.0, 0.0, None
    for _ in range(args.steps):
        last = cpu_baseline(inp, cfg, per_step)
        total_s += last["seconds"]
        total_flops += last["value"] * 1e12 * last["seconds"]
    value = total_flops / total_s / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian inputs)",
        "config": {"workload": f"{cfg.name}-class TP-MLP fwd+bwd", "T": cfg.T, "h": cfg.h,
                   "F": cfg.F, "p": cfg.p},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                         "sample": "per step: " + last["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    from tensor_transformer_mlp_block_b200 import configs
    cfg = configs.get(args.config)
    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        line = bench_reference(args, cfg, world, rank)
    else:
        line = bench_ours(args, cfg, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
