"""Run one phase of the MLP block (forward or backward) a few times on one
GPU, with only the buffers that phase needs: a small, self-contained command
for a profiler to attach to.

  python -m tensor_transformer_mlp_block_b200.run_phase --config 175b --phase fwd --steps 2
  python -m tensor_transformer_mlp_block_b200.run_phase --config 175b --F 12288 --phase bwd

--F narrows the hidden (FFN) width of a named workload (p stays that of the
workload unless --p is given), so that a backward capture holds a few GB
while its products keep the workload's tile shapes and K depths. Inputs are
the seeded synthetic ones of inputs.make_inputs; H and Y for the backward
come from one forward. Prints one line with the phase's time per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import json

import torch

from . import binding, configs
from .inputs import make_inputs, torch_dtype


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--config", default="175b")
    ap.add_argument("--F", type=int, default=None, help="hidden (FFN) width instead of the workload's")
    ap.add_argument("--p", type=int, default=None, help="shard count instead of the workload's")
    ap.add_argument("--phase", choices=["fwd", "bwd"], default="fwd")
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--split-policy", type=int, choices=[0, 1, 2, 3], default=0)
    args = ap.parse_args(argv)

    cfg = configs.get(args.config)
    if args.F is not None or args.p is not None:
        cfg = dataclasses.replace(cfg, F=args.F or cfg.F, p=args.p or cfg.p,
                                  name=f"{cfg.name}-F{args.F or cfg.F}-p{args.p or cfg.p}")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    binding.set_split_policy(args.split_policy)
    inp = make_inputs(cfg)
    T, h, F, p = cfg.T, cfg.h, cfg.F, cfg.p
    dt = torch_dtype(cfg.dtype)
    X, A, a, B, b = (inp[k].to(dev) for k in ("X", "A", "a", "B", "b"))
    ws = torch.empty(max(binding.workspace_size(T, h, F, p, dt), 1), dtype=torch.uint8, device=dev)
    H = torch.empty((T, F), dtype=dt, device=dev)
    Y = torch.empty((T, F), dtype=dt, device=dev)
    if args.phase == "fwd":
        Z = torch.empty((T, h), dtype=dt, device=dev)

        def run():
            binding.forward(X, A, a, B, b, p, out=(H, Y, Z), workspace=ws)
    else:
        Z = torch.empty((T, h), dtype=dt, device=dev)
        binding.forward(X, A, a, B, b, p, out=(H, Y, Z), workspace=ws)
        del Z
        dZ = inp["dZ"].to(dev)
        f32 = torch.float32
        g = dict(dX=torch.empty((T, h), dtype=dt, device=dev),
                 dA=torch.empty((h, F), dtype=f32, device=dev),
                 da=torch.empty((F,), dtype=f32, device=dev),
                 dB=torch.empty((F, h), dtype=f32, device=dev),
                 db=torch.empty((h,), dtype=f32, device=dev),
                 dH=torch.empty((T, F), dtype=dt, device=dev))

        def run():
            binding.backward(dZ, X, A, B, H, Y, p, out=g, workspace=ws)

    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    status = binding.last_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    flops = (4.0 if args.phase == "fwd" else 8.0) * T * h * F
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"workload": cfg.name, "T": T, "h": h, "F": F, "p": p, "phase": args.phase,
                      "ms_per_step": ms, "tflops": flops / ms / 1e9,
                      "schedules": binding.plan_schedules(T, h, F, p, dt),
                      "dynamic": binding.plan_dynamic(T, h, F, p, dt),
                      "device_bytes": torch.cuda.max_memory_allocated(dev)}))


if __name__ == "__main__":
    main()
