"""B200-native tensor-parallel Transformer MLP block.

Z = GeLU(X·A + a)·B + b with A split by columns and B by rows into p shards,
forward and backward, on one GPU (page "Megatron", zzmblog.top, section
"张量并行 / 数学原理"). The compute runs in the CUDA library ``libtpmlp.so``
(hand-written sm_100a kernels behind a C ABI); this package is its thin
Python binding plus the workload presets and seeded input generators.
"""
from .configs import CONFIGS, MLPConfig, get  # noqa: F401

__version__ = "0.1.0"


def __getattr__(name):
    # The binding loads libtpmlp.so on first use and raises if it is missing;
    # there is no other implementation behind these names.
    if name in ("forward", "backward", "lib", "workspace_size", "set_split_policy",
                "last_device_status", "TPMLPError", "launch_count"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
