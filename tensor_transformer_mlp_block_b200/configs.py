"""Workload presets for the MLP block: shapes, shard counts and input scales.

T = tokens (micro-batch × sequence length), h = hidden size, F = FFN size
(4h for the pages' MLP: A ∈ R^{h×4h}, B ∈ R^{4h×h}, page "Megatron",
section "张量并行 / 数学原理"), p = tensor-parallel degree (number of shards).

Sources of the shapes:
- tiny: hidden_size 12 with fp32 and CPU initialisation, sequence 64
  (page "最完整的Megatron-LM技术文档体系：从安装到训练的全流程指南", §3.2 and §3.3),
  micro-batch 8, F = 4h, p = 2.
- gpt2-small: hidden 768, ffn 3072 (page "Megatron", section
  "实战使用 / 基础训练示例"), micro-batch 4 × sequence 1024 with TP 2
  (page "保姆级教程：用Megatron-LM在单机多卡上跑通你的第一个LLM分布式训练", §3.2).
- 350m: TP 4 and micro-batch 6 from the 8×A100 case study of the same
  tutorial page (§7); h = 1024 and sequence 1024 are this library's reading.
- 7b, 175b: the TP degrees 2 and 8 from the 3D-parallelism table (page
  "Megatron", section "3D并行"); the hidden sizes 4096 / 12288 are the usual
  sizes of those model classes, not numbers on the pages.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class MLPConfig:
    name: str
    T: int
    h: int
    F: int
    p: int
    dtype: str  # "fp32" or "bf16"
    std_X: float
    std_A: float
    std_B: float
    std_a: float  # 0.0 = zero bias
    std_b: float
    std_dZ: float = 1.0

    @property
    def flops_fwd_bwd(self) -> float:
        """Algorithmic GEMM flops of one forward + backward: six T·h·F
        products (two forward, four backward), 2 flops per multiply-add."""
        return 12.0 * self.T * self.h * self.F

    @property
    def flops_fwd(self) -> float:
        return 4.0 * self.T * self.h * self.F


CONFIGS = {
    "tiny": MLPConfig("tiny", 512, 12, 48, 2, "fp32", 1.0, 0.02, 0.02, 0.01, 0.01),
    "gpt2-small": MLPConfig("gpt2-small", 4096, 768, 3072, 2, "bf16", 1.0, 0.02, 0.02, 0.0, 0.0),
    "350m": MLPConfig("350m", 6144, 1024, 4096, 4, "bf16", 1.0, 0.02, 0.02, 0.01, 0.01),
    "7b": MLPConfig("7b", 8192, 4096, 16384, 2, "bf16", 1.0, 0.02, 0.02 / math.sqrt(2 * 32),
                    0.0, 0.0),
    "175b": MLPConfig("175b", 2048, 12288, 49152, 8, "bf16", 1.0, 0.006, 0.006, 0.0, 0.0),
}


def get(name: str) -> MLPConfig:
    try:
        return CONFIGS[name]
    except KeyError:
        raise KeyError(f"unknown config {name!r}; known: {sorted(CONFIGS)}") from None
