"""Oracle for the tensor-parallel Transformer MLP block — TEST INFRASTRUCTURE.

A plain, slow, obviously correct fp64 CPU implementation of the block
Z = GeLU(X·A + a)·B + b and of its gradients, written from page "Megatron"
(zzmblog.top), section "张量并行 / 数学原理" (column split of A, row split of B,
and the all-reduce that sums the row-parallel partials), plus the chain rule.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package. The CUDA library never calls it, and the two
share no code: the oracle is C (``tpmlp_oracle.c``, gcc) behind ctypes, plus a
pure-Python brute-force checker (``bruteforce.py``) for tiny shapes.

Pins (in ``tests/test_oracle_pins.py``): brute force on tiny shapes, central
finite differences of L = Σ dZ⊙Z, the pages' two partition identities for
every p dividing F, textbook values of the normal distribution function,
a hand-worked example, special cases (A = 0, B = 0, bias linearity) and a
float64 torch CPU cross-check. No function here is left unpinned.
"""
from .oracle import (  # noqa: F401
    Oracle,
    compile_variant,
    default,
    source_text,
    backward,
    backward_sharded,
    build,
    cols,
    colsum,
    forward,
    forward_sharded,
    gelu,
    gelu_grad,
    gelu_tanh,
    gelu_tanh_grad,
    get_threads,
    linear_backward,
    linear_backward_sharded,
    linear_forward,
    linear_forward_sharded,
    normal_cdf,
    normal_pdf,
    rows,
    set_threads,
)
