"""CPU oracle for the single-GPU MoE layer forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The CUDA library never calls it and has no CPU fallback.

The oracle shares no code with the CUDA path: no kernels, headers, helpers,
tables or pre/post-processing.  Its only shared dependency is the seeded
input generator package ``moe_inputs``, which holds none of the method's
arithmetic.

Every function is pinned by ``tests/test_oracle_*.py`` against brute force,
closed forms, library routines and the figures the pages print.  See the
module docstrings of :mod:`oracle.moe_oracle` (the layer forward) and
:mod:`oracle.mx_oracle` (MX block-scaled operands, the next FFN variant) and
:mod:`oracle.backward_oracle` (the layer's backward pass) for the lists of
pins.
"""
from .moe_oracle import (  # noqa: F401
    bf16_round,
    e4m3_decode,
    e4m3_encode,
    e4m3_values,
    topk_gate,
    add_shared,
    align_sort,
    quant_rows_e4m3,
    ffn_bf16,
    ffn_a8w8,
    combine,
    moe_forward,
    expected_sizes,
)
