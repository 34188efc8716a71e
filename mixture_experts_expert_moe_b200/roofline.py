"""Work and traffic accounting for the MoE layer forward (no compute).

Conventions follow the aiter a8w8 issue ("[Feature]: Add more configuration
options for MoE assembly kernels", "Estimated Performance Scaling" table):
the FLOP count of an expert FFN pass is ``pairs * 6 * H * I`` (gate, up and
down projections, 2 FLOPs per multiply-add; padding and the router
excluded), and its I/O is dominated by the expert weights it streams.
"""
from __future__ import annotations


def moe_flops(pairs: int, H: int, I: int) -> float:
    """FLOPs of the gated expert FFN over ``pairs`` (token, expert) pairs."""
    return 6.0 * pairs * H * I


def expert_weight_bytes(H: int, I: int, a8w8: bool) -> int:
    """Bytes of one expert's gate, up and down weights (+ fp32 channel scales)."""
    if a8w8:
        return 3 * H * I + 4 * (2 * I + H)
    return 2 * 3 * H * I


def tile_io_bytes(experts: int, m_tiles_per_expert: int, H: int, I: int,
                  elem_bytes: int = 1) -> int:
    """Weight traffic when every M tile of an expert re-streams its weights."""
    return experts * m_tiles_per_expert * 3 * H * I * elem_bytes


def layer_bytes(T: int, H: int, E: int, k: int, touched: int, I: int,
                a8w8: bool, out_bytes: int = 2) -> int:
    """Algorithmic bytes of one layer forward: touched experts' weights once,
    x read once, out written once, logits read, ids + weights written."""
    return (touched * expert_weight_bytes(H, I, a8w8) + T * H * 2 + T * H * out_bytes
            + T * E * 4 + T * k * 8)


def align_bytes(n_slots: int, num_post: int, block_size: int) -> int:
    """Algorithmic bytes of MoE Align & Sort: ids read once; sorted ids,
    per-block expert ids and the padded total written once."""
    return 4 * n_slots + 4 * num_post + 4 * (num_post // block_size) + 4


def gateup_kernel_bytes(T: int, H: int, I: int, touched: int, pairs: int, a8w8: bool) -> int:
    """Algorithmic bytes of the gate/up GEMM launch: the touched experts' gate
    and up weights once (+ fp32 channel scales in a8w8), the tokens' x once
    (at the operand precision) and the routing it reads (one sorted slot id
    per pair).  The permuted copy of x, h and padding are not counted."""
    eb = 1 if a8w8 else 2
    w = touched * (2 * I * H * eb + (2 * I * 4 if a8w8 else 0))
    return w + T * H * eb + pairs * 4


def down_kernel_bytes(T: int, H: int, I: int, touched: int, pairs: int, a8w8: bool) -> int:
    """Algorithmic bytes of the down GEMM launch: the touched experts' down
    weights once (+ fp32 channel scales in a8w8), the fp32 token outputs
    written once and the routing it reads (slot id and weight per pair).
    The h operand and padding are not counted."""
    eb = 1 if a8w8 else 2
    w = touched * (H * I * eb + (H * 4 if a8w8 else 0))
    return w + T * H * 4 + pairs * 8
