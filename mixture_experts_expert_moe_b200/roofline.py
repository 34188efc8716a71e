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


def expert_weight_bytes(H: int, I: int, a8w8: bool, mx: str = "") -> int:
    """Bytes of one expert's gate, up and down weights: bf16; E4M3 + fp32
    channel scales (a8w8); or MX codes (1 byte, or half a byte for E2M1) + one
    E8M0 byte per 32 elements."""
    if mx:
        return 3 * H * I // (1 if mx == "mxfp8" else 2) + 3 * H * I // 32
    if a8w8:
        return 3 * H * I + 4 * (2 * I + H)
    return 2 * 3 * H * I


def tile_io_bytes(experts: int, m_tiles_per_expert: int, H: int, I: int,
                  elem_bytes: int = 1) -> int:
    """Weight traffic when every M tile of an expert re-streams its weights."""
    return experts * m_tiles_per_expert * 3 * H * I * elem_bytes


def layer_bytes(T: int, H: int, E: int, k: int, touched: int, I: int,
                a8w8: bool, out_bytes: int = 2, mx: str = "") -> int:
    """Algorithmic bytes of one layer forward: touched experts' weights once,
    x read once, out written once, logits read, ids + weights written."""
    return (touched * expert_weight_bytes(H, I, a8w8, mx) + T * H * 2 + T * H * out_bytes
            + T * E * 4 + T * k * 8)


def align_bytes(n_slots: int, num_post: int, block_size: int) -> int:
    """Algorithmic bytes of MoE Align & Sort: ids read once; sorted ids,
    per-block expert ids and the padded total written once."""
    return 4 * n_slots + 4 * num_post + 4 * (num_post // block_size) + 4


def _weight_matrix_bytes(rows: int, K: int, a8w8: bool, mx: str) -> int:
    """Bytes of a [rows, K] weight matrix with its scales."""
    if mx:
        return rows * K // (1 if mx == "mxfp8" else 2) + rows * K // 32
    if a8w8:
        return rows * K + rows * 4
    return rows * K * 2


def gateup_kernel_bytes(T: int, H: int, I: int, touched: int, pairs: int, a8w8: bool, mx: str = "") -> int:
    """Algorithmic bytes of the gate/up GEMM launch: the touched experts' gate
    and up weights once (+ their scales), the tokens' x once (at the operand
    precision, one byte for FP8 and MX) and the routing it reads (one sorted
    slot id per pair).  The permuted copy of x, h and padding are not
    counted."""
    eb = 1 if (a8w8 or mx) else 2
    return touched * _weight_matrix_bytes(2 * I, H, a8w8, mx) + T * H * eb + pairs * 4


def down_kernel_bytes(T: int, H: int, I: int, touched: int, pairs: int, a8w8: bool, mx: str = "") -> int:
    """Algorithmic bytes of the down GEMM launch: the touched experts' down
    weights once (+ their scales), the fp32 token outputs written once and the
    routing it reads (slot id and weight per pair).  The h operand and
    padding are not counted."""
    return touched * _weight_matrix_bytes(H, I, a8w8, mx) + T * H * 4 + pairs * 8


def backward_flops(pairs: int, H: int, I: int) -> float:
    """FLOPs of the expert FFN's backward with the gate/up projection
    recomputed: z = Wd^T dout (2 pairs H I), gate/up again (4), dx (4), dW2
    (2) and dW13 (4) -> 16 pairs H I."""
    return 16.0 * pairs * H * I


def backward_bytes(T: int, H: int, I: int, E_all: int, touched: int, E_logits: int) -> int:
    """Algorithmic bytes of moe_backward (bf16 weights): the touched experts'
    gate/up weights read twice (recomputation, dx) and down weights once; the
    fp32 weight gradients of every expert written once; x and dout read once
    (bf16), dx written once (fp32), logits read and their gradient written."""
    return (touched * (2 * (2 * I * H * 2) + H * I * 2) + E_all * 3 * H * I * 4
            + 2 * T * H * 2 + T * H * 4 + 2 * T * E_logits * 4)
