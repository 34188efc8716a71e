"""CPU oracle for MX block-scaled operands (the next FFN variant after the
per-token FP8 one).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing in the CUDA
library imports, links or runs this file.

Source: the GC-MoE abstract (zhuanzhiai.com) describes block-scaled,
operand-swapped tensor-core MMAs for Blackwell MoE decode, with FP4 weights.
The pages do not define the formats, so the OCP Microscaling (MX)
specification's formats are used:

* an MX block is 32 consecutive elements along the reduction dimension K that
  share one scale X = 2^s, stored as an E8M0 code (s = code - 127; code 255
  is NaN);
* elements are FP8 E4M3 (MXFP8; the OCP E4M3FN codec of ``moe_oracle``) or
  FP4 E2M1 (MXFP4: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit;
  values 0, 0.5, 1, 1.5, 2, 3, 4, 6; no inf or NaN);
* quantisation of a block: s = floor(log2(amax)) - emax, where emax is the
  exponent of the element format's largest normal (8 for E4M3: 448 = 1.75 *
  2^8; 2 for E2M1: 6 = 1.5 * 2^2), clamped to [-127, 127]; each element is
  v / X rounded to the nearest element value, ties to even, and saturated to
  the format's largest magnitude.

Readings (listed with the design notes):

1. A block whose elements are all zero gets scale code 127 (X = 1) and zero
   codes (the specification leaves X free there).
2. The MX FFN quantises the activations (x, then h after SwiGLU) to MXFP8
   along K, per token row, and takes weights in MXFP4 or MXFP8 along K;
   each GEMM is the sum over blocks of X_a * X_w * (sum of the decoded
   element products), accumulated here in float64.
3. h is rounded to bf16 before its quantisation, as in the per-token FP8
   path.

Pins (tests/test_oracle_mx.py): the E2M1 value table of the format; round
trip of every code; brute-force nearest value with ties to the even code at
every midpoint; saturation; E8M0 special codes; MX quantisation of blocks
built as exact element values times a power of two reconstructs them and
their scale exactly; the block's largest magnitude lands in the element
format's top binade (or saturates at its largest value); zero blocks; MXFP8
elements equal torch's float8_e4m3fn cast of v / X; the block-sum GEMM
equals a library matmul of the decoded operands; an MX FFN whose experts are
identical equals a dense SwiGLU FFN computed with library matmuls on the
same quantised operands.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import _silu, add_shared, bf16_round, combine, e4m3_decode, e4m3_encode, topk_gate

MX_BLOCK = 32

# ---------------------------------------------------------------------------
# E2M1 (FP4) and E8M0 codecs
# ---------------------------------------------------------------------------


def _e2m1_formula(c) -> np.ndarray:
    """Value of E2M1 codes (low 4 bits): sign bit 3, exponent bits 2..1
    (bias 1), mantissa bit 0; exponent 0 is subnormal (0 or 0.5)."""
    c = np.asarray(c).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, (1.0 + 0.5 * m) * np.power(2.0, e - 1))
    return sign * mag


# the formula evaluated once for every byte value (only the low 4 bits count)
_E2M1_TABLE = _e2m1_formula(np.arange(256))


def e2m1_decode(codes) -> np.ndarray:
    """Value of E2M1 codes (the formula of ``_e2m1_formula``, looked up)."""
    return _E2M1_TABLE[np.asarray(codes).astype(np.uint8, copy=False)]


def e2m1_values() -> np.ndarray:
    """The 8 non-negative E2M1 values, codes 0..7 ascending."""
    return e2m1_decode(np.arange(8))


def _encode_rne(v, values: np.ndarray, sign_bit: int) -> np.ndarray:
    """Nearest of the ascending non-negative `values` (code = index), ties to
    the even code, saturating at the largest; the sign goes to `sign_bit`."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), values[-1])
    hi = np.searchsorted(values, a, side="left")          # values[hi] >= a
    hi = np.minimum(hi, len(values) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo = a - values[lo]
    dhi = values[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.int64)
    code = np.where(a == values[hi], hi, code)
    return (code | np.where(np.signbit(v), sign_bit, 0)).astype(np.uint8)


def e2m1_encode(v) -> np.ndarray:
    """Encode to E2M1 codes: round to nearest, ties to even, saturate at 6."""
    return _encode_rne(v, e2m1_values(), 0x8)


def e8m0_decode(codes) -> np.ndarray:
    """X = 2^(code - 127); code 255 is NaN."""
    c = np.asarray(codes).astype(np.int64)
    return np.where(c == 255, np.nan, np.ldexp(1.0, c - 127))


# element formats: (decode, encode, largest magnitude, exponent of the largest normal)
_ELEM = {
    "e4m3": (e4m3_decode, e4m3_encode, 448.0, 8),
    "e2m1": (e2m1_decode, e2m1_encode, 6.0, 2),
}

# ---------------------------------------------------------------------------
# MX quantisation along the last axis
# ---------------------------------------------------------------------------


def mx_quantize(a, elem: str = "e4m3"):
    """MX-quantise `a` [..., K] (K a multiple of 32) along its last axis.

    Returns (codes uint8 [..., K], scale codes uint8 [..., K/32]).
    """
    _, enc, _, emax = _ELEM[elem]
    a = np.asarray(a, dtype=np.float64)
    K = a.shape[-1]
    if K % MX_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = a.reshape(*a.shape[:-1], K // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    with np.errstate(divide="ignore"):
        s = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - emax, 0.0)
    s = np.clip(s, -127, 127).astype(np.int64)
    X = np.ldexp(1.0, s)
    codes = enc(blocks / X[..., None])
    return codes.reshape(a.shape).astype(np.uint8), (s + 127).astype(np.uint8)


def mx_dequantize(codes, scales, elem: str = "e4m3") -> np.ndarray:
    """Values of MX codes [..., K] with scale codes [..., K/32]."""
    dec = _ELEM[elem][0]
    codes = np.asarray(codes)
    K = codes.shape[-1]
    v = dec(codes).reshape(*codes.shape[:-1], K // MX_BLOCK, MX_BLOCK)
    return (v * e8m0_decode(scales)[..., None]).reshape(codes.shape)


def mx_dot_blocks(a_codes, a_scales, a_elem, w_codes, w_scales, w_elem) -> np.ndarray:
    """a [M, K] x w [N, K]^T in MX form, written as the block sum
    sum_b X_a[m, b] X_w[n, b] sum_i qa[m, b, i] qw[n, b, i]  (float64)."""
    da, dw = _ELEM[a_elem][0], _ELEM[w_elem][0]
    M, K = np.asarray(a_codes).shape
    N = np.asarray(w_codes).shape[0]
    nb = K // MX_BLOCK
    qa = da(a_codes).reshape(M, nb, MX_BLOCK)
    qw = dw(w_codes).reshape(N, nb, MX_BLOCK)
    inner = np.einsum("mbi,nbi->mnb", qa, qw)
    xa = e8m0_decode(a_scales)           # [M, nb]
    xw = e8m0_decode(w_scales)           # [N, nb]
    return np.einsum("mnb,mb,nb->mn", inner, xa, xw)


# ---------------------------------------------------------------------------
# per-slot SwiGLU FFN with MX operands
# ---------------------------------------------------------------------------


def ffn_mx(x, ids, w13_codes, w13_scales, w2_codes, w2_scales, w_elem: str = "e2m1", slots=None):
    """Per-slot expert FFN, MXFP8 activations and MX (`w_elem`) weights.

    x [T, H] (bf16 values as float); ids [T, k]; w13_codes [E, 2I, H] with
    w13_scales [E, 2I, H/32]; w2_codes [E, H, I] with w2_scales [E, H, I/32].
    Returns y float64 [len(slots), H] for the flat slots (all when None).
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    flat = ids.reshape(-1)
    slots = np.arange(T * k) if slots is None else np.asarray(slots, dtype=np.int64)
    x = np.asarray(x, dtype=np.float64)
    H = x.shape[1]
    I = np.asarray(w2_codes[0]).shape[1]
    y = np.zeros((len(slots), H))
    for n, sl in enumerate(slots):
        t, e = sl // k, int(flat[sl])
        xq, xs = mx_quantize(x[t:t + 1], "e4m3")
        gu = mx_dot_blocks(xq, xs, "e4m3", w13_codes[e], w13_scales[e], w_elem)[0]
        h = bf16_round(_silu(gu[:I]) * gu[I:])
        hq, hs = mx_quantize(h[None, :], "e4m3")
        y[n] = mx_dot_blocks(hq, hs, "e4m3", w2_codes[e], w2_scales[e], w_elem)[0]
    return y


def moe_forward_mx(x, logits, k, w13_codes, w13_scales, w2_codes, w2_scales, w_elem="e2m1", bias=None,
                   bias_mode="logits", n_shared=0, tokens=None):
    """Gate -> MX expert FFN -> combine (the layer of ``moe_oracle.moe_forward``
    with MX operands).  Returns (out float64, ids, weights)."""
    ids, w = topk_gate(logits, k, bias, bias_mode)
    if n_shared:
        ids, w = add_shared(ids, w, np.asarray(logits).shape[1], n_shared)
    T, kk = ids.shape
    toks = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    slots = (toks[:, None] * kk + np.arange(kk)[None, :]).reshape(-1)
    y = ffn_mx(x, ids, w13_codes, w13_scales, w2_codes, w2_scales, w_elem=w_elem, slots=slots)
    return combine(y, w[toks]), ids, w


__all__ = ["MX_BLOCK", "e2m1_decode", "e2m1_values", "e2m1_encode", "e8m0_decode", "mx_quantize",
           "mx_dequantize", "mx_dot_blocks", "ffn_mx", "moe_forward_mx"]

