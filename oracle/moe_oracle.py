"""Plain, slow, obviously-correct CPU oracle of the MoE layer forward.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing in the CUDA
library imports, links or runs this file.

Sources (page title, section):

* [AS] "AMD GPU efficiency up 7x, optimised algorithm open-sourced: efficient
  MoE supports any number of experts" (dignews.cc, the MoE Align & Sort
  article).  Sections used: the opening definition of the MoE layer (Top-K
  gating scores route tokens to expert FFNs computed by a Group GEMM); the
  paragraph on MoE Align & Sort (sort tokens by expert id; aligned sorting
  lets each expert consume tokens in whole blocks); "FasterTransformer"
  (moe_softmax + moe_top_k fused as topk_gating_softmax, permute, group
  GEMM); "Megatron" (unpermute); "CK" (count occurrences to get offsets,
  then place in parallel; fused per-group token quantisation); "Writing
  AMD-friendly CUDA code with 3x~7x speed-up" (the D-C-P structure:
  distributed counting, cumsum -- unaligned local, merged, aligned global --
  and parallel placement).
* [P5] "[Feature]: Add more configuration options for MoE assembly kernels"
  (ROCm/aiter issue 1248), "Suggestion Description" (the a8w8 kernel
  fmoe_bf16_pertokenFp8_g1u1_silu: bf16 in/out, per-token FP8 activations,
  gate+up ("g1u1") with SiLU) and the "Estimated Performance Scaling" table.
* [GC] GC-MoE abstract (zhuanzhiai.com): fused SwiGLU with requantisation
  between the two grouped GEMMs.

Readings where the pages are silent (the same list is kept with the design notes):

1. Top-k ties go to the lower expert index; ids are listed by descending
   logit.  Weights are the softmax over all E logits, renormalised over the
   k selected ones.  A bias, when given, is added to the logits in fp32,
   either before both selection and softmax ("logits") or for the selection
   only ("select", the weights then use the raw logits).
1a. Shared experts have the routed experts' shape, see every token and enter
   the combine with weight 1; they are stored after the routed experts.
2. Within an expert's segment, slots keep ascending flat order
   (slot = t*k + j), as a counting sort gives.  Padding entries hold the
   sentinel T*k.  Experts with no slot get zero blocks.
3. FP8 is OCP E4M3FN, round-to-nearest-even, saturating to +-448.  Scales are
   fp32 ``amax / 448`` (``1`` when ``amax == 0``); the quotient ``v / s`` is an
   fp32 IEEE division.  Both are taken in fp32, the precision the kernels use,
   because they decide integer codes.
4. The gate/up output h is rounded to bf16 (the second GEMM's operand type)
   before the down projection and before its FP8 requantisation.
5. Everything else is computed in float64 (at least as accurate as the
   fp32-accumulated reference the tolerances are quoted against).

Pins (tests/test_oracle_*.py): brute-force top-k over all subsets; the k=E
case equals a library softmax; both bias modes against brute-force selection
on logit + bias with library-softmax weights (of the biased or the raw
logits), a constant bias and a bias that forces a set of experts;
brute-force align via Python ``sorted``; align invariants; bf16 rounding
equals torch's fp32->bf16 cast; the e4m3 codec round-trips all 256 codes,
matches torch's e4m3 cast in range and saturates beyond; identical experts
reproduce a dense SwiGLU FFN computed with library matmuls; k=1 forced
routing reproduces the dense FFN; shared experts add exactly their dense
FFNs (the layer with them minus the layer without them; routed outputs
forced to zero); x=0 gives 0; token permutation equivariance; expert
relabelling invariance; FP8 with exactly representable operands equals the
unquantised product.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_round(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits and fp32's exponent range; the spacing
    of representable values at magnitude 2**e is 2**(e-7), never below the
    subnormal quantum 2**-133.  Returned as float64.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = np.isfinite(v) & (v != 0)
    a = v[nz]
    _, E = np.frexp(a)                      # |a| = m * 2**E, 0.5 <= m < 1
    lead = np.maximum(E - 1, -126)          # exponent of the leading bit
    spacing = np.ldexp(1.0, (lead - 7).astype(np.int64))
    r = np.rint(a / spacing) * spacing      # np.rint rounds half to even
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, r), r)
    out[nz] = r
    out[~np.isfinite(v)] = v[~np.isfinite(v)]
    out[v == 0] = v[v == 0]
    return out


def _e4m3_formula(c) -> np.ndarray:
    """Value of OCP FP8 E4M3FN codes: 1 sign, 4 exponent (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN; no inf."""
    c = np.asarray(c, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6,
                   (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7).astype(np.int64)))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


# the formula evaluated once for each of the 256 codes; decoding indexes it
_E4M3_TABLE = _e4m3_formula(np.arange(256))


def e4m3_decode(codes) -> np.ndarray:
    """Value of OCP FP8 E4M3FN codes (the formula of ``_e4m3_formula``, looked
    up per code)."""
    # the uint8 cast keeps the low 8 bits, as the formula's & 0xFF does
    return _E4M3_TABLE[np.asarray(codes).astype(np.uint8, copy=False)]


def e4m3_values() -> np.ndarray:
    """The 127 finite non-negative E4M3FN values, codes 0..126 ascending."""
    return e4m3_decode(np.arange(127))


_E4M3_POS = None


def e4m3_encode(v) -> np.ndarray:
    """Encode float values to E4M3FN codes (uint8): nearest representable
    value, ties to the even code (mantissa LSB 0), magnitudes beyond 448
    saturate to 448 ("satfinite"), NaN maps to 0x7F."""
    global _E4M3_POS
    if _E4M3_POS is None:
        _E4M3_POS = e4m3_values()
    tab = _E4M3_POS
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    a_sat = np.minimum(a, tab[-1])
    hi = np.clip(np.searchsorted(tab, a_sat, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a_sat - tab[lo]
    d_hi = tab[hi] - a_sat
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.int64)
    code = np.where(np.signbit(v), code | 0x80, code)
    code = np.where(np.isnan(v), 0x7F, code)
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# A1: softmax top-k gating  ([AS] "FasterTransformer": topk_gating_softmax;
#     opening definition: Top-K gating scores, with a gating bias in DSv3)
# ---------------------------------------------------------------------------

def topk_gate(logits, k: int, bias=None, bias_mode: str = "logits"):
    """Top-k softmax gating.

    logits: float32 [T, E]; bias: float32 [E] or None (added in fp32).
    Returns ids int32 [T, k] (descending score, ties to the lower index) and
    weights float32 [T, k] = softmax(l)[sel] / sum(softmax(l)[sel]).

    bias_mode "logits": the biased logits are both the selection score and
    the l of the weights.  "select" ([AS] opening: DeepSeek's gating bias for
    auxiliary-loss-free balancing): the biased logits only pick the experts;
    the weights use the raw logits.
    """
    if bias_mode not in ("logits", "select"):
        raise ValueError(bias_mode)
    l32 = np.asarray(logits, dtype=np.float32)
    score = l32
    if bias is not None:
        score = (l32 + np.asarray(bias, dtype=np.float32)[None, :]).astype(np.float32)
    T, E = l32.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    # stable sort of the negated scores keeps equal values in index order
    order = np.argsort(-score, axis=1, kind="stable")
    ids = order[:, :k].astype(np.int32)
    l = (score if bias_mode == "logits" else l32).astype(np.float64)
    p = np.exp(l - l.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    psel = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    w = psel / psel.sum(axis=1, keepdims=True)
    return ids, w.astype(np.float32)


def add_shared(ids, w, E: int, n_shared: int):
    """Append the always-on shared experts ([AS] opening: DeepSeek's shared
    expert, one of them) to every token's routing: experts E..E+n_shared-1,
    weight 1 each, after the k routed choices."""
    ids = np.asarray(ids, dtype=np.int32)
    w = np.asarray(w, dtype=np.float32)
    T = ids.shape[0]
    sid = np.broadcast_to(E + np.arange(n_shared, dtype=np.int32), (T, n_shared))
    return (np.concatenate([ids, sid], axis=1),
            np.concatenate([w, np.ones((T, n_shared), np.float32)], axis=1))


# ---------------------------------------------------------------------------
# A2: block-aligned MoE Align & Sort  ([AS] D-C-P section; "CK")
# ---------------------------------------------------------------------------

def expected_sizes(T: int, k: int, E: int, bm: int):
    """Capacity of the sorted buffer: every expert pads by at most bm-1."""
    P = T * k + E * (bm - 1)
    NB = -(-P // bm)
    return P, NB


def align_sort(topk_ids, E: int, bm: int):
    """Counting sort of the T*k flat slots by expert, each expert's segment
    padded to a multiple of bm.

    Steps in the article's order: (D) count slots per expert; (C) pad each
    count to a multiple of bm and take the exclusive cumulative sum as the
    segment offsets; (P) place every slot at its expert's offset plus its
    rank among earlier slots of the same expert.  Padding holds T*k.

    Returns (sorted_ids int32 [num_post], expert_ids int32 [num_post//bm],
    num_post int).
    """
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    N = ids.size
    if N and (ids.min() < 0 or ids.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(ids, minlength=E)                      # (D)
    padded = -(-counts // bm) * bm                              # (C)
    offsets = np.concatenate([[0], np.cumsum(padded)[:-1]])
    num_post = int(padded.sum())
    order = np.argsort(ids, kind="stable")                      # (P)
    first = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank = np.arange(N) - first[ids[order]]
    dest = offsets[ids[order]] + rank
    sorted_ids = np.full(num_post, N, dtype=np.int64)
    sorted_ids[dest] = order
    expert_ids = np.repeat(np.arange(E), padded // bm)
    return sorted_ids.astype(np.int32), expert_ids.astype(np.int32), num_post


# ---------------------------------------------------------------------------
# A3 / A5: per-row FP8 quantisation  ([P5] "pertokenFp8"; [GC] requant)
# ---------------------------------------------------------------------------

def quant_rows_e4m3(a):
    """Per-row E4M3 quantisation: s = amax/448 (fp32; 1 if amax is 0),
    codes = e4m3(fp32(a / s)).  Returns (codes uint8 [R, C], s float32 [R])."""
    a32 = np.asarray(a, dtype=np.float32)
    amax = np.abs(a32).max(axis=1) if a32.shape[1] else np.zeros(a32.shape[0], np.float32)
    s = (amax / np.float32(448.0)).astype(np.float32)
    s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
    q = (a32 / s[:, None]).astype(np.float32)
    return e4m3_encode(q), s


# ---------------------------------------------------------------------------
# A4 + A6: gated expert FFN per slot ([AS] opening definition; [P5] g1u1_silu)
# ---------------------------------------------------------------------------

def _silu(g):
    return g / (1.0 + np.exp(-g))


def _slot_groups(ids_flat, E):
    for e in range(E):
        slots = np.nonzero(ids_flat == e)[0]
        if slots.size:
            yield e, slots


def ffn_bf16(x, ids, w13, w2, slots=None):
    """Per-slot SwiGLU expert FFN with bf16 operands.

    x [T, H]; ids [T, k]; w13 [E, 2I, H] (rows 0..I-1 gate, I..2I-1 up);
    w2 [E, H, I].  For slot i = t*k + j with expert e:
      g = Wg[e] x_t, u = Wu[e] x_t, h = bf16(silu(g) * u), y_i = W2[e] h.
    Returns y float64 [len(slots), H] (all T*k slots when slots is None).
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    E, twoI, H = w13.shape
    I = twoI // 2
    flat = ids.reshape(-1)
    sel = np.arange(T * k) if slots is None else np.asarray(slots, dtype=np.int64)
    y = np.zeros((sel.size, H), dtype=np.float64)
    sub = flat[sel]
    for e, pos in _slot_groups(sub, E):
        xe = x[sel[pos] // k]
        W = np.asarray(w13[e], dtype=np.float64)
        g = xe @ W[:I].T
        u = xe @ W[I:].T
        h = bf16_round(_silu(g) * u)
        y[pos] = h @ np.asarray(w2[e], dtype=np.float64).T
    return y


def ffn_a8w8(x, ids, w13_q, w13_s, w2_q, w2_s, slots=None):
    """Per-slot SwiGLU expert FFN, per-token FP8 activations ("a8w8").

    x bf16 values [T, H]; w13_q E4M3 codes [E, 2I, H] with per-output-channel
    fp32 scales w13_s [E, 2I]; w2_q [E, H, I] with w2_s [E, H].
      (q_x, s_x) = quant_rows_e4m3(x)                       (per token)
      g = (Wg_q[e] . q_x) * s_x * sg[e]; u likewise
      h = bf16(silu(g) * u); (q_h, s_h) = quant_rows_e4m3(h)  (requant)
      y = (W2_q[e] . q_h) * s_h * s2[e]
    Products of E4M3 values are exact in float64 and so are the sums here.
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    E, twoI, H = w13_q.shape
    I = twoI // 2
    qx, sx = quant_rows_e4m3(np.asarray(x, dtype=np.float32))
    xq = e4m3_decode(qx)
    flat = ids.reshape(-1)
    sel = np.arange(T * k) if slots is None else np.asarray(slots, dtype=np.int64)
    y = np.zeros((sel.size, H), dtype=np.float64)
    sub = flat[sel]
    for e, pos in _slot_groups(sub, E):
        tok = sel[pos] // k
        W = e4m3_decode(np.asarray(w13_q[e]))
        s13 = np.asarray(w13_s[e], dtype=np.float64)
        acc = xq[tok] @ W.T
        gu = acc * sx[tok].astype(np.float64)[:, None] * s13[None, :]
        g, u = gu[:, :I], gu[:, I:]
        h = bf16_round(_silu(g) * u)
        qh, sh = quant_rows_e4m3(h)
        W2 = e4m3_decode(np.asarray(w2_q[e]))
        acc2 = e4m3_decode(qh) @ W2.T
        y[pos] = acc2 * sh.astype(np.float64)[:, None] * np.asarray(w2_s[e], dtype=np.float64)[None, :]
    return y


# ---------------------------------------------------------------------------
# A7: top-k weighted combine  ([AS] "Megatron": unpermute)
# ---------------------------------------------------------------------------

def combine(y, w):
    """out[t] = sum_j w[t, j] * y[t*k + j]  (float64)."""
    w = np.asarray(w, dtype=np.float64)
    T, k = w.shape
    y = np.asarray(y, dtype=np.float64)
    y = y.reshape(T, k, y.shape[-1])      # rows t*k .. t*k+k-1 are token t's slots
    return np.einsum("tk,tkh->th", w, y)


# ---------------------------------------------------------------------------
# whole layer
# ---------------------------------------------------------------------------

def moe_forward(x, logits, k, w13, w2, bias=None, a8w8=False, w13_s=None,
                w2_s=None, tokens=None, n_shared=0, bias_mode="logits"):
    """Gate -> (align, which only reorders) -> expert FFN -> combine.

    The weights hold E = logits.shape[1] routed experts followed by
    ``n_shared`` shared experts; every token also goes to each shared expert
    with weight 1.  Returns (out float64 [len(tokens) or T, H], ids, weights)
    with ids/weights [T, k + n_shared].  ``tokens`` restricts the FFN and
    combine to a subset of tokens (routing is computed for all of them).
    """
    ids, w = topk_gate(logits, k, bias, bias_mode)
    if n_shared:
        ids, w = add_shared(ids, w, np.asarray(logits).shape[1], n_shared)
    T, kk = ids.shape
    toks = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    slots = (toks[:, None] * kk + np.arange(kk)[None, :]).reshape(-1)
    if a8w8:
        y = ffn_a8w8(x, ids, w13, w13_s, w2, w2_s, slots=slots)
    else:
        y = ffn_bf16(x, ids, w13, w2, slots=slots)
    out = combine(y, w[toks])
    return out, ids, w


def silu_ref(g):
    """SiLU written out, exposed for the pins."""
    return _silu(np.asarray(g, dtype=np.float64))


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "math", "np")]
