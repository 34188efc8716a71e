"""CPU oracle of the MoE layer's backward pass (bf16 weights).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing in the CUDA
library imports, links or runs this file.

Source: the MoE Align & Sort article ("Megatron": the combine's gradient is
the unpermute; the opening definition of the layer).  The pages give no
formulas for the backward pass; the gradients below are the chain rule
applied to the forward of ``moe_oracle.moe_forward``, step by step in
reverse:

    out[t] = sum_j w[t,j] y[t,j]        (combine)
    y      = h Wd[e]^T                  (down projection)
    h      = silu(g) * u                (SwiGLU; g, u = x Wg[e]^T, x Wu[e]^T)
    w[t,:] = softmax of the chosen logits (renormalised top-k)

Readings (listed with the design notes):

1. The bf16 rounding of h is passed through unchanged (straight-through):
   dh is the gradient of the unrounded product, while dWd uses the rounded h
   the forward computed.
2. The top-k choice is piecewise constant: only the chosen experts' logits
   receive gradient.  With a selection-only bias the weights depend on the
   raw logits, so the gradient lands on them; with the bias added to the
   logits it lands on the logits as well (the bias is a constant shift).
3. Shared experts enter with the constant weight 1: no logit gradient.

Pins (tests/test_oracle_backward.py): torch autograd through an independent
dense torch formulation of the same forward, and central finite differences
of ``moe_forward`` on tiny layers.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import _silu, add_shared, bf16_round, topk_gate


def _sigmoid(g):
    return 1.0 / (1.0 + np.exp(-g))


def moe_backward(x, logits, k, w13, w2, dout, bias=None, bias_mode="logits", n_shared=0, tokens=None,
                 experts=None):
    """Gradients of sum(out * dout) for the layer of ``moe_forward``.

    x [T, H], logits [T, E] (E routed experts), w13 [E+S, 2I, H],
    w2 [E+S, H, I], dout [T, H].  Returns (dx [T, H], dlogits [T, E],
    dw13 [E+S, 2I, H], dw2 [E+S, H, I]) in float64.

    ``tokens`` / ``experts`` (for large layers) restrict the work: dx and
    dlogits are computed for the listed tokens only and the weight gradients
    for the listed experts only (the other entries are left zero); each
    computed entry is the same sum as without the restriction.
    """
    x = np.asarray(x, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    T, H = x.shape
    E = np.asarray(logits).shape[1]
    ids, w = topk_gate(logits, k, bias, bias_mode)
    if n_shared:
        ids, w = add_shared(ids, w, E, n_shared)
    kk = ids.shape[1]
    w = w.astype(np.float64)
    I = np.asarray(w2[0]).shape[1]
    EW = E + n_shared

    dx = np.zeros_like(x)
    dw13 = np.zeros((EW, 2 * I, H))
    dw2 = np.zeros((EW, H, I))
    dwt = np.zeros((T, kk))            # d loss / d w[t, j]

    want_t = np.ones(T, dtype=bool) if tokens is None else np.isin(np.arange(T), np.asarray(tokens))
    want_e = None if experts is None else set(int(e) for e in experts)
    for t in range(T):
        for j in range(kk):
            e = int(ids[t, j])
            for_t = bool(want_t[t])
            for_e = want_e is None or e in want_e
            if not (for_t or for_e):
                continue
            W13 = np.asarray(w13[e], dtype=np.float64)
            Wd = np.asarray(w2[e], dtype=np.float64)
            # forward of this slot, as the oracle computes it
            gu = W13 @ x[t]
            g, u = gu[:I], gu[I:]
            a = _silu(g)
            h = bf16_round(a * u)
            y = Wd @ h
            # combine: out[t] += w y  ->  dy = w dout, dw = <dout, y>
            dwt[t, j] = dout[t] @ y
            dy = w[t, j] * dout[t]
            # down projection
            if for_e:
                dw2[e] += np.outer(dy, h)
            dh = Wd.T @ dy                 # straight through the bf16 rounding
            # SwiGLU
            du = dh * a
            da = dh * u
            s = _sigmoid(g)
            dg = da * (s * (1.0 + g * (1.0 - s)))
            # gate/up projection
            dgu = np.concatenate([dg, du])
            if for_e:
                dw13[e] += np.outer(dgu, x[t])
            if for_t:
                dx[t] += W13.T @ dgu

    # renormalised softmax over the k routed choices (shared columns have w = 1)
    dlogits = np.zeros((T, E))
    for t in np.nonzero(want_t)[0]:
        wr = w[t, :k]
        g_w = dwt[t, :k]
        dl_sel = wr * (g_w - np.dot(wr, g_w))
        for j in range(k):
            dlogits[t, int(ids[t, j])] += dl_sel[j]
    return dx, dlogits, dw13, dw2


__all__ = ["moe_backward"]
