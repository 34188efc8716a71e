"""Pins for the backward-pass oracle (oracle/backward_oracle.py).

* torch autograd through a dense torch formulation of the same forward,
  written here independently (per-slot weights gathered by expert, softmax
  over the chosen logits, bf16 rounding of h as a straight-through step),
  in float64;
* central finite differences of oracle.moe_forward for the parameters the
  forward is smooth in: the router logits (with a fixed top-k choice) and
  the down weights (h does not depend on them).
"""
import numpy as np
import pytest
import torch

import oracle.backward_oracle as bo
import oracle.moe_oracle as mo


def _layer(T, H, I, E, k, S=0, seed=0):
    rng = np.random.default_rng(seed)
    x = mo.bf16_round(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = mo.bf16_round(rng.standard_normal((E + S, 2 * I, H)) * 0.1)
    w2 = mo.bf16_round(rng.standard_normal((E + S, H, I)) * 0.1)
    dout = rng.standard_normal((T, H))
    bias = rng.standard_normal(E).astype(np.float32)
    return x, logits, w13, w2, dout, bias


def _torch_grads(x, logits, w13, w2, dout, k, bias, bias_mode, S):
    X = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    L = torch.tensor(logits.astype(np.float64), requires_grad=True)
    W13 = torch.tensor(w13, requires_grad=True)
    W2 = torch.tensor(w2, requires_grad=True)
    E = logits.shape[1]
    score = torch.tensor((logits + bias[None]).astype(np.float32), dtype=torch.float64) if bias is not None else L.detach()
    ids = torch.topk(score, k, dim=1).indices                     # the same choice as the forward
    src = L + torch.tensor(bias, dtype=torch.float64)[None] if (bias is not None and bias_mode == "logits") else L
    w = torch.softmax(src.gather(1, ids), dim=1)
    if S:
        ids = torch.cat([ids, torch.arange(E, E + S).expand(ids.shape[0], S)], dim=1)
        w = torch.cat([w, torch.ones(ids.shape[0], S, dtype=torch.float64)], dim=1)
    I = w2.shape[2]
    out = torch.zeros_like(X)
    for j in range(ids.shape[1]):
        e = ids[:, j]
        gu = torch.einsum("th,tnh->tn", X, W13[e])
        a = torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]
        h = a + (a.float().to(torch.bfloat16).double() - a).detach()   # rounded value, identity gradient
        y = torch.einsum("ti,thi->th", h, W2[e])
        out = out + w[:, j:j + 1] * y
    (out * torch.tensor(dout)).sum().backward()
    return X.grad.numpy(), L.grad.numpy(), W13.grad.numpy(), W2.grad.numpy(), ids.numpy()


@pytest.mark.parametrize("bias_mode,use_bias,S", [("logits", False, 0), ("logits", True, 0), ("select", True, 1),
                                                  ("logits", False, 2)])
def test_backward_matches_autograd(bias_mode, use_bias, S):
    x, logits, w13, w2, dout, bias = _layer(T=9, H=64, I=32, E=6, k=2, S=S, seed=3)
    b = bias if use_bias else None
    dx, dl, dw13, dw2 = bo.moe_backward(x, logits, 2, w13, w2, dout, bias=b, bias_mode=bias_mode, n_shared=S)
    tx, tl, tw13, tw2, tids = _torch_grads(x, logits, w13, w2, dout, 2, b, bias_mode, S)
    ids, _ = mo.topk_gate(logits, 2, b, bias_mode)
    np.testing.assert_array_equal(tids[:, :2], ids)
    # the oracle's routing weights are float32 (as in the forward), torch's
    # softmax stays float64: differences of ~1e-7 relative, far below any
    # mistake in a derivative (those are O(1e-2) and up)
    for got, ref in ((dx, tx), (dl, tl), (dw13, tw13), (dw2, tw2)):
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-7)


def _loss(x, logits, w13, w2, dout, k, bias, bias_mode, S):
    out, _, _ = mo.moe_forward(x, logits, k, w13, w2, bias=bias, n_shared=S, bias_mode=bias_mode)
    return float((out * dout).sum())


def test_backward_finite_differences_logits_and_down_weights():
    x, logits, w13, w2, dout, bias = _layer(T=4, H=32, I=32, E=5, k=2, S=1, seed=7)
    _, dl, _, dw2 = bo.moe_backward(x, logits, 2, w13, w2, dout, bias=bias, bias_mode="select", n_shared=1)
    rng = np.random.default_rng(0)
    eps = 1e-3
    ids, _ = mo.topk_gate(logits, 2, bias, "select")
    for _ in range(6):   # chosen logits (the choice itself is left unchanged by eps)
        t = int(rng.integers(4))
        e = int(ids[t, rng.integers(2)])
        lp, lm = logits.astype(np.float64).copy(), logits.astype(np.float64).copy()
        lp[t, e] += eps
        lm[t, e] -= eps
        fd = (_loss(x, lp, w13, w2, dout, 2, bias, "select", 1) - _loss(x, lm, w13, w2, dout, 2, bias, "select", 1)) / (2 * eps)
        assert abs(fd - dl[t, e]) <= 1e-4 * max(1.0, abs(dl[t, e]))
    for _ in range(8):   # down weights, routed and shared experts
        e, hh, ii = int(rng.integers(6)), int(rng.integers(32)), int(rng.integers(32))
        wp, wm = w2.copy(), w2.copy()
        wp[e, hh, ii] += eps
        wm[e, hh, ii] -= eps
        fd = (_loss(x, logits, w13, wp, dout, 2, bias, "select", 1) - _loss(x, logits, w13, wm, dout, 2, bias, "select", 1)) / (2 * eps)
        assert abs(fd - dw2[e, hh, ii]) <= 1e-6 * max(1.0, abs(dw2[e, hh, ii]))
    # unchosen logits get no gradient
    mask = np.ones_like(dl, dtype=bool)
    for t in range(4):
        mask[t, ids[t]] = False
    assert np.all(dl[mask] == 0)


def test_restricted_backward_equals_the_full_one():
    """Restricting the oracle to some tokens and experts leaves the computed
    entries unchanged and the others zero."""
    x, logits, w13, w2, dout, bias = _layer(T=12, H=16, I=8, E=5, k=2, S=1, seed=4)
    full = bo.moe_backward(x, logits, 2, w13, w2, dout, bias=bias, bias_mode="select", n_shared=1)
    toks, exps = [1, 7], [0, 5]
    part = bo.moe_backward(x, logits, 2, w13, w2, dout, bias=bias, bias_mode="select", n_shared=1,
                           tokens=toks, experts=exps)
    for a, b in zip(full[:2], part[:2]):
        np.testing.assert_array_equal(b[toks], a[toks])
        assert not np.any(np.delete(b, toks, axis=0))
    for a, b in zip(full[2:], part[2:]):
        np.testing.assert_array_equal(b[exps], a[exps])
        assert not np.any(np.delete(b, exps, axis=0))
