"""Pins for the oracle's expert FFN, combine and whole-layer forward.

* identical experts with weights summing to 1 reproduce a dense SwiGLU FFN
  computed with library matmuls (torch, float64) -- bf16 and a8w8 (the a8w8
  dense reference uses torch's float8_e4m3fn cast as its codec);
* routing everything to one expert (k = 1, forced logit) is the dense FFN of
  that expert;
* x = 0 gives out = 0;
* permuting tokens permutes the output; relabelling experts (weights and
  logit columns together) leaves it unchanged;
* the combine is the weighted sum written with a library einsum-free loop;
* shared experts add their dense FFN with weight 1 (the layer with them minus
  the layer without them; routed outputs forced to zero);
* a planted mistake (gate and up swapped) fails the dense pin.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as mo
from moe_inputs import MoEConfig, make_layer, to_numpy


def _layer(T=24, H=64, I=32, E=4, k=2, a8w8=False, seed=11):
    cfg = MoEConfig("t", T=T, H=H, I=I, E=E, k=k, bm=8, a8w8=a8w8, seed=seed)
    return cfg, make_layer(cfg)


def _dense_swiglu_bf16(x, w13, w2):
    """Dense FFN with torch float64 matmuls; h rounded to bf16 by torch."""
    x = torch.from_numpy(x)
    W = torch.from_numpy(w13)
    I = W.shape[0] // 2
    g = x @ W[:I].T
    u = x @ W[I:].T
    h = (torch.nn.functional.silu(g) * u).float().to(torch.bfloat16).double()
    return (h @ torch.from_numpy(w2).T).numpy()


def _dense_swiglu_a8w8(x, w13q, w13s, w2q, w2s):
    """Dense a8w8 FFN with torch's e4m3 cast and float64 matmuls."""
    def q(a):
        a = torch.from_numpy(np.asarray(a, np.float32))
        amax = a.abs().amax(1)
        s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        c = (a / s[:, None]).clamp(-448, 448).to(torch.float8_e4m3fn).double()
        return c, s.double()
    dec = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).double()
    I = w13q.shape[0] // 2
    cx, sx = q(x)
    gu = (cx @ dec(w13q).T) * sx[:, None] * torch.from_numpy(w13s).double()[None]
    g, u = gu[:, :I], gu[:, I:]
    h = (torch.nn.functional.silu(g) * u).float().to(torch.bfloat16).float()
    ch, sh = q(h.numpy())
    return ((ch @ dec(w2q).T) * sh[:, None] * torch.from_numpy(w2s).double()[None]).numpy()


def test_identical_experts_equal_dense_bf16():
    cfg, d = _layer()
    w13 = to_numpy(d["w13"])
    w2 = to_numpy(d["w2"])
    w13[:] = w13[0]
    w2[:] = w2[0]
    x = to_numpy(d["x"])
    out, ids, w = mo.moe_forward(x, to_numpy(d["logits"]), cfg.k, w13, w2)
    ref = _dense_swiglu_bf16(x, w13[0], w2[0])
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6)


def test_identical_experts_equal_dense_a8w8():
    cfg, d = _layer(a8w8=True)
    w13q, w13s = to_numpy(d["w13_q"]), to_numpy(d["w13_s"])
    w2q, w2s = to_numpy(d["w2_q"]), to_numpy(d["w2_s"])
    for a in (w13q, w13s, w2q, w2s):
        a[:] = a[0]
    x = to_numpy(d["x"])
    out, _, _ = mo.moe_forward(x, to_numpy(d["logits"]), cfg.k, w13q, w2q,
                               a8w8=True, w13_s=w13s, w2_s=w2s)
    ref = _dense_swiglu_a8w8(x, w13q[0], w13s[0], w2q[0], w2s[0])
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6)


def test_forced_single_expert_is_dense():
    cfg, d = _layer(k=1)
    logits = to_numpy(d["logits"]).astype(np.float32)
    logits[:, 2] = 100.0
    x, w13, w2 = to_numpy(d["x"]), to_numpy(d["w13"]), to_numpy(d["w2"])
    out, ids, w = mo.moe_forward(x, logits, 1, w13, w2)
    assert np.all(ids == 2) and np.all(w == 1.0)
    np.testing.assert_allclose(out, _dense_swiglu_bf16(x, w13[2], w2[2]), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("a8w8", [False, True])
def test_shared_expert_adds_its_dense_ffn(a8w8):
    """Shared experts enter with weight 1 for every token: the layer with
    n_shared = 2 minus the same layer without them is the sum of the two
    shared experts' dense FFNs (torch float64 matmuls)."""
    cfg = MoEConfig("t", T=24, H=64, I=32, E=4, k=2, bm=8, a8w8=a8w8, n_shared=2, seed=17)
    d = make_layer(cfg)
    x, logits = to_numpy(d["x"]), to_numpy(d["logits"])
    E = cfg.E
    if a8w8:
        w13q, w13s, w2q, w2s = (to_numpy(d[n]) for n in ("w13_q", "w13_s", "w2_q", "w2_s"))
        out2, ids, w = mo.moe_forward(x, logits, cfg.k, w13q, w2q, a8w8=True, w13_s=w13s, w2_s=w2s,
                                      n_shared=2)
        out0, _, _ = mo.moe_forward(x, logits, cfg.k, w13q[:E], w2q[:E], a8w8=True, w13_s=w13s[:E],
                                    w2_s=w2s[:E])
        dense = sum(_dense_swiglu_a8w8(x, w13q[e], w13s[e], w2q[e], w2s[e]) for e in (E, E + 1))
    else:
        w13, w2 = to_numpy(d["w13"]), to_numpy(d["w2"])
        out2, ids, w = mo.moe_forward(x, logits, cfg.k, w13, w2, n_shared=2)
        out0, _, _ = mo.moe_forward(x, logits, cfg.k, w13[:E], w2[:E])
        dense = sum(_dense_swiglu_bf16(x, w13[e], w2[e]) for e in (E, E + 1))
    assert ids.shape == (cfg.T, cfg.k + 2)
    np.testing.assert_array_equal(ids[:, cfg.k:], np.broadcast_to([E, E + 1], (cfg.T, 2)))
    np.testing.assert_array_equal(w[:, cfg.k:], 1.0)
    np.testing.assert_allclose(out2 - out0, dense, rtol=1e-5, atol=1e-6)


def test_shared_expert_alone_when_routed_outputs_vanish():
    """With every routed expert's down projection zero, the layer is the
    shared expert's dense FFN whatever the routing."""
    cfg = MoEConfig("t", T=16, H=64, I=32, E=6, k=3, bm=8, n_shared=1, bias=True, bias_mode="select",
                    seed=19)
    d = make_layer(cfg)
    x, w13, w2 = to_numpy(d["x"]), to_numpy(d["w13"]), to_numpy(d["w2"])
    w2[:cfg.E] = 0.0
    out, _, _ = mo.moe_forward(x, to_numpy(d["logits"]), cfg.k, w13, w2, bias=to_numpy(d["bias"]),
                               n_shared=1, bias_mode="select")
    np.testing.assert_allclose(out, _dense_swiglu_bf16(x, w13[cfg.E], w2[cfg.E]), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("a8w8", [False, True])
def test_zero_input_gives_zero(a8w8):
    cfg, d = _layer(a8w8=a8w8)
    x = np.zeros((cfg.T, cfg.H))
    if a8w8:
        out, _, _ = mo.moe_forward(x, to_numpy(d["logits"]), cfg.k, to_numpy(d["w13_q"]),
                                   to_numpy(d["w2_q"]), a8w8=True, w13_s=to_numpy(d["w13_s"]),
                                   w2_s=to_numpy(d["w2_s"]))
    else:
        out, _, _ = mo.moe_forward(x, to_numpy(d["logits"]), cfg.k, to_numpy(d["w13"]), to_numpy(d["w2"]))
    assert np.all(out == 0)


def test_token_permutation_and_expert_relabelling():
    cfg, d = _layer(T=16, E=6, k=3)
    x, lg, w13, w2 = to_numpy(d["x"]), to_numpy(d["logits"]), to_numpy(d["w13"]), to_numpy(d["w2"])
    out, _, _ = mo.moe_forward(x, lg, cfg.k, w13, w2)
    rng = np.random.default_rng(0)
    pt = rng.permutation(cfg.T)
    out_p, _, _ = mo.moe_forward(x[pt], lg[pt], cfg.k, w13, w2)
    np.testing.assert_allclose(out_p, out[pt], rtol=0, atol=0)
    pe = rng.permutation(cfg.E)
    # expert pe[j] of the relabelled layer is expert j of the original one
    w13r, w2r, lgr = np.empty_like(w13), np.empty_like(w2), np.empty_like(lg)
    w13r[pe], w2r[pe], lgr[:, pe] = w13, w2, lg
    out_r, _, _ = mo.moe_forward(x, lgr, cfg.k, w13r, w2r)
    np.testing.assert_allclose(out_r, out, rtol=1e-12, atol=1e-14)


def test_combine_against_loop():
    rng = np.random.default_rng(5)
    T, k, H = 7, 3, 5
    y = rng.standard_normal((T * k, H))
    w = rng.random((T, k))
    out = mo.combine(y, w)
    for t in range(T):
        ref = np.zeros(H)
        for j in range(k):
            ref += w[t, j] * y[t * k + j]
        np.testing.assert_allclose(out[t], ref, rtol=1e-14)


def test_combine_of_no_tokens():
    out = mo.combine(np.zeros((0, 5)), np.zeros((0, 3)))
    assert out.shape == (0, 5)


def test_tokens_subset_matches_full():
    cfg, d = _layer()
    x, lg, w13, w2 = to_numpy(d["x"]), to_numpy(d["logits"]), to_numpy(d["w13"]), to_numpy(d["w2"])
    full, _, _ = mo.moe_forward(x, lg, cfg.k, w13, w2)
    sub, _, _ = mo.moe_forward(x, lg, cfg.k, w13, w2, tokens=[3, 0, 17])
    np.testing.assert_array_equal(sub, full[[3, 0, 17]])


def test_planted_gate_up_swap_is_caught(monkeypatch):
    """Swapping the gate and up halves inside the oracle breaks the dense pin."""
    orig = mo.ffn_bf16

    def swapped(x, ids, w13, w2, slots=None):
        I = w13.shape[1] // 2
        w13s = np.concatenate([w13[:, I:], w13[:, :I]], axis=1)
        return orig(x, ids, w13s, w2, slots)

    monkeypatch.setattr(mo, "ffn_bf16", swapped)
    with pytest.raises(AssertionError):
        test_identical_experts_equal_dense_bf16()
