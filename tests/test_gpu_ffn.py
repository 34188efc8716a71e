"""GPU parity of moe_grouped_ffn, moe_combine and moe_forward on layers the
oracle computes in full (seconds on the CPU): several weight tiles, token
groups of every tile size, ragged expert segments, bf16 and a8w8.

Gate: max-abs and relative-Frobenius error of 2e-2 / 1e-2 (bf16) and
5e-2 / 3e-2 (a8w8) against the float64 oracle.
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
from moe_inputs import CONFIGS, MoEConfig, make_layer, to_numpy
from parity_util import TOL_BF16, TOL_FP8, assert_close, bf16_ulp

pytestmark = pytest.mark.gpu

SMALL = [
    CONFIGS["tiny"],
    MoEConfig("ragged", T=300, H=384, I=256, E=16, k=4, bm=32, seed=101),
    MoEConfig("wide", T=200, H=512, I=384, E=5, k=3, bm=64, seed=102),
    MoEConfig("skew", T=257, H=256, I=128, E=32, k=8, bm=16, bias=True, seed=103),
    # few tokens per expert
    MoEConfig("fewtok", T=3, H=1024, I=512, E=16, k=2, bm=16, seed=104),
    # many tokens per expert: 256-token tiles, several tiles per expert
    MoEConfig("manytok", T=1024, H=512, I=384, E=4, k=2, bm=64, seed=105),
    # two tokens, four slots each: the forward fuses the combine, and routes
    # its 8 slots with the few-slot routing kernel
    MoEConfig("tinybatch", T=2, H=512, I=512, E=16, k=4, bm=16, seed=109),
]


def _dev(d, dev):
    return {k: (v.to(dev) if v is not None else None) for k, v in d.items()}


def _oracle_y(cfg, d, ids):
    if cfg.a8w8:
        return oracle.ffn_a8w8(to_numpy(d["x"]), ids, to_numpy(d["w13_q"]), to_numpy(d["w13_s"]),
                               to_numpy(d["w2_q"]), to_numpy(d["w2_s"]))
    return oracle.ffn_bf16(to_numpy(d["x"]), ids, to_numpy(d["w13"]), to_numpy(d["w2"]))


def _weights(cfg, g):
    if cfg.a8w8:
        return g["w13_q"], g["w2_q"], g["w13_s"], g["w2_s"]
    return g["w13"], g["w2"], None, None


@pytest.mark.parametrize("a8w8", [False, True])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
@pytest.mark.parametrize("tile", [0, 16, 64, 256])
def test_grouped_ffn_parity(cuda_device, cfg, a8w8, tile):
    cfg = cfg.with_(a8w8=a8w8)
    d = make_layer(cfg)
    g = _dev(d, cuda_device)
    ids, w = m.topk_gate(g["logits"], cfg.k, g["bias"])
    s, b, n = m.align_sort(ids, cfg.E, cfg.bm)
    w13, w2, s13, s2 = _weights(cfg, g)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    y = m.grouped_ffn(g["x"], w13, w2, s, b, n, cfg.k, cfg.bm, s13, s2, tile_tokens=tile, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref_ids, _ = oracle.topk_gate(to_numpy(d["logits"]), cfg.k, to_numpy(d["bias"]))
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    ref_y = _oracle_y(cfg, d, ref_ids)
    assert_close(y.cpu().numpy(), ref_y, TOL_FP8 if a8w8 else TOL_BF16, f"{cfg.name} y")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_combine_parity(cuda_device, out_dtype):
    gen = torch.Generator().manual_seed(9)
    T, k, H = 333, 6, 1024
    y = torch.randn(T * k, H, generator=gen)
    w = torch.rand(T, k, generator=gen)
    out = m.combine(y.to(cuda_device), w.to(cuda_device), out_dtype)
    torch.cuda.synchronize()
    ref = oracle.combine(y.numpy(), w.numpy())
    got = out.float().cpu().numpy()
    if out_dtype == torch.float32:
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-5)
    else:
        assert np.all(np.abs(got - ref) <= bf16_ulp(ref) * 0.5 + 1e-6)


@pytest.mark.parametrize("a8w8", [False, True])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_forward_parity_small(cuda_device, cfg, a8w8):
    cfg = cfg.with_(a8w8=a8w8)
    d = make_layer(cfg)
    g = _dev(d, cuda_device)
    w13, w2, s13, s2 = _weights(cfg, g)
    ref, ref_ids, ref_w = oracle.moe_forward(
        to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k,
        to_numpy(d["w13_q"] if a8w8 else d["w13"]), to_numpy(d["w2_q"] if a8w8 else d["w2"]),
        bias=to_numpy(d["bias"]), a8w8=a8w8, w13_s=to_numpy(d.get("w13_s")), w2_s=to_numpy(d.get("w2_s")))
    tol = TOL_FP8 if a8w8 else TOL_BF16
    for out_dtype in (torch.float32, torch.bfloat16):
        layer = m.MoELayer(w13, w2, cfg.k, cfg.bm, s13, s2, out_dtype=out_dtype)
        ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=cuda_device)
        tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=cuda_device)
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        out = layer(g["x"], g["logits"], g["bias"], topk_ids=ids, topk_w=tw, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
        assert np.max(np.abs(tw.cpu().numpy() - ref_w)) <= 1e-6
        assert_close(out.float().cpu().numpy(), ref, tol, f"{cfg.name} out {out_dtype}")


# many experts: 32 logits per lane in the routing launch; T=8 routes in one
# CTA (the few-slot launch of 8 warps), T=200 over several CTAs
MANY = [
    MoEConfig("many_e1000_t8", T=8, H=256, I=128, E=1000, k=8, bm=16, seed=110),
    MoEConfig("many_e1000_t200", T=200, H=256, I=128, E=1000, k=8, bm=16, seed=111),
    MoEConfig("many_e600_t16", T=16, H=256, I=128, E=600, k=6, bm=32, bias=True, seed=112),
]


@pytest.mark.parametrize("cfg", MANY, ids=lambda c: c.name)
def test_forward_parity_many_experts(cuda_device, cfg):
    d = make_layer(cfg)
    g = _dev(d, cuda_device)
    ref, ref_ids, ref_w = oracle.moe_forward(to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k,
                                             to_numpy(d["w13"]), to_numpy(d["w2"]), bias=to_numpy(d["bias"]))
    layer = m.MoELayer(g["w13"], g["w2"], cfg.k, cfg.bm, out_dtype=torch.float32)
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=cuda_device)
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = layer(g["x"], g["logits"], g["bias"], topk_ids=ids, topk_w=tw, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) <= 1e-6
    assert_close(out.float().cpu().numpy(), ref, TOL_BF16, f"{cfg.name} out")


@pytest.mark.parametrize("a8w8", [False, True])
def test_forward_parity_few_slots_wide_rows(cuda_device, a8w8):
    """32 slots (the few-slot routing kernel) with the fused combine over a
    token accumulator too large for that one-CTA kernel to zero (T*H > 65536
    floats): the accumulator is cleared by a memset instead."""
    cfg = MoEConfig("few_wide", T=4, H=16512, I=128, E=16, k=8, bm=16, seed=113).with_(a8w8=a8w8)
    d = make_layer(cfg)
    g = _dev(d, cuda_device)
    w13, w2, s13, s2 = _weights(cfg, g)
    ref, _, _ = oracle.moe_forward(
        to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k,
        to_numpy(d["w13_q"] if a8w8 else d["w13"]), to_numpy(d["w2_q"] if a8w8 else d["w2"]),
        a8w8=a8w8, w13_s=to_numpy(d.get("w13_s")), w2_s=to_numpy(d.get("w2_s")))
    layer = m.MoELayer(w13, w2, cfg.k, cfg.bm, s13, s2, out_dtype=torch.float32)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    for _ in range(2):      # the second call must not add to the first one's sums
        out = layer(g["x"], g["logits"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close(out.cpu().numpy(), ref, TOL_FP8 if a8w8 else TOL_BF16, "few slots, wide rows")


SHARED = [
    # DeepSeek-style: selection-only bias and one shared expert
    MoEConfig("shared1", T=300, H=384, I=256, E=16, k=4, bm=32, bias=True, n_shared=1, bias_mode="select",
              seed=106),
    MoEConfig("shared2", T=64, H=256, I=128, E=8, k=2, bm=16, bias=True, n_shared=2, seed=107),
    # shared expert with many tokens next to routed experts with few
    MoEConfig("shared_big", T=700, H=512, I=384, E=32, k=2, bm=64, n_shared=1, bias=True, bias_mode="select",
              seed=108),
]


@pytest.mark.parametrize("a8w8", [False, True])
@pytest.mark.parametrize("cfg", SHARED, ids=lambda c: c.name)
def test_forward_parity_shared_and_bias_modes(cuda_device, cfg, a8w8):
    cfg = cfg.with_(a8w8=a8w8)
    d = make_layer(cfg)
    g = _dev(d, cuda_device)
    w13, w2, s13, s2 = _weights(cfg, g)
    ref, ref_ids, ref_w = oracle.moe_forward(
        to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k,
        to_numpy(d["w13_q"] if a8w8 else d["w13"]), to_numpy(d["w2_q"] if a8w8 else d["w2"]),
        bias=to_numpy(d["bias"]), a8w8=a8w8, w13_s=to_numpy(d.get("w13_s")), w2_s=to_numpy(d.get("w2_s")),
        n_shared=cfg.n_shared, bias_mode=cfg.bias_mode)
    tol = TOL_FP8 if a8w8 else TOL_BF16
    kk = cfg.k + cfg.n_shared
    layer = m.MoELayer(w13, w2, cfg.k, cfg.bm, s13, s2, out_dtype=torch.float32, n_shared=cfg.n_shared,
                       bias_mode=cfg.bias_mode)
    ids = torch.empty(cfg.T, kk, dtype=torch.int32, device=cuda_device)
    tw = torch.empty(cfg.T, kk, dtype=torch.float32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = layer(g["x"], g["logits"], g["bias"], topk_ids=ids, topk_w=tw, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) <= 1e-6
    assert_close(out.float().cpu().numpy(), ref, tol, f"{cfg.name} out")


def test_forward_zero_input(cuda_device):
    cfg = SMALL[1]
    d = make_layer(cfg)
    g = _dev(d, cuda_device)
    layer = m.MoELayer(g["w13"], g["w2"], cfg.k, cfg.bm, out_dtype=torch.float32)
    out = layer(torch.zeros_like(g["x"]), g["logits"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
