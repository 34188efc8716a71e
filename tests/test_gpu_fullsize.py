"""Parity at the full workload sizes, in the launch configuration bench.py
times (MoELayer defaults): routing is compared bit-exactly for every token,
every output must be finite, and the layer output of a seeded sample of
tokens is compared with the oracle computed token by token.

Workloads: Mixtral-shaped prefill (bf16), DeepSeek-V3-shaped prefill (bf16
and a8w8, block sizes 32/64/128, with and without the skewing bias; with its
shared expert and the selection-only bias) and the a8w8 decode sweep
(T = 1, 16, 64, 256).
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
from moe_inputs import CONFIGS, make_layer, to_numpy
from parity_util import TOL_BF16, TOL_FP8, ExpertView, assert_close

pytestmark = pytest.mark.gpu

CASES = [
    ("mixtral", CONFIGS["mixtral"], 12),
    ("deepseek_bf16_bm64", CONFIGS["deepseek"], 5),
    ("deepseek_a8w8_bm32", CONFIGS["deepseek"].with_(a8w8=True, bm=32), 6),
    ("deepseek_a8w8_bm64", CONFIGS["deepseek"].with_(a8w8=True), 6),
    ("deepseek_a8w8_bm128", CONFIGS["deepseek"].with_(a8w8=True, bm=128), 6),
    ("deepseek_a8w8_bias", CONFIGS["deepseek"].with_(a8w8=True, bias=True), 6),
    ("deepseek_bf16_bias", CONFIGS["deepseek"].with_(bias=True), 4),
    ("deepseek_shared_bf16", CONFIGS["deepseek_shared"], 4),
    ("deepseek_shared_a8w8", CONFIGS["deepseek_shared"].with_(a8w8=True), 4),
    ("decode_T1", CONFIGS["decode"].with_(T=1), 1),
    ("decode_T16", CONFIGS["decode"].with_(T=16), 4),
    ("decode_T64", CONFIGS["decode"].with_(T=64), 4),
    ("decode_T256", CONFIGS["decode"].with_(T=256), 4),
]


@pytest.mark.parametrize("name,cfg,n_sample", CASES, ids=[c[0] for c in CASES])
def test_fullsize_sampled_parity(cuda_device, name, cfg, n_sample):
    d = make_layer(cfg, device=cuda_device)
    if cfg.a8w8:
        w13, w2, s13, s2 = d["w13_q"], d["w2_q"], d["w13_s"], d["w2_s"]
    else:
        w13, w2, s13, s2 = d["w13"], d["w2"], None, None
    layer = m.MoELayer(w13, w2, cfg.k, cfg.bm, s13, s2, out_dtype=torch.float32, n_shared=cfg.n_shared,
                       bias_mode=cfg.bias_mode)
    ids = torch.empty(cfg.T, cfg.k + cfg.n_shared, dtype=torch.int32, device=cuda_device)
    tw = torch.empty(cfg.T, cfg.k + cfg.n_shared, dtype=torch.float32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = layer(d["x"], d["logits"], d["bias"], topk_ids=ids, topk_w=tw, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.isfinite(out).all()
    rng = np.random.default_rng(cfg.seed)
    toks = np.sort(rng.choice(cfg.T, size=min(n_sample, cfg.T), replace=False))
    ref, ref_ids, ref_w = oracle.moe_forward(
        to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k, ExpertView(w13, codes=cfg.a8w8),
        ExpertView(w2, codes=cfg.a8w8), bias=to_numpy(d["bias"]), a8w8=cfg.a8w8,
        w13_s=to_numpy(s13), w2_s=to_numpy(s2), tokens=toks, n_shared=cfg.n_shared, bias_mode=cfg.bias_mode)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) <= 1e-6
    got = out[torch.from_numpy(toks).to(cuda_device)].cpu().numpy()
    assert_close(got, ref, TOL_FP8 if cfg.a8w8 else TOL_BF16, name)
