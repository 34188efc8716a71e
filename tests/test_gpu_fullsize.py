"""Parity at the full workload sizes, in the launch configuration bench.py
times (MoELayer defaults): routing is compared bit-exactly for every token,
every output must be finite, and the layer output of a chosen sample of
tokens is compared with the oracle computed token by token.

The sample is chosen from the oracle's own routing (never from the GPU's):
the first and the last token, a greedy cover that reaches every expert the
layer touches, and, for the 8 most loaded experts, the tokens of the last
slot and of the first slot of the last 64-, 128- and 256-row token group
(the partial groups a GEMM tile ends on).  Block size changes only how the
GPU tiles the work, not the values, so the oracle output of one routing is
reused for every block size of that layer.

Workloads: Mixtral-shaped prefill (bf16), DeepSeek-V3-shaped prefill (bf16
and a8w8, block sizes 32/64/128, with and without the skewing bias added to
the logits; with its shared expert and the selection-only bias) and the a8w8
decode sweep (T = 1, 16, 64, 256).
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
from moe_inputs import CONFIGS, make_layer, to_numpy
from parity_util import TOL_BF16, TOL_FP8, ExpertView, assert_close, cover_sample

pytestmark = pytest.mark.gpu

DS = CONFIGS["deepseek"]
CASES = [
    ("mixtral", CONFIGS["mixtral"]),
    ("deepseek_bf16_bm32", DS.with_(bm=32)),
    ("deepseek_bf16_bm64", DS),
    ("deepseek_bf16_bm128", DS.with_(bm=128)),
    ("deepseek_a8w8_bm32", DS.with_(a8w8=True, bm=32)),
    ("deepseek_a8w8_bm64", DS.with_(a8w8=True)),
    ("deepseek_a8w8_bm128", DS.with_(a8w8=True, bm=128)),
    ("deepseek_a8w8_bias", DS.with_(a8w8=True, bias=True)),
    ("deepseek_bf16_bias", DS.with_(bias=True)),
    ("deepseek_shared_bf16", CONFIGS["deepseek_shared"]),
    ("deepseek_shared_a8w8", CONFIGS["deepseek_shared"].with_(a8w8=True)),
    ("decode_T1", CONFIGS["decode"].with_(T=1)),
    ("decode_T16", CONFIGS["decode"].with_(T=16)),
    ("decode_T64", CONFIGS["decode"].with_(T=64)),
    ("decode_T256", CONFIGS["decode"].with_(T=256)),
]

# oracle results keyed by the layer without its block size
_ORACLE = {}


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_fullsize_sampled_parity(cuda_device, name, cfg):
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

    key = cfg.with_(bm=0)
    if key not in _ORACLE:
        logits, bias = to_numpy(d["logits"]), to_numpy(d["bias"])
        r_ids, _ = oracle.topk_gate(logits, cfg.k, bias, cfg.bias_mode)
        if cfg.n_shared:
            r_ids, _ = oracle.add_shared(r_ids, _, cfg.E, cfg.n_shared)
        toks, covered, touched = cover_sample(r_ids)
        ref, ref_ids, ref_w = oracle.moe_forward(
            to_numpy(d["x"]), logits, cfg.k, ExpertView(w13, codes=cfg.a8w8), ExpertView(w2, codes=cfg.a8w8),
            bias=bias, a8w8=cfg.a8w8, w13_s=to_numpy(s13), w2_s=to_numpy(s2), tokens=toks, n_shared=cfg.n_shared,
            bias_mode=cfg.bias_mode)
        _ORACLE[key] = (toks, ref, ref_ids, ref_w, covered, touched)
    toks, ref, ref_ids, ref_w, covered, touched = _ORACLE[key]
    print(f"{name}: {len(toks)} sampled tokens reach {covered} of the {touched} touched experts")
    assert covered >= 0.9 * touched
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) <= 1e-6
    got = out[torch.from_numpy(toks).to(cuda_device)].cpu().numpy()
    assert_close(got, ref, TOL_FP8 if cfg.a8w8 else TOL_BF16, name)
