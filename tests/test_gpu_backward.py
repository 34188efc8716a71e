"""GPU parity of the layer's backward pass (moe_backward, bf16 weights)
against the backward oracle (oracle/backward_oracle.py, float64): dx,
dlogits, dW13 and dW2 element by element within the bf16 tolerance, on small
layers that span several tiles and a ragged tail, with both bias modes and a
shared expert.  The oracle is pinned by torch autograd and finite differences
(tests/test_oracle_backward.py).
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle.backward_oracle as bo
from moe_inputs import CONFIGS, MoEConfig, make_layer, normal, to_numpy
from parity_util import TOL_BF16, assert_close_scaled

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", CONFIGS["tiny"]),
    ("ragged", MoEConfig("ragged", T=37, H=384, I=256, E=6, k=3, bm=16, seed=0x5EED0201)),
    ("manytok", MoEConfig("manytok", T=300, H=256, I=128, E=4, k=2, bm=32, seed=0x5EED0202)),
    ("wide", MoEConfig("wide", T=24, H=1024, I=512, E=16, k=4, bm=16, seed=0x5EED0203)),
    ("bias_logits", MoEConfig("bias_logits", T=48, H=256, I=256, E=8, k=2, bm=16, bias=True,
                              seed=0x5EED0204)),
    ("shared_select", MoEConfig("shared_select", T=40, H=256, I=128, E=8, k=2, bm=16, bias=True, n_shared=1,
                                bias_mode="select", seed=0x5EED0205)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_backward_parity(cuda_device, name, cfg):
    d = make_layer(cfg, device=cuda_device)
    dout = normal((cfg.T, cfg.H), 1.0, cfg.seed * 16 + 9, cuda_device, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    dx, dl, dw13, dw2 = m.backward(d["x"], d["logits"], d["w13"], d["w2"], dout, cfg.k, cfg.bm, bias=d["bias"],
                                   bias_mode=cfg.bias_mode, n_shared=cfg.n_shared, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rdx, rdl, rdw13, rdw2 = bo.moe_backward(to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k, to_numpy(d["w13"]),
                                            to_numpy(d["w2"]), to_numpy(dout), bias=to_numpy(d["bias"]),
                                            bias_mode=cfg.bias_mode, n_shared=cfg.n_shared)
    for what, got, ref in (("dx", dx, rdx), ("dlogits", dl, rdl), ("dw13", dw13, rdw13), ("dw2", dw2, rdw2)):
        err = assert_close_scaled(got.cpu().numpy(), ref, TOL_BF16, f"{name} {what}")
        print(f"{name} {what}: max abs {err[0]:.2e}, rel fro {err[1]:.2e}, max |ref| {np.abs(ref).max():.2e}")
    # experts no token reached get exactly zero weight gradients
    used = np.unique(bo.topk_gate(to_numpy(d["logits"]), cfg.k, to_numpy(d["bias"]), cfg.bias_mode)[0])
    unused = [e for e in range(cfg.E) if e not in used]
    for e in unused:
        assert float(dw13[e].abs().max()) == 0.0 and float(dw2[e].abs().max()) == 0.0


def test_backward_repeatable_and_no_tokens(cuda_device):
    """Two calls give the same weight gradients up to the order of fp32
    additions; an empty batch zeroes the weight gradients."""
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg, device=cuda_device)
    dout = normal((cfg.T, cfg.H), 1.0, 77, cuda_device, torch.bfloat16)
    a = m.backward(d["x"], d["logits"], d["w13"], d["w2"], dout, cfg.k, cfg.bm)
    b = m.backward(d["x"], d["logits"], d["w13"], d["w2"], dout, cfg.k, cfg.bm)
    torch.cuda.synchronize()
    for u, v in zip(a[2:], b[2:]):
        assert torch.equal(u, v)          # weight gradients: one MMA chain per element, deterministic
    e = m.backward(d["x"][:0], d["logits"][:0], d["w13"], d["w2"], dout[:0], cfg.k, cfg.bm)
    torch.cuda.synchronize()
    assert float(e[2].abs().max()) == 0.0 and float(e[3].abs().max()) == 0.0
