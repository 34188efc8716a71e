"""Backward parity at the DeepSeek-V3 layer's full size (T=2048, hidden 7168,
inter 2048, 256 experts, top-8, block 64, bf16), in the configuration
bench.py times: every gradient must be finite, experts no token reached get
zero weight gradients, and the oracle (restricted to a sample, each computed
entry the same sum as the full oracle's) is matched element by element on
the dx and dlogits rows of sampled tokens and on the whole dW13 / dW2 of the
most loaded, a median and the least loaded touched expert.  The sample is
chosen from the oracle's routing.
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
import oracle.backward_oracle as bo
from moe_inputs import CONFIGS, make_layer, normal, to_numpy
from parity_util import TOL_BF16, assert_close_scaled

pytestmark = pytest.mark.gpu


class _Experts:
    """float64 view of a device weight tensor: the listed experts converted
    once and kept, others on each access."""

    def __init__(self, t, keep):
        self.t = t
        self.shape = tuple(t.shape)
        self.kept = {int(e): t[int(e)].cpu().double().numpy() for e in keep}

    def __getitem__(self, e):
        e = int(e)
        return self.kept[e] if e in self.kept else self.t[e].cpu().double().numpy()


def test_backward_fullsize_sampled(cuda_device):
    cfg = CONFIGS["deepseek"]
    d = make_layer(cfg, device=cuda_device)
    dout = normal((cfg.T, cfg.H), 1.0, cfg.seed * 16 + 9, cuda_device, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    dx, dl, dw13, dw2 = m.backward(d["x"], d["logits"], d["w13"], d["w2"], dout, cfg.k, cfg.bm, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for g in (dx, dl, dw13, dw2):
        assert torch.isfinite(g).all()

    logits = to_numpy(d["logits"])
    ids, _ = oracle.topk_gate(logits, cfg.k)
    counts = np.bincount(ids.reshape(-1), minlength=cfg.E)
    touched = np.nonzero(counts)[0]
    for e in np.nonzero(counts == 0)[0]:
        assert float(dw13[e].abs().max()) == 0.0 and float(dw2[e].abs().max()) == 0.0
    by_load = touched[np.argsort(counts[touched], kind="stable")]
    exps = sorted({int(by_load[-1]), int(by_load[len(by_load) // 2]), int(by_load[0])})
    rng = np.random.default_rng(cfg.seed)
    toks = sorted({0, cfg.T - 1, *rng.choice(cfg.T, size=2, replace=False).tolist()})
    rdx, rdl, rdw13, rdw2 = bo.moe_backward(to_numpy(d["x"]), logits, cfg.k, _Experts(d["w13"], exps),
                                            _Experts(d["w2"], exps), to_numpy(dout), tokens=toks, experts=exps)
    t_idx = torch.tensor(toks, device=cuda_device)
    for what, got, ref in (("dx", dx[t_idx], rdx[toks]), ("dlogits", dl[t_idx], rdl[toks])):
        err = assert_close_scaled(got.cpu().numpy(), ref, TOL_BF16, f"deepseek backward {what}")
        print(f"{what}: max abs {err[0]:.2e}, rel fro {err[1]:.2e}, max |ref| {np.abs(ref).max():.2e}")
    for e in exps:
        for what, got, ref in (("dw13", dw13[e], rdw13[e]), ("dw2", dw2[e], rdw2[e])):
            err = assert_close_scaled(got.cpu().numpy(), ref, TOL_BF16, f"deepseek backward {what}[{e}]")
            print(f"{what}[expert {e}, {counts[e]} slots]: max abs {err[0]:.2e}, rel fro {err[1]:.2e}, "
                  f"max |ref| {np.abs(ref).max():.2e}")
