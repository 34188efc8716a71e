"""GPU parity of the MX block-scaled path (GC-MoE abstract: block-scaled,
operand-swapped tensor-core MMAs with FP4 weights on Blackwell; OCP MX
formats) against the MX oracle (oracle/mx_oracle.py):

* the MXFP8 row quantiser: codes and scale codes bit-exact, including zero
  blocks, subnormal and near-overflow magnitudes and saturation;
* the weight-scale tiling: every scale lands where the documented layout says;
* the layer forward with MXFP8 and MXFP4 weights (tiny, ragged and DeepSeek-
  V3-decode shapes) and the stand-alone grouped FFN, element-wise within the
  FP8 tolerance, routing bit-exact.
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle.mx_oracle as mxo
from moe_inputs import CONFIGS, MoEConfig, make_layer, mx_weights, pack_e2m1, to_numpy
from parity_util import TOL_FP8, ExpertView, assert_close

pytestmark = pytest.mark.gpu


def _bf16_rows(R, C, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(R, C, generator=g) * torch.exp2(torch.randint(-20, 20, (R, 1), generator=g).float())
    x[0, :64] = 0.0                                        # two all-zero blocks
    x[1, :32] = torch.tensor(3.0e38)                       # near the bf16 maximum
    x[1, 32:64] = torch.tensor(1.0e-39)                    # subnormal block
    x[2, 5] = -448.0 * 2 ** 10                             # block max lands exactly on 448 * X
    x[3, :32] = torch.linspace(-1, 1, 32)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("R,C", [(7, 64), (64, 256), (33, 7168), (5, 2048)])
def test_mx_quantize_rows_bit_exact(cuda_device, R, C):
    x = _bf16_rows(R, C, seed=R * 1000 + C)
    codes, scales = m.mx_quantize_rows(x.to(cuda_device))
    torch.cuda.synchronize()
    rc, rs = mxo.mx_quantize(to_numpy(x), "e4m3")
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


def test_mx_tile_scales_layout(cuda_device):
    rows, K = 384, 512
    sf = np.random.default_rng(1).integers(0, 255, size=(rows, K // 32), dtype=np.uint8)
    out = m.mx_tile_scales(torch.from_numpy(sf).to(cuda_device)).cpu().numpy().reshape(-1)
    nk = K // 128
    for r in range(rows):
        for kb in range(K // 32):
            chunk = (r // 128) * nk + kb // 4
            off = chunk * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
            assert out[off] == sf[r, kb], (r, kb)


def _mx_layer(cfg, elem, scale_mean, dev):
    """Inputs of cfg with MX weights drawn directly as codes + scales on the
    device (E routed experts; no shared ones).  Returns the make_layer dict,
    the oracle's per-expert views of the unpacked codes and scales, and the
    kernel's operands (E2M1 packed two per byte, scales tiled)."""
    d = make_layer(cfg, device="cpu", weights=False)
    E, H, I = cfg.E, cfg.H, cfg.I
    w13c, w13s = mx_weights(E, 2 * I, H, elem, seed=cfg.seed * 16 + 7, scale_code_mean=scale_mean, device=dev)
    w2c, w2s = mx_weights(E, H, I, elem, seed=cfg.seed * 16 + 8, scale_code_mean=scale_mean, device=dev)
    pack = pack_e2m1 if elem == "e2m1" else (lambda c: c)
    g = dict(x=d["x"].to(dev), logits=d["logits"].to(dev),
             bias=None if d["bias"] is None else d["bias"].to(dev),
             w13=pack(w13c), w2=pack(w2c), w13_sf=m.mx_tile_scales(w13s), w2_sf=m.mx_tile_scales(w2s))
    views = tuple(ExpertView(t, codes=True) for t in (w13c, w13s, w2c, w2s))
    return d, views, g


# Scale codes per element format that give outputs of order 0.1..1 (the layer
# is about cubic in the weight scale): codes drawn uniformly over E4M3 have an
# rms near 100, over E2M1 near 3.
SMALL = {"e4m3": 116, "e2m1": 121}
WIDE = {"e4m3": 114, "e2m1": 119}     # hidden 7168 / inter 2048
MX_CASES = [
    ("tiny", CONFIGS["tiny"], SMALL, None),
    ("ragged", MoEConfig("ragged", T=37, H=384, I=256, E=6, k=3, bm=16, seed=0x5EED0101), SMALL, None),
    ("manytok", MoEConfig("manytok", T=512, H=256, I=128, E=4, k=2, bm=32, seed=0x5EED0102), SMALL, None),
    ("decode_T1", CONFIGS["decode"].with_(T=1, a8w8=False), WIDE, None),
    ("decode_T16", CONFIGS["decode"].with_(T=16, a8w8=False), WIDE, 6),
]


@pytest.mark.parametrize("elem", ["e2m1", "e4m3"])
@pytest.mark.parametrize("name,cfg,smean,n_sample", MX_CASES, ids=[c[0] for c in MX_CASES])
def test_mx_forward_parity(cuda_device, name, cfg, smean, n_sample, elem):
    d, (w13c, w13s, w2c, w2s), g = _mx_layer(cfg, elem, smean[elem], cuda_device)
    mx = "mxfp4" if elem == "e2m1" else "mxfp8"
    layer = m.MoELayer(g["w13"], g["w2"], cfg.k, cfg.bm, out_dtype=torch.float32, mx=mx,
                       w13_mx_scale=g["w13_sf"], w2_mx_scale=g["w2_sf"])
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = layer(g["x"], g["logits"], g["bias"], topk_ids=ids, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    toks = np.arange(cfg.T) if n_sample is None else np.sort(
        np.random.default_rng(cfg.seed).choice(cfg.T, size=n_sample, replace=False))
    ref, ref_ids, _ = mxo.moe_forward_mx(to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k, w13c, w13s, w2c, w2s,
                                         w_elem=elem, bias=to_numpy(d["bias"]), tokens=toks)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    got = out[torch.from_numpy(toks).to(cuda_device)].cpu().numpy()
    err = assert_close(got, ref, TOL_FP8, f"{name} {mx}")
    print(f"{name} {mx}: max abs {err[0]:.2e}, rel fro {err[1]:.2e}, max |ref| {np.abs(ref).max():.2e}")


@pytest.mark.parametrize("elem", ["e2m1", "e4m3"])
def test_mx_grouped_ffn_parity(cuda_device, elem):
    """The stand-alone grouped FFN (its own tile plan) on align & sort's outputs."""
    cfg = MoEConfig("ffn", T=48, H=256, I=256, E=5, k=2, bm=16, seed=0x5EED0103)
    d, (w13c, w13s, w2c, w2s), g = _mx_layer(cfg, elem, SMALL[elem], cuda_device)
    ids, _ = m.topk_gate(g["logits"], cfg.k)
    s, b, n = m.align_sort(ids, cfg.E, cfg.bm)
    y = m.grouped_ffn(g["x"], g["w13"], g["w2"], s, b, n, cfg.k, cfg.bm, mx="mxfp4" if elem == "e2m1" else "mxfp8",
                      w13_mx_scale=g["w13_sf"], w2_mx_scale=g["w2_sf"])
    torch.cuda.synchronize()
    ref = mxo.ffn_mx(to_numpy(d["x"]), ids.cpu().numpy(), w13c, w13s, w2c, w2s, w_elem=elem)
    assert_close(y.cpu().numpy(), ref, TOL_FP8, f"grouped ffn {elem}")


@pytest.mark.parametrize("fmt", ["mxfp4", "mxfp8"])
def test_mx_fullsize_prefill_sampled(cuda_device, fmt):
    """The DeepSeek-V3-shaped prefill layer with MX weights, in the launch
    configuration bench.py times (make_layer's MX weights, bf16 output):
    routing bit-exact, every output finite, and sampled tokens (first, last,
    the last slot of the most loaded expert, random ones) within the FP8
    tolerance of the MX oracle."""
    cfg = CONFIGS["deepseek"].with_(mx=fmt)
    d = make_layer(cfg, device=cuda_device)
    pack = pack_e2m1 if fmt == "mxfp4" else (lambda c: c)
    layer = m.MoELayer(pack(d["w13_codes"]), pack(d["w2_codes"]), cfg.k, cfg.bm, out_dtype=torch.float32, mx=fmt,
                       w13_mx_scale=m.mx_tile_scales(d["w13_sf"]), w2_mx_scale=m.mx_tile_scales(d["w2_sf"]))
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = layer(d["x"], d["logits"], topk_ids=ids, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.isfinite(out).all()
    logits = to_numpy(d["logits"])
    r_ids, _ = mxo.topk_gate(logits, cfg.k)
    flat = r_ids.reshape(-1)
    hot = np.argmax(np.bincount(flat, minlength=cfg.E))
    rng = np.random.default_rng(cfg.seed)
    toks = np.array(sorted({0, cfg.T - 1, int(np.nonzero(flat == hot)[0][-1] // cfg.k),
                            *rng.choice(cfg.T, size=9, replace=False).tolist()}))
    elem = "e2m1" if fmt == "mxfp4" else "e4m3"
    views = [ExpertView(d[k], codes=True) for k in ("w13_codes", "w13_sf", "w2_codes", "w2_sf")]
    ref, ref_ids, _ = mxo.moe_forward_mx(to_numpy(d["x"]), logits, cfg.k, *views, w_elem=elem, tokens=toks)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    got = out[torch.from_numpy(toks).to(cuda_device)].cpu().numpy()
    err = assert_close(got, ref, TOL_FP8, f"deepseek {fmt}")
    print(f"deepseek {fmt}: {len(toks)} tokens, max abs {err[0]:.2e}, rel fro {err[1]:.2e}, "
          f"max |ref| {np.abs(ref).max():.2e}")
