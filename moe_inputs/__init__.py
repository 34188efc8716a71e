"""Seeded synthetic inputs for the MoE layer forward.

Shared by the tests, ``bench.py``, ``__graft_entry__.smoke()`` and the CPU
oracle.  This module draws random numbers and lays them out; it contains
none of the layer's arithmetic (no gating, sorting, FFN or combine).

Recipes (workload shapes from the MoE Align & Sort article's DeepSeek-V3
workloads -- E=256, top-8 -- and the aiter a8w8 issue's hidden 7168 /
inter 2048 shape):

* activations ``x`` ~ N(0, 1), rounded to bf16 by torch's cast;
* expert weights ~ N(0, 0.02), generated directly in the library's
  K-contiguous layout ``w13 [E, 2I, H]`` (rows 0..I-1 gate, I..2I-1 up) and
  ``w2 [E, H, I]``; the entries are i.i.d., so the layout is only a choice
  of which random number lands where;
* FP8 weights: model preparation, not part of the forward pass.  Per output
  channel the fp32 draw is divided by ``amax / 448`` and cast to E4M3FN by
  torch (after clamping to +-448); the codes and the fp32 scales are the
  layer's parameters and both sides read the same bytes;
* router logits: ``x @ Wr`` with Wr ~ N(0, 0.02) in fp32 for the tiny
  layer, i.i.d. N(0, 1) otherwise (so the top-k set is a uniformly random
  k-subset); the skewed variant adds a per-expert N(0, 1) bias;
* shared experts (DeepSeek-V3 has one) are drawn like the routed ones and
  stored after them in the same weight tensors;
* align-only ids: k distinct experts per token drawn one after another
  without replacement from Zipf(s) popularity over a seeded permutation of
  the experts (Gumbel-top-k, which has exactly that law), or uniformly.

Large weights are drawn on the target device with a seeded
``torch.Generator`` on that device.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

SEED_BASE = 0x5EED0000


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    bm: int
    a8w8: bool = False
    bias: bool = False
    router: str = "normal"      # "normal": logits ~ N(0,1); "linear": x @ Wr
    seed: int = SEED_BASE
    n_shared: int = 0           # always-on shared experts stored after the E routed ones
    bias_mode: str = "logits"   # "logits": bias feeds selection and weights; "select": selection only
    mx: str = ""                # "mxfp8" / "mxfp4": MX block-scaled weights drawn as codes + scales

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


CONFIGS = {
    # tiny layer used for full parity
    "tiny": MoEConfig("tiny", T=64, H=256, I=128, E=8, k=2, bm=16,
                      router="linear", seed=SEED_BASE + 0),
    # Mixtral-shaped prefill, bf16
    "mixtral": MoEConfig("mixtral", T=4096, H=4096, I=14336, E=8, k=2, bm=128,
                         seed=SEED_BASE + 2),
    # DeepSeek-V3-shaped prefill (uniform routing); a8w8 / bias / bm variants
    "deepseek": MoEConfig("deepseek", T=2048, H=7168, I=2048, E=256, k=8, bm=64,
                          seed=SEED_BASE + 3),
    # the aiter a8w8 issue's shape: 32 local experts, ~64 tokens each
    "p5": MoEConfig("p5", T=256, H=7168, I=2048, E=32, k=8, bm=64, seed=SEED_BASE + 5),
    # DeepSeek-V3-shaped layer with its shared expert and the selection-only
    # gating bias (aux-loss-free balancing)
    "deepseek_shared": MoEConfig("deepseek_shared", T=2048, H=7168, I=2048, E=256, k=8, bm=64,
                                 bias=True, n_shared=1, bias_mode="select", seed=SEED_BASE + 6),
    # decode sweep, FP8 a8w8 (T in 1, 16, 64, 256)
    "decode": MoEConfig("decode", T=64, H=7168, I=2048, E=256, k=8, bm=16,
                        a8w8=True, seed=SEED_BASE + 4),
}

# E8M0 scale code around which MX weight scales are drawn (codes uniform over
# E4M3 have an rms near 100, over E2M1 near 3)
MX_SCALE_CODE = {"mxfp8": 114, "mxfp4": 119}

ALIGN_CONFIG = dict(T=16384, E=256, k=8, bm=64, zipf_s=1.0, seed=SEED_BASE + 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std, seed, device="cpu", dtype=torch.float32):
    g = _gen(device, seed)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(dtype)


def fp8_weights(E, rows, cols, std, seed, device="cpu"):
    """E4M3FN codes [E, rows, cols] and fp32 per-row scales [E, rows]."""
    codes = torch.empty(E, rows, cols, dtype=torch.float8_e4m3fn, device=device)
    scales = torch.empty(E, rows, dtype=torch.float32, device=device)
    g = _gen(device, seed)
    for e in range(E):
        w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
        amax = w.abs().amax(dim=1)
        s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        codes[e] = (w / s[:, None]).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
        scales[e] = s
    return codes, scales


def mx_weights(E, rows, cols, elem, seed, scale_code_mean=122, device=None):
    """MX block-scaled weights drawn directly (no quantisation step): uint8
    element codes [E, rows, cols] uniform over the finite codes of `elem`
    ("e2m1": 4-bit codes 0..15; "e4m3": the E4M3FN codes except NaN), and
    E8M0 scale codes [E, rows, cols/32] = scale_code_mean + {-1, 0, +1}
    (powers of two around 2^(mean-127)).

    device None: numpy arrays from a numpy generator; a torch device: uint8
    tensors drawn there by a seeded torch generator (for large layers; the
    two paths draw different, equally distributed values)."""
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    if elem not in ("e2m1", "e4m3"):
        raise ValueError(elem)
    if device is not None:
        g = _gen(device, seed)
        hi = 16 if elem == "e2m1" else 255
        codes = torch.randint(0, hi, (E, rows, cols), generator=g, device=device, dtype=torch.uint8)
        if elem == "e4m3":
            codes[(codes & 0x7F) == 0x7F] = 0          # no NaN codes
        off = torch.randint(-1, 2, (E, rows, cols // 32), generator=g, device=device, dtype=torch.int32)
        return codes, (scale_code_mean + off).to(torch.uint8)
    rng = np.random.default_rng(seed)
    if elem == "e2m1":
        codes = rng.integers(0, 16, size=(E, rows, cols), dtype=np.uint8)
    else:
        codes = rng.integers(0, 255, size=(E, rows, cols), dtype=np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0          # no NaN codes
    scales = (scale_code_mean + rng.integers(-1, 2, size=(E, rows, cols // 32))).astype(np.uint8)
    return codes, scales


def pack_e2m1(codes):
    """E2M1 codes (uint8 values 0..15) [..., K] packed two per byte [..., K/2]:
    element 2j in the low nibble, 2j+1 in the high nibble (the layout the MX
    kernels read; packing only moves bits).  numpy array or torch tensor."""
    if codes.shape[-1] % 2:
        raise ValueError("K must be even")
    if isinstance(codes, torch.Tensor):
        return ((codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)).contiguous()
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)


def make_layer(cfg: MoEConfig, device="cpu", weights=True):
    """All inputs of one MoE layer forward for ``cfg``.

    Returns a dict with x (bf16 [T,H]), logits (f32 [T,E]), bias (f32 [E] or
    None) and, when ``weights``: w13/w2 (bf16) or w13_q/w13_s/w2_q/w2_s
    (float8_e4m3fn codes + f32 scales) for the E routed experts followed by
    the cfg.n_shared shared ones.
    """
    T, H, I, E = cfg.T, cfg.H, cfg.I, cfg.E
    EW = E + cfg.n_shared
    s = cfg.seed
    d = {}
    d["x"] = normal((T, H), 1.0, s * 16 + 1, device, torch.bfloat16)
    if cfg.router == "linear":
        wr = normal((H, E), 0.02, s * 16 + 2, device)
        d["logits"] = (d["x"].float() @ wr).contiguous()
    else:
        d["logits"] = normal((T, E), 1.0, s * 16 + 3, device)
    d["bias"] = normal((E,), 1.0, s * 16 + 4, device) if cfg.bias else None
    if weights:
        if cfg.mx:
            # MX weights drawn directly as codes + E8M0 scales, scale codes
            # chosen so the layer's outputs are of order 0.1..1 at hidden 7168
            elem = "e2m1" if cfg.mx == "mxfp4" else "e4m3"
            mean = MX_SCALE_CODE[cfg.mx]
            d["w13_codes"], d["w13_sf"] = mx_weights(EW, 2 * I, H, elem, s * 16 + 7, mean, device=device)
            d["w2_codes"], d["w2_sf"] = mx_weights(EW, H, I, elem, s * 16 + 8, mean, device=device)
        elif cfg.a8w8:
            d["w13_q"], d["w13_s"] = fp8_weights(EW, 2 * I, H, 0.02, s * 16 + 5, device)
            d["w2_q"], d["w2_s"] = fp8_weights(EW, H, I, 0.02, s * 16 + 6, device)
        else:
            d["w13"] = normal((EW, 2 * I, H), 0.02, s * 16 + 5, device, torch.bfloat16)
            d["w2"] = normal((EW, H, I), 0.02, s * 16 + 6, device, torch.bfloat16)
    return d


def align_ids(T, E, k, seed, dist="zipf", zipf_s=1.0):
    """int32 [T, k]: k distinct experts per token.

    ``zipf``: popularity of the expert at rank r (r = 1..E, ranks assigned by
    a seeded permutation) is proportional to r**-s; the k experts are drawn
    one after another without replacement, renormalising each time.  The
    Gumbel-top-k construction (keys log p + Gumbel noise, take the k largest
    in descending order) has exactly that distribution.  ``uniform``: every
    expert equally likely.
    """
    rng = np.random.default_rng(seed)
    perm = rng.permutation(E)
    if dist == "zipf":
        p_rank = np.arange(1, E + 1, dtype=np.float64) ** (-zipf_s)
        logp = np.empty(E)
        logp[perm] = np.log(p_rank)            # expert perm[r] has rank r+1
    elif dist == "uniform":
        logp = np.zeros(E)
    else:
        raise ValueError(dist)
    keys = logp[None, :] + rng.gumbel(size=(T, E))
    top = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    return top.astype(np.int32)


def to_numpy(t):
    """float64 / int numpy view of a (possibly device, bf16 or fp8) tensor."""
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.float().numpy().astype(np.float64)
    return t.numpy()
