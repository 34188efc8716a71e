"""Routing metadata that a caller hands to moe_grouped_ffn itself (not the
output of moe_align_sort): invalid entries stay inside the buffers and are
reported in the device status word.

- a negative slot id in sorted_ids: the row is skipped like padding in both
  builds, and the MOE_DEBUG build (libmoe_b200_debug.so) reports
  MOE_DEV_BOUNDS;
- an expert whose blocks form two runs in expert_ids, or a num_post outside
  [0, len(sorted_ids)] or off the block size: MOE_DEV_BAD_PLAN, and no GEMM
  tile runs (y is not written).

Every index these inputs reach was checked against its buffer by reading the
kernels: the gathers and quantisers treat an id outside [0, T*k) as padding
and clamp their row count to the buffer; the plan drops an invalid plan
before any tile is claimed; the GEMM epilogue writes only ids in [0, T*k).

The last test runs this file and the FFN / forward / backward parity files
again in a child process on the debug build: its checks must stay silent on
valid inputs, and its results match the oracle.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
from mixture_experts_expert_moe_b200 import build_lib
from moe_inputs import MoEConfig, make_layer, pack_e2m1, to_numpy
from parity_util import TOL_BF16, TOL_FP8, assert_close

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG = os.path.abspath(m.LIB_PATH) == os.path.abspath(build_lib.DEBUG_LIB)
CFG = MoEConfig("ragged", T=300, H=384, I=256, E=16, k=4, bm=32, seed=101)


def _layer(kind, dev):
    """The layer's inputs on ``dev`` and grouped_ffn's weight arguments."""
    if kind in ("mxfp8", "mxfp4"):
        cfg = CFG.with_(mx=kind, H=512)
        d = make_layer(cfg, device=dev)
        pack = pack_e2m1 if kind == "mxfp4" else (lambda c: c)
        w = dict(w13=pack(d["w13_codes"]), w2=pack(d["w2_codes"]), mx=kind,
                 w13_mx_scale=m.mx_tile_scales(d["w13_sf"]), w2_mx_scale=m.mx_tile_scales(d["w2_sf"]))
        return cfg, d, w
    cfg = CFG.with_(a8w8=kind == "a8w8")
    d = make_layer(cfg, device=dev)
    if cfg.a8w8:
        return cfg, d, dict(w13=d["w13_q"], w2=d["w2_q"], w13_scale=d["w13_s"], w2_scale=d["w2_s"])
    return cfg, d, dict(w13=d["w13"], w2=d["w2"])


def _ffn(cfg, d, w, s, b, n, st):
    """grouped_ffn into a NaN-filled y (rows it does not write stay NaN)."""
    kw = dict(w)
    w13, w2 = kw.pop("w13"), kw.pop("w2")
    y = torch.full((cfg.T * cfg.k, cfg.H), float("nan"), dtype=torch.float32, device=d["x"].device)
    m.grouped_ffn(d["x"], w13, w2, s, b, n, cfg.k, cfg.bm, dev_status=st, y=y, **kw)
    torch.cuda.synchronize()
    return y


def _route(cfg, d):
    ids, _ = m.topk_gate(d["logits"], cfg.k, d["bias"])
    s, b, n = m.align_sort(ids, cfg.E, cfg.bm)
    torch.cuda.synchronize()
    return ids, s, b, n


@pytest.mark.parametrize("kind", ["bf16", "a8w8", "mxfp8", "mxfp4"])
def test_negative_slot_ids_are_skipped(cuda_device, kind):
    cfg, d, w = _layer(kind, cuda_device)
    ids, s, b, n = _route(cfg, d)
    N = cfg.T * cfg.k
    sh = s.cpu()
    real = torch.nonzero((sh >= 0) & (sh < N)).flatten()
    rng = np.random.default_rng(0x1D5)
    pick = torch.from_numpy(rng.choice(real.numpy(), size=len(real) // 10, replace=False))
    dropped = sh[pick].clone()
    bad, pad = sh.clone(), sh.clone()
    bad[pick] = torch.from_numpy(rng.choice([-1, -7, -N, -(2 ** 31)], size=len(pick)).astype(np.int32))
    pad[pick] = N
    st_bad = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    st_pad = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    y_bad = _ffn(cfg, d, w, bad.to(cuda_device), b, n, st_bad)
    y_pad = _ffn(cfg, d, w, pad.to(cuda_device), b, n, st_pad)
    assert int(st_pad.item()) == 0
    assert int(st_bad.item()) == (m.MOE_DEV_BOUNDS if DEBUG else 0)
    # the same plan and the same gathered rows: the kept slots match bit for bit
    nan_bad, nan_pad = torch.isnan(y_bad), torch.isnan(y_pad)
    assert torch.equal(nan_bad, nan_pad)
    assert torch.equal(y_bad[~nan_bad], y_pad[~nan_pad])
    # the dropped slots were not written; every other slot was
    written = ~nan_bad.all(dim=1).cpu()
    expect = torch.ones(N, dtype=torch.bool)
    expect[dropped.long()] = False
    assert torch.equal(written, expect)
    if kind in ("bf16", "a8w8"):
        ref_ids = ids.cpu().numpy()
        ref = (oracle.ffn_a8w8(to_numpy(d["x"]), ref_ids, to_numpy(d["w13_q"]), to_numpy(d["w13_s"]),
                               to_numpy(d["w2_q"]), to_numpy(d["w2_s"])) if kind == "a8w8"
               else oracle.ffn_bf16(to_numpy(d["x"]), ref_ids, to_numpy(d["w13"]), to_numpy(d["w2"])))
        keep = expect.numpy()
        assert_close(y_bad.cpu().numpy()[keep], ref[keep], TOL_FP8 if kind == "a8w8" else TOL_BF16, kind)


def _split_runs(b_host, nb):
    """expert_ids with one expert's blocks split into two runs (a block of
    another expert moved between them), or None if the plan has too few."""
    e = b_host[:nb].tolist()
    for i in range(1, nb - 1):
        if e[i - 1] == e[i] and e[i + 1] != e[i]:
            out = b_host.clone()
            out[i], out[i + 1] = e[i + 1], e[i]
            return out
    return None


@pytest.mark.parametrize("kind", ["bf16", "a8w8"])
def test_split_expert_runs_are_a_bad_plan(cuda_device, kind):
    cfg, d, w = _layer(kind, cuda_device)
    _, s, b, n = _route(cfg, d)
    nb = int(n.item()) // cfg.bm
    bad_b = _split_runs(b.cpu(), nb)
    assert bad_b is not None, "the routing has no expert with two blocks next to another expert"
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    y = _ffn(cfg, d, w, s, bad_b.to(cuda_device), n, st)
    assert int(st.item()) == m.MOE_DEV_BAD_PLAN
    assert torch.isnan(y).all(), "an invalid plan ran GEMM tiles"
    # the stream and the context stay usable: the valid plan runs afterwards
    st.zero_()
    y = _ffn(cfg, d, w, s, b, n, st)
    assert int(st.item()) == 0 and not torch.isnan(y).all()


@pytest.mark.parametrize("kind", ["bf16", "a8w8"])
@pytest.mark.parametrize("which", ["past_end", "negative", "off_block"])
def test_num_post_outside_the_buffer_is_a_bad_plan(cuda_device, kind, which):
    cfg, d, w = _layer(kind, cuda_device)
    _, s, b, n = _route(cfg, d)
    P = s.numel()
    bad = {"past_end": P + cfg.bm, "negative": -cfg.bm, "off_block": int(n.item()) - 1}[which]
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    y = _ffn(cfg, d, w, s, b, torch.tensor([bad], dtype=torch.int32, device=cuda_device), st)
    assert int(st.item()) == m.MOE_DEV_BAD_PLAN
    assert torch.isnan(y).all()


def test_debug_build_checks_stay_silent_on_valid_inputs(cuda_device):
    """The parity files (and this one, expecting MOE_DEV_BOUNDS for negative
    ids) on libmoe_b200_debug.so, in a child process."""
    if DEBUG:
        pytest.skip("already running on the debug build")
    if not os.path.exists(build_lib.DEBUG_LIB):
        build_lib.build(debug=True)
    env = dict(os.environ, MOE_B200_LIB=build_lib.DEBUG_LIB)
    files = ["tests/test_gpu_invalid_routing.py", "tests/test_gpu_ffn.py", "tests/test_gpu_gate_align.py",
             "tests/test_gpu_backward.py", "tests/test_gpu_ep.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
