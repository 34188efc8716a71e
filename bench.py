#!/usr/bin/env python
"""Benchmark of the MoE layer forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full layer forward through the C ABI (``moe_forward``): top-k
gating, align & sort, gather, gate/up GEMM with SiLU*mul, down GEMM with the
per-slot expert outputs, weighted combine.  The headline workload is the
DeepSeek-V3-shaped prefill layer (T=2048 tokens, hidden 7168, inter 2048,
256 experts, top-8, block 64, bf16, router logits ~ N(0,1)).  Its expert
weights (22.5 GB) are far larger than L2, so no flush is needed between
steps.  Extra objects in the line report the a8w8 variant, the
Mixtral-shaped prefill, the a8w8 decode sweep and align & sort alone
(16384 tokens, top-8 of 256, Zipf s=1, block 64; L2 flushed between calls).

Multi-GPU: the layer does not shard here, so N GPUs run N independent
replicas ("scaling": "weak"); the time is the maximum over ranks.

``--impl reference`` times the CPU oracle (float64 numpy) on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import ALIGN_CONFIG, CONFIGS, align_ids, make_layer, pack_e2m1  # noqa: E402
from mixture_experts_expert_moe_b200.roofline import (  # noqa: E402
    align_bytes, backward_bytes, backward_flops, down_kernel_bytes, gateup_kernel_bytes, layer_bytes, moe_flops)

METRIC = "MoE layer tokens/s & TFLOPS vs roofline (bf16/fp8); align&sort µs, GB/s"
PRIMARY = CONFIGS["deepseek"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_name(cfg, dtype):
    bias = ""
    if cfg.bias:
        bias = " +bias(selection only)" if cfg.bias_mode == "select" else " +bias"
    shared = f" +{cfg.n_shared} shared" if cfg.n_shared else ""
    return (f"{cfg.name}_{dtype}: T={cfg.T} H={cfg.H} I={cfg.I} E={cfg.E} k={cfg.k} bm={cfg.bm}"
            f"{bias}{shared}")


def slot_pairs(cfg):
    """(token, expert) pairs the FFN computes: k routed + the shared experts."""
    return cfg.T * (cfg.k + cfg.n_shared)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"moe_bench_clocks_{os.getpid()}.csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu = str(device.index or 0)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            lines = f.readlines()
        os.remove(self.path)
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        smax = max(r[1] for r in rows)
        load = [r for r in rows if r[2] > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in load])), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def build_layer(m, cfg, dev, out_dtype=torch.bfloat16, tile_tokens=0, data=None):
    d = make_layer(cfg, device=dev) if data is None else data
    if cfg.mx:
        # model preparation: E2M1 codes packed two per byte, scales tiled for the MMA
        pack = pack_e2m1 if cfg.mx == "mxfp4" else (lambda c: c)
        w13, w2 = pack(d["w13_codes"]), pack(d["w2_codes"])
        s13, s2 = m.mx_tile_scales(d["w13_sf"]), m.mx_tile_scales(d["w2_sf"])
        for key in ("w13_codes", "w2_codes", "w13_sf", "w2_sf"):    # the packed / tiled copies replace them
            del d[key]
        layer = m.MoELayer(w13, w2, cfg.k, cfg.bm, out_dtype=out_dtype, tile_tokens=tile_tokens,
                           n_shared=cfg.n_shared, bias_mode=cfg.bias_mode, mx=cfg.mx, w13_mx_scale=s13,
                           w2_mx_scale=s2)
    elif cfg.a8w8:
        layer = m.MoELayer(d["w13_q"], d["w2_q"], cfg.k, cfg.bm, d["w13_s"], d["w2_s"], out_dtype=out_dtype,
                           tile_tokens=tile_tokens, n_shared=cfg.n_shared, bias_mode=cfg.bias_mode)
    else:
        layer = m.MoELayer(d["w13"], d["w2"], cfg.k, cfg.bm, out_dtype=out_dtype, tile_tokens=tile_tokens,
                           n_shared=cfg.n_shared, bias_mode=cfg.bias_mode)
    return d, layer


def touched_experts(layer, d):
    ids = torch.empty(d["x"].shape[0], layer.k + layer.n_shared, dtype=torch.int32, device=d["x"].device)
    layer(d["x"], d["logits"], d["bias"], topk_ids=ids)
    torch.cuda.synchronize()
    return int(torch.unique(ids).numel()), ids


def max_over_ranks(value, device):
    """The largest of every rank's value (the value itself in a one-process
    run); every rank must call it, in the same order."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, steps, ms):
    """Whole-job units/s of `world` replicas that each process `units_per_rank`
    units per step, `steps` steps in `ms` milliseconds (the max over ranks)."""
    return world * units_per_rank * steps / (ms * 1e-3)


def kernels_per_step(cfg, out_dtype):
    """Kernels of this library one moe_forward launches: the routing kernel
    (gate + align + plan), the gather, the gate/up and down GEMMs and the
    combine; a8w8 adds the requantisation, and above 4096 slots it
    quantises each token once before the gather instead of inside it.  (The
    memset of the routing kernel's grid-wait counter is a runtime call, not a
    kernel of this library.)"""
    n = 5
    if cfg.a8w8 and not cfg.mx:
        n += 1 + (1 if slot_pairs(cfg) > 4096 else 0)
    return n


def time_layer(m, cfg, layer, d, steps, warmup, stage_times=True):
    dev = d["x"].device
    out = torch.empty(cfg.T, cfg.H, dtype=layer.out_dtype, device=dev)
    for _ in range(warmup):
        layer(d["x"], d["logits"], d["bias"], out=out)
    nst = len(m.STAGES) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(steps)] if stage_times else None
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        layer(d["x"], d["logits"], d["bias"], out=out, stage_events=evs[i] if evs else None)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    st = None
    if evs:
        st = {name: float(np.mean([e[j].elapsed_time(e[j + 1]) for e in evs])) for j, name in enumerate(m.STAGES)}
    return ms, st


def time_graph(m, cfg, layer, d, steps, warmup):
    """Replays of one captured forward (CUDA graph); None if capture fails."""
    out = torch.empty(cfg.T, cfg.H, dtype=layer.out_dtype, device=d["x"].device)
    try:
        g, _ = m.capture_graph(layer, d["x"], d["logits"], d["bias"], out=out)
    except Exception as exc:  # report eager numbers only
        sys.stderr.write(f"graph capture failed: {exc}\n")
        return None
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        g.replay()
    t1.record()
    torch.cuda.synchronize()
    del g
    return t0.elapsed_time(t1)


def time_e2e(cfg, layer, d, steps, warmup):
    """Same layer through the C ABI with host buffers: pinned x and logits
    copied in and the output copied out inside the timed region."""
    dev = d["x"].device
    xh = d["x"].cpu().pin_memory()
    lh = d["logits"].cpu().pin_memory()
    oh = torch.empty(cfg.T, cfg.H, dtype=layer.out_dtype).pin_memory()
    xd, ld = torch.empty_like(d["x"]), torch.empty_like(d["logits"])
    out = torch.empty(cfg.T, cfg.H, dtype=layer.out_dtype, device=dev)

    def step():
        xd.copy_(xh, non_blocking=True)
        ld.copy_(lh, non_blocking=True)
        layer(xd, ld, d["bias"], out=out)
        oh.copy_(out, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    h2d = xh.numel() * xh.element_size() + lh.numel() * lh.element_size()
    d2h = oh.numel() * oh.element_size()
    return ms, h2d, d2h


def gateup_bytes(cfg, touched):
    """Algorithmic bytes of one gate/up GEMM launch (touched gate+up weights
    once, x once, routing)."""
    return gateup_kernel_bytes(cfg.T, cfg.H, cfg.I, touched, slot_pairs(cfg), cfg.a8w8, cfg.mx)


def down_bytes(cfg, touched):
    """Algorithmic bytes of one down GEMM launch (touched down weights once,
    fp32 token outputs once, routing)."""
    return down_kernel_bytes(cfg.T, cfg.H, cfg.I, touched, slot_pairs(cfg), cfg.a8w8, cfg.mx)


TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "traffic.json")


def traffic_for(kernel, workload, table=TRAFFIC_TABLE):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu traffic table, only while the kernel source still
    has the hash recorded with the capture; None otherwise."""
    if not os.path.exists(table):
        return None
    with open(table) as f:
        entries = json.load(f)["entries"]
    for ent in entries:
        if ent["kernel"] != kernel or ent["workload"] != workload:
            continue
        src = os.path.join(ROOT, ent["source"])
        if not os.path.exists(src):
            return None
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return int(ent["bytes_per_launch"]) if h == ent["sha256_16"] else None
    return None


def layer_report(m, cfg, steps, warmup, dev, pk, dtype_name, primary=False, tile_tokens=0, data=None):
    """Time one workload (eager with stage events, then CUDA-graph replay) and
    report it against its layer roofline and its dominant kernel's roofline.
    ``data``: inputs from make_layer(cfg) to reuse (block-size sweeps)."""
    d, layer = build_layer(m, cfg, dev, tile_tokens=tile_tokens, data=data)
    touched, ids = touched_experts(layer, d)
    load = torch.bincount(ids[:, :cfg.k].reshape(-1).long(), minlength=cfg.E)
    ms_eager, st = time_layer(m, cfg, layer, d, steps, warmup)
    ms_graph = time_graph(m, cfg, layer, d, steps, warmup)
    ms = ms_graph if ms_graph is not None else ms_eager
    step_ms = ms / steps
    pairs = slot_pairs(cfg)
    fl = moe_flops(pairs, cfg.H, cfg.I)
    by = layer_bytes(cfg.T, cfg.H, cfg.E, cfg.k + cfg.n_shared, touched, cfg.I, cfg.a8w8, mx=cfg.mx)
    # E4M3 and MX (kind::mxf8f6f4, FP8 rate also with E2M1 weights): twice the bf16 tensor rate
    tf_peak = pk["bf16_tflops_sustained"] * (2.0 if (cfg.a8w8 or cfg.mx) else 1.0)
    t_roof = max(fl / (tf_peak * 1e12), by / (pk["hbm_gbs"] * 1e9)) * 1e3
    rep = {"workload": workload_name(cfg, dtype_name), "tokens_per_s": cfg.T / (step_ms * 1e-3),
           "ms_per_step": step_ms, "tflops": fl / (step_ms * 1e-3) / 1e12, "touched_experts": touched,
           "layer_roofline_ms": t_roof, "layer_roofline_frac": t_roof / step_ms,
           "layer_bound": "tensor" if fl / (tf_peak * 1e12) > by / (pk["hbm_gbs"] * 1e9) else "hbm",
           "max_tokens_per_expert": int(load.max().item()),
           "stages_ms": st, "launch": "cuda_graph" if ms_graph is not None else "eager",
           "eager_ms_per_step": ms_eager / steps}
    # dominant kernel
    dom = max(st, key=st.get)
    kb = {"gateup": gateup_bytes(cfg, touched), "down": down_bytes(cfg, touched)}
    kfl = {"gateup": 4.0 * pairs * cfg.H * cfg.I, "down": 2.0 * pairs * cfg.H * cfg.I}
    roof = None
    if dom in kb:
        t = st[dom] * 1e-3
        hbm_t = kb[dom] / (pk["hbm_gbs"] * 1e9)
        ten_t = kfl[dom] / (tf_peak * 1e12)
        if ten_t > hbm_t:
            roof = {"kernel": f"grouped_gemm_kernel ({dom})", "bound": "tensor", "achieved": kfl[dom] / t / 1e12,
                    "peak": tf_peak, "unit": "TFLOP/s"}
        else:
            roof = {"kernel": f"grouped_gemm_kernel ({dom})", "bound": "hbm", "achieved": kb[dom] / t / 1e9,
                    "peak": pk["hbm_gbs"], "unit": "GB/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = traffic_for(f"grouped_gemm_{dom}", rep["workload"])
        roof["algorithmic_bytes"] = kb[dom]
        roof["launch_ms"] = st[dom]
    rep["dominant"] = roof
    e2e = None
    if primary:
        ems, h2d, d2h = time_e2e(cfg, layer, d, max(10, steps // 2), 3)
        e2e = {"value": cfg.T * max(10, steps // 2) / (ems * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del layer
    if data is None:
        del d
    torch.cuda.empty_cache()
    return rep, e2e, ms


def backward_report(m, cfg, steps, warmup, dev, pk):
    """One moe_backward (gradients of x, the router logits and both weight
    tensors; bf16 weights) on the layer, timed with CUDA events."""
    from moe_inputs import normal
    d = make_layer(cfg, device=dev)
    dout = normal((cfg.T, cfg.H), 1.0, cfg.seed * 16 + 9, dev, torch.bfloat16)
    outs = (torch.empty(cfg.T, cfg.H, dtype=torch.float32, device=dev),
            torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev),
            torch.empty(d["w13"].shape, dtype=torch.float32, device=dev),
            torch.empty(d["w2"].shape, dtype=torch.float32, device=dev))
    ws = None

    def call():
        m.backward(d["x"], d["logits"], d["w13"], d["w2"], dout, cfg.k, cfg.bm, bias=d["bias"],
                   bias_mode=cfg.bias_mode, n_shared=cfg.n_shared, outs=outs, ws=ws)

    call()
    torch.cuda.synchronize()
    ids = torch.topk(d["logits"], cfg.k, dim=1).indices
    touched = int(torch.unique(ids).numel()) + cfg.n_shared
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        call()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    pairs = slot_pairs(cfg)
    fl = backward_flops(pairs, cfg.H, cfg.I)
    by = backward_bytes(cfg.T, cfg.H, cfg.I, cfg.E + cfg.n_shared, touched, cfg.E)
    t_roof = max(fl / (pk["bf16_tflops_sustained"] * 1e12), by / (pk["hbm_gbs"] * 1e9)) * 1e3
    del d, dout, outs
    torch.cuda.empty_cache()
    return {"workload": "backward " + workload_name(cfg, "bf16"), "ms_per_step": ms,
            "tokens_per_s": cfg.T / (ms * 1e-3), "tflops": fl / (ms * 1e-3) / 1e12, "touched_experts": touched,
            "roofline_ms": t_roof, "roofline_frac": t_roof / ms,
            "bound": "tensor" if fl / (pk["bf16_tflops_sustained"] * 1e12) > by / (pk["hbm_gbs"] * 1e9) else "hbm",
            "algorithmic_bytes": by, "flops": fl,
            "note": "dW13/dW2 in fp32 for all experts; gate/up recomputed; eager launches"}


def ep_report(m, cfg, steps, warmup, dev):
    """The expert-parallel layer (ep.py) over a one-rank NCCL group on this GPU:
    gating, routing to ranks, permute, the exchange (trivial with one rank),
    the grouped FFN over the received rows, the reverse exchange, un-permute
    and combine, next to moe_forward on the same inputs (eager launches both).
    With one rank the exchange moves nothing across GPUs: this measures the
    per-rank steps' overhead, not the cost of the all-to-alls."""
    import socket
    import torch.distributed as dist
    from mixture_experts_expert_moe_b200.ep import EPMoELayer
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1, device_id=dev)
    try:
        d, layer = build_layer(m, cfg, dev)
        ep = EPMoELayer(d["w13"], d["w2"], cfg.E, cfg.k, cfg.bm)

        def timed(fn):
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            for _ in range(steps):
                fn()
            t1.record()
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / steps

        ms_ep = timed(lambda: ep(d["x"], d["logits"]))
        ms_fw = timed(lambda: layer(d["x"], d["logits"]))
        del d, layer, ep
        torch.cuda.empty_cache()
        return {"workload": "expert-parallel layer, 1 rank: " + workload_name(cfg, "bf16"), "ms_per_step": ms_ep,
                "tokens_per_s": cfg.T / (ms_ep * 1e-3), "moe_forward_ms_per_step": ms_fw,
                "note": "one NCCL rank: the all-to-alls move nothing; eager launches; split sizes read on the host"}
    finally:
        dist.destroy_process_group()


def bm_sweep(m, cfg, steps, warmup, dev, pk, sizes=(32, 64, 128)):
    """The layer at several block sizes (routing and values unchanged; the
    padding and the GEMM token groups change), in bf16 and a8w8, each
    precision's weights drawn once."""
    out = []
    for a8 in (False, True):
        c = cfg.with_(a8w8=a8)
        data = make_layer(c, device=dev)
        for bm in sizes:
            r, _, _ = layer_report(m, c.with_(bm=bm), steps, warmup, dev, pk, "a8w8" if a8 else "bf16", data=data)
            out.append(r)
        del data
        torch.cuda.empty_cache()
    return out


def align_report(m, dev, pk, T, iters=100):
    E, k, bm = ALIGN_CONFIG["E"], ALIGN_CONFIG["k"], ALIGN_CONFIG["bm"]
    ids = torch.from_numpy(align_ids(T, E, k, seed=ALIGN_CONFIG["seed"], dist="zipf",
                                     zipf_s=ALIGN_CONFIG["zipf_s"])).to(dev)
    P, NB, wsb = m.align_sort_sizes(T, k, E, bm)
    out = (torch.empty(P, dtype=torch.int32, device=dev), torch.empty(NB, dtype=torch.int32, device=dev),
           torch.empty(1, dtype=torch.int32, device=dev))
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(5):
        m.align_sort(ids, E, bm, ws=ws, out=out)
    torch.cuda.synchronize()
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            m.align_sort(ids, E, bm, ws=ws, out=out)
    except Exception as exc:
        sys.stderr.write(f"align graph capture failed: {exc}\n")
        graph = None
    ts = []
    for it in range(iters + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        if graph is not None:
            graph.replay()
        else:
            m.align_sort(ids, E, bm, ws=ws, out=out)
        b.record()
        torch.cuda.synchronize()
        if it >= 3:
            ts.append(a.elapsed_time(b))
    us = float(np.median(ts)) * 1e3
    n = int(out[2].item())
    by = align_bytes(T * k, n, bm)
    gbs = by / (us * 1e-6) / 1e9
    return {"workload": f"align_sort: T={T} E={E} k={k} bm={bm} zipf s=1, L2 flushed",
            "launch": "cuda_graph" if graph is not None else "eager", "us": us,
            "gb_per_s": gbs, "frac_hbm": gbs / pk["hbm_gbs"], "algorithmic_bytes": by}


def run_ours(args):
    import mixture_experts_expert_moe_b200 as m
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    m.load_library()
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    pk, pk_src = peaks()
    cfg = PRIMARY
    d, layer = build_layer(m, cfg, dev)
    touched, _ = touched_experts(layer, d)
    ms_eager, stages = time_layer(m, cfg, layer, d, args.steps, args.warmup)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    graph = None
    try:
        graph, _ = m.capture_graph(layer, d["x"], d["logits"], d["bias"], out=out)
    except Exception as exc:
        sys.stderr.write(f"graph capture failed, timing eager launches: {exc}\n")

    def step():
        if graph is not None:
            graph.replay()
        else:
            layer(d["x"], d["logits"], d["bias"], out=out)

    for _ in range(args.warmup):
        step()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    used_graph = graph is not None
    del graph
    step_ms = ms / args.steps
    pairs = slot_pairs(cfg)
    fl = moe_flops(pairs, cfg.H, cfg.I)
    by = layer_bytes(cfg.T, cfg.H, cfg.E, cfg.k + cfg.n_shared, touched, cfg.I, False)
    t_roof = max(fl / (pk["bf16_tflops_sustained"] * 1e12), by / (pk["hbm_gbs"] * 1e9)) * 1e3
    dom = max(stages, key=stages.get)
    kbytes = {"gateup": gateup_bytes(cfg, touched), "down": down_bytes(cfg, touched)}.get(dom)
    roof = None
    if kbytes is not None:
        ach = kbytes / (stages[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"],
                "traffic": traffic_for(f"grouped_gemm_{dom}", workload_name(cfg, "bf16")),
                "kernel": f"grouped_gemm_kernel ({dom} projection)", "launch_ms": stages[dom],
                "algorithmic_bytes": kbytes, "peak_source": f"{pk_src} hbm_gbs (copy)"}
    e2e_steps = max(10, args.steps // 2)
    if world > 1:
        torch.distributed.barrier()
    ems, h2d, d2h = time_e2e(cfg, layer, d, e2e_steps, 3)
    ems = max_over_ranks(ems, dev)
    e2e = {"value": job_throughput(world, cfg.T, e2e_steps, ems), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del layer, d
    torch.cuda.empty_cache()

    extra = {}
    if world == 1 and not args.quick:   # single-GPU reports (other ranks would idle in a barrier)
        extra["deepseek_bm_sweep"] = bm_sweep(m, cfg, 30, 3, dev, pk)
        extra["a8w8"] = next(r for r in extra["deepseek_bm_sweep"] if r["workload"].startswith("deepseek_a8w8")
                             and r["workload"].endswith("bm=64"))
        extra["deepseek_bias_4b"] = [layer_report(m, cfg.with_(bias=True, a8w8=a8), 30, 3, dev, pk,
                                                  "a8w8" if a8 else "bf16")[0] for a8 in (False, True)]
        extra["mixtral"], _, _ = layer_report(m, CONFIGS["mixtral"], 20, 3, dev, pk, "bf16")
        extra["deepseek_shared"], _, _ = layer_report(m, CONFIGS["deepseek_shared"], 50, 5, dev, pk, "bf16")
        extra["decode_a8w8"] = []
        for T in (1, 16, 64, 256):
            r, _, _ = layer_report(m, CONFIGS["decode"].with_(T=T), 100, 5, dev, pk, "a8w8")
            extra["decode_a8w8"].append(r)
        extra["decode_mx"] = []
        for fmt in ("mxfp4", "mxfp8"):
            for T in (1, 16, 64, 256):
                c = CONFIGS["decode"].with_(T=T, a8w8=False, mx=fmt)
                extra["decode_mx"].append(layer_report(m, c, 100, 5, dev, pk, fmt)[0])
        extra["deepseek_mx"] = [layer_report(m, cfg.with_(mx=fmt), 30, 3, dev, pk, fmt)[0]
                                for fmt in ("mxfp4", "mxfp8")]
        extra["backward"] = backward_report(m, cfg, 10, 3, dev, pk)
        try:
            extra["expert_parallel"] = ep_report(m, cfg, 20, 3, dev)
        except Exception as exc:      # a process-group set-up problem must not cost the bench line
            extra["expert_parallel"] = {"error": str(exc)[:300]}
        extra["align_sort"] = align_report(m, dev, pk, ALIGN_CONFIG["T"])
        extra["align_sort_large"] = align_report(m, dev, pk, 1 << 22, iters=20)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cfg)
        if not args.quick:
            extra["oracle_ops"] = oracle_op_times()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": job_throughput(world, cfg.T, args.steps, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations and logits, N(0,0.02) random-init expert weights)",
        "config": {"workload": workload_name(cfg, "bf16"), "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (22.5 GB of expert weights streamed per step)",
                   "touched_experts": touched,
                   "launch": "cuda_graph replay of one moe_forward" if used_graph else "eager moe_forward"},
        "eager_ms_per_step": ms_eager / args.steps,
        "tflops": fl / (step_ms * 1e-3) / 1e12,
        "layer_roofline": {"ms": t_roof, "frac": t_roof / step_ms, "bound": "hbm",
                           "bytes": by, "flops": fl, "peak_source": pk_src},
        "stages_ms": stages,
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": kernels_per_step(cfg, torch.bfloat16) * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    line.update(extra)
    emit(line)


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
class _HostExperts:
    """Expert weights of the experts a sample touches, copied to the host once
    (float32, or bf16 converted on access); the oracle converts each expert it
    uses to float64 itself."""

    def __init__(self, t, needed, as_f32):
        self.shape = tuple(t.shape)
        self.as_f32 = as_f32
        self.host = {int(e): (t[int(e)].float().cpu().numpy() if as_f32 else t[int(e)].cpu()) for e in needed}

    def __getitem__(self, e):
        w = self.host[int(e)]
        return w if self.as_f32 else w.float().numpy()


def _oracle_inputs(cfg, n_tokens, as_f32, seed=0):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))) if torch.cuda.is_available() else "cpu"
    d = make_layer(cfg, device=dev)
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(cfg.T, size=n_tokens, replace=False))
    x = d["x"][torch.from_numpy(toks).to(d["x"].device)].float().cpu().numpy()
    logits = d["logits"][torch.from_numpy(toks).to(d["x"].device)].cpu().numpy()
    # experts the sampled tokens route to (for the host copy only; the oracle routes itself)
    need = torch.topk(d["logits"][torch.from_numpy(toks).to(d["x"].device)], cfg.k, dim=1).indices.unique().cpu()
    w13 = _HostExperts(d["w13"], need, as_f32)
    w2 = _HostExperts(d["w2"], need, as_f32)
    del d
    if torch.cuda.is_available():
        torch.cuda.empty_cache()
    return x, logits, w13, w2


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name (lscpu, else /proc/cpuinfo)."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name:"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def _timed(fn, min_s=0.5):
    """Mean seconds per call of fn over enough calls to last min_s."""
    fn()
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            return dt / n


def oracle_op_times(n_ffn_tokens=2):
    """The oracle per step of the path, on the host cores, at one thread and at
    every thread BLAS offers: gating of the DeepSeek-V3-shaped layer's 2048
    tokens (top-8 of 256 logits), align & sort of the 16384-token Zipf
    workload (top-8 of 256, block 64), both in full, and the expert FFN +
    combine of a sample of that layer's tokens (bf16 weights)."""
    import oracle
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        threadpool_limits = None
    cfg = PRIMARY
    logits = make_layer(cfg, device="cpu", weights=False)["logits"].numpy()
    ids = align_ids(ALIGN_CONFIG["T"], ALIGN_CONFIG["E"], ALIGN_CONFIG["k"], seed=ALIGN_CONFIG["seed"],
                    dist="zipf", zipf_s=ALIGN_CONFIG["zipf_s"])
    x, lg, w13, w2 = _oracle_inputs(cfg, n_ffn_tokens, as_f32=False)
    all_threads = _threads()
    res = {"cpu_model": cpu_model(), "host_cpus": os.cpu_count(), "kind": "oracle", "levels": []}
    for threads in sorted({1, all_threads}):
        ctx = threadpool_limits(threads) if threadpool_limits else None
        if ctx is not None:
            ctx.__enter__()
        try:
            t_gate = _timed(lambda: oracle.topk_gate(logits, cfg.k))
            t_align = _timed(lambda: oracle.align_sort(ids, ALIGN_CONFIG["E"], ALIGN_CONFIG["bm"]))
            t0 = time.perf_counter()
            oracle.moe_forward(x, lg, cfg.k, w13, w2)
            t_ffn = time.perf_counter() - t0
        finally:
            if ctx is not None:
                ctx.__exit__(None, None, None)
        res["levels"].append({
            "threads": threads,
            "gate_ms": t_gate * 1e3, "gate_tokens_per_s": cfg.T / t_gate,
            "align_sort_ms": t_align * 1e3,
            "align_sort_slots_per_s": ALIGN_CONFIG["T"] * ALIGN_CONFIG["k"] / t_align,
            "ffn_combine_s": t_ffn, "ffn_tokens_per_s": n_ffn_tokens / t_ffn})
    res["sample"] = (f"gate: {cfg.T} x {cfg.E} logits, top-{cfg.k}; align & sort: {ALIGN_CONFIG['T']} tokens x "
                     f"top-{ALIGN_CONFIG['k']} of {ALIGN_CONFIG['E']}, block {ALIGN_CONFIG['bm']}, in full; "
                     f"FFN + combine: {n_ffn_tokens} seeded tokens of {workload_name(cfg, 'bf16')} "
                     "(float64 numpy, bf16 weights converted per expert)")
    return res


def cpu_baseline(cfg, n_tokens=6):
    import oracle
    x, logits, w13, w2 = _oracle_inputs(cfg, n_tokens, as_f32=False)
    t = time.perf_counter()
    oracle.moe_forward(x, logits, cfg.k, w13, w2)
    dt = time.perf_counter() - t
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "sample": f"a batch of {n_tokens} seeded tokens of {workload_name(cfg, 'bf16')} through the "
                      f"whole layer (float64 numpy; bf16 weights converted per expert), {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cfg = PRIMARY
    n_tokens = 1
    x, logits, w13, w2 = _oracle_inputs(cfg, n_tokens, as_f32=True)
    for _ in range(args.warmup):
        oracle.moe_forward(x, logits, cfg.k, w13, w2)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.moe_forward(x, logits, cfg.k, w13, w2)
    dt = time.perf_counter() - t
    v = n_tokens * args.steps / dt
    world = int(os.environ.get("WORLD_SIZE", "1"))
    sample = (f"a batch of {n_tokens} seeded token per step of {workload_name(cfg, 'bf16')} through the "
              f"whole layer (float64 numpy on the host; the token's experts' weights held as float32)")
    emit({
        "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(cfg, "bf16"), "parallelism": "host cores"},
        "impl": "reference",
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })


def run_only(args):
    import mixture_experts_expert_moe_b200 as m
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk, _ = peaks()
    steps = 20 if args.steps is None else args.steps
    warmup = 3 if args.warmup is None else max(3, args.warmup)
    parts = args.only.split("_")
    if parts[0] == "backward":      # backward_<config>[_T<N>][_E<N>]
        cfg = CONFIGS[parts[1]]
        for q in parts[2:]:
            if q.startswith("T"):
                cfg = cfg.with_(T=int(q[1:]))
            elif q.startswith("E"):
                cfg = cfg.with_(E=int(q[1:]))
        emit(backward_report(m, cfg, steps, warmup, dev, pk))
        return
    if parts[0] == "ep":          # ep_<config>: the expert-parallel layer over one rank
        emit(ep_report(m, CONFIGS[parts[1]], steps, warmup, dev))
        return
    if parts[0] == "align":
        emit(align_report(m, dev, pk, int(parts[1]), iters=steps))
        return
    if len(parts) > 2 and f"{parts[0]}_{parts[1]}" in CONFIGS:     # e.g. deepseek_shared
        parts = [f"{parts[0]}_{parts[1]}"] + parts[2:]
    cfg = CONFIGS[parts[0]].with_(a8w8=parts[1] == "a8w8", mx=parts[1] if parts[1].startswith("mx") else "")
    tile = 0
    for p in parts[2:]:
        if p.startswith("bm"):
            cfg = cfg.with_(bm=int(p[2:]))
        elif p.startswith("T"):
            cfg = cfg.with_(T=int(p[1:]))
        elif p.startswith("E"):
            cfg = cfg.with_(E=int(p[1:]))
        elif p.startswith("tn"):
            tile = int(p[2:])
        elif p.startswith("H"):
            cfg = cfg.with_(H=int(p[1:]))
        elif p.startswith("I"):
            cfg = cfg.with_(I=int(p[1:]))
        elif p == "bias":
            cfg = cfg.with_(bias=True)
    rep, _, _ = layer_report(m, cfg, steps, warmup, dev, pk, parts[1], tile_tokens=tile)
    emit(rep)


_OUT = sys.stdout


def emit(obj):
    """The run's one JSON line, on the process's original stdout."""
    _OUT.write(json.dumps(obj) + "\n")
    _OUT.flush()


def _reserve_stdout():
    """Send file descriptor 1 to stderr for the rest of the run, so that a
    library writing to stdout (NCCL's version banner, for one) cannot put a
    line next to the JSON line; returns a stream on the original stdout."""
    sys.stdout.flush()
    out = os.fdopen(os.dup(1), "w")
    os.dup2(2, 1)
    return out


def main():
    global _OUT
    _OUT = _reserve_stdout()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="headline workload only")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--only", default=None,
                    help="time one workload and print its report: <config>_<bf16|a8w8|mxfp8|mxfp4>"
                         "[_bm<N>][_T<N>][_E<N>][_H<N>][_I<N>][_tn<N>] "
                         "(configs: tiny, p5, deepseek, deepseek_shared, mixtral, decode) or align_<T>")
    args = ap.parse_args()
    if args.only:
        run_only(args)
        return
    if args.impl == "reference":
        args.steps = 3 if args.steps is None else args.steps
        args.warmup = 1 if args.warmup is None else args.warmup
        run_reference(args)
    else:
        args.steps = 100 if args.steps is None else args.steps
        args.warmup = 5 if args.warmup is None else max(3, args.warmup)
        run_ours(args)


if __name__ == "__main__":
    main()
