"""bench.py's accounting, checked by hand on small numbers (CPU).

The roofline objects divide these byte and FLOP counts by measured times, so
a wrong count would silently scale every reported fraction.
"""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from moe_inputs import CONFIGS, MoEConfig  # noqa: E402


def test_slot_pairs_count_shared_experts():
    assert bench.slot_pairs(MoEConfig("t", T=10, H=128, I=128, E=8, k=2, bm=16)) == 20
    assert bench.slot_pairs(MoEConfig("t", T=10, H=128, I=128, E=8, k=2, bm=16, n_shared=1)) == 30


def test_kernels_per_step():
    bf16 = MoEConfig("t", T=2048, H=128, I=128, E=256, k=8, bm=64)
    assert bench.kernels_per_step(bf16, None) == 5            # route, gather, gate/up, down, combine/round
    assert bench.kernels_per_step(bf16.with_(a8w8=True), None) == 7   # + quant (16384 slots > 4096) + requant
    assert bench.kernels_per_step(bf16.with_(T=16, a8w8=True), None) == 6   # fused quant + gather


def test_gateup_and_down_bytes_by_hand():
    cfg = MoEConfig("t", T=4, H=256, I=128, E=8, k=2, bm=16)
    touched = 3
    # bf16: 3 experts x (2*128*256 weights x 2 B) + x once (4 x 256 x 2 B) + 8 pairs x 4 B of slot ids
    assert bench.gateup_bytes(cfg, touched) == 3 * 2 * 128 * 256 * 2 + 4 * 256 * 2 + 8 * 4
    # down: 3 x 256*128 x 2 + fp32 token rows once (4 x 256 x 4) + 8 pairs x (slot id + weight)
    assert bench.down_bytes(cfg, touched) == 3 * 256 * 128 * 2 + 4 * 256 * 4 + 8 * 8
    a8 = cfg.with_(a8w8=True)
    # E4M3 weights + fp32 per-channel scales; x at one byte per element
    assert bench.gateup_bytes(a8, touched) == 3 * (2 * 128 * 256 + 2 * 128 * 4) + 4 * 256 + 8 * 4
    assert bench.down_bytes(a8, touched) == 3 * (256 * 128 + 256 * 4) + 4 * 256 * 4 + 8 * 8


def test_headline_kernel_bytes_are_the_weight_stream():
    # DeepSeek-V3 gate/up: all 256 experts' gate+up weights dominate (15.03 GB of 15.06 GB)
    cfg = CONFIGS["deepseek"]
    b = bench.gateup_bytes(cfg, 256)
    assert b == 256 * 2 * 2048 * 7168 * 2 + 2048 * 7168 * 2 + 2048 * 8 * 4


def test_headline_workload_name():
    name = bench.workload_name(CONFIGS["deepseek"], "bf16")
    assert name == "deepseek_bf16: T=2048 H=7168 I=2048 E=256 k=8 bm=64"
    assert bench.workload_name(CONFIGS["deepseek_shared"], "bf16").endswith("+bias(selection only) +1 shared")


def test_traffic_lookup_needs_matching_source(tmp_path):
    # the committed table is keyed by the kernel source hash: a made-up workload has no entry
    assert bench.traffic_for("grouped_gemm_gateup", "no such workload") is None
    import hashlib
    import json
    src = "mixture_experts_expert_moe_b200/roofline.py"
    h = hashlib.sha256(open(os.path.join(bench.ROOT, src), "rb").read()).hexdigest()[:16]
    t = tmp_path / "t.json"
    ent = {"kernel": "k", "workload": "w", "bytes_per_launch": 123, "source": src, "sha256_16": h}
    t.write_text(json.dumps({"entries": [ent]}))
    assert bench.traffic_for("k", "w", table=str(t)) == 123
    ent["sha256_16"] = "0" * 16          # the source changed since the capture
    t.write_text(json.dumps({"entries": [ent]}))
    assert bench.traffic_for("k", "w", table=str(t)) is None


@pytest.mark.parametrize("world,units,steps,ms", [(1, 2048, 100, 400.0), (8, 2048, 50, 210.0)])
def test_job_throughput(world, units, steps, ms):
    assert bench.job_throughput(world, units, steps, ms) == pytest.approx(world * units * steps / (ms / 1000))


def test_mx_weight_bytes_by_hand():
    from mixture_experts_expert_moe_b200.roofline import expert_weight_bytes
    H, I = 256, 128
    # E2M1 codes at half a byte, E4M3 at one, plus one E8M0 byte per 32 elements
    assert expert_weight_bytes(H, I, False, "mxfp4") == 3 * H * I // 2 + 3 * H * I // 32
    assert expert_weight_bytes(H, I, False, "mxfp8") == 3 * H * I + 3 * H * I // 32
    cfg = MoEConfig("t", T=4, H=H, I=I, E=8, k=2, bm=16, mx="mxfp4")
    assert bench.gateup_bytes(cfg, 3) == 3 * (2 * I * H // 2 + 2 * I * H // 32) + 4 * H + 8 * 4
    assert bench.down_bytes(cfg, 3) == 3 * (H * I // 2 + H * I // 32) + 4 * H * 4 + 8 * 8


def test_backward_accounting_by_hand():
    from mixture_experts_expert_moe_b200.roofline import backward_bytes, backward_flops
    # z (2) + gate/up again (4) + dx (4) + dW2 (2) + dW13 (4) multiply-add FLOPs per pair, H, I
    assert backward_flops(10, 256, 128) == 16 * 10 * 256 * 128
    T, H, I, E, touched, EL = 4, 256, 128, 8, 3, 8
    w_read = touched * (2 * 2 * I * H * 2 + H * I * 2)       # W13 twice, Wd once (bf16)
    dw = E * 3 * H * I * 4                                     # fp32 gradients of every expert
    act = 2 * T * H * 2 + T * H * 4 + 2 * T * EL * 4           # x, dout in; dx out; logits in, dlogits out
    assert backward_bytes(T, H, I, E, touched, EL) == w_read + dw + act


def test_bench_stdout_carries_only_the_json_line():
    """Writes to file descriptor 1 by libraries (NCCL's version banner) and
    stray prints go to stderr once bench.py has reserved stdout; the JSON
    line alone reaches the original stdout."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import os, bench; bench._OUT = bench._reserve_stdout(); os.write(1, b'NCCL version x\\n'); "
            "print('stray'); bench.emit({'metric': 'm', 'value': 1.0})")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout == '{"metric": "m", "value": 1.0}\n'
    assert "NCCL version x" in r.stderr and "stray" in r.stderr
