"""The FLOP / I/O accounting used by bench.py, pinned to the figures printed
in the aiter a8w8 issue ("[Feature]: Add more configuration options for MoE
assembly kernels", "Estimated Performance Scaling" table; fixture
tests/golden/p5_a8w8_table.json)."""
import json
import os

import pytest

from mixture_experts_expert_moe_b200.roofline import moe_flops, tile_io_bytes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p5_a8w8_table.json")


@pytest.fixture(scope="module")
def table():
    with open(GOLDEN) as f:
        return json.load(f)


def test_flops_reproduce_measured_tflops(table):
    r = table["rows"][0]
    pairs = r["experts"] * r["tokens_per_expert"]
    f = moe_flops(pairs, table["hidden_dim"], table["inter_dim"])
    assert abs(f / (r["time_us"] * 1e-6) / 1e12 - r["tflops"]) < 0.01


def test_io_row1_is_weights_streamed_once_per_m_tile(table):
    r = table["rows"][0]
    m_tiles = r["tokens_per_expert"] // r["block_m"]
    io = tile_io_bytes(r["experts"], m_tiles, table["hidden_dim"], table["inter_dim"])
    assert abs(io / 1e9 - r["io_gb"]) < 0.01


def test_estimated_rows_scale_time_by_io(table):
    r0 = table["rows"][0]
    for r in table["rows"][1:]:
        t = r0["time_us"] * r["io_gb"] / r0["io_gb"]
        assert abs(t - r["time_us"]) / r["time_us"] < 0.005
        pairs = r["experts"] * r["tokens_per_expert"]
        tf = moe_flops(pairs, table["hidden_dim"], table["inter_dim"]) / (r["time_us"] * 1e-6) / 1e12
        assert abs(tf - r["tflops"]) / r["tflops"] < 0.005
