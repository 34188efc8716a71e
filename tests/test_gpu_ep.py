"""GPU tests of the expert-parallel steps on the library's kernels:

* moe_ep_route: order, per-rank counts and local expert ids bit-exact
  against the definition (stable grouping of the slots by rank);
* moe_permute_rows / moe_scatter_rows: bit-exact row moves;
* the EP forward of 4 ranks emulated on one GPU: each rank's steps on the
  library's kernels, the all-to-alls done by slicing the ranks' buffers in
  the order all_to_all_single uses (no rank waits on another), against the
  oracle layer;
* EPMoELayer over a one-rank NCCL process group against the oracle layer,
  with one exchange and with the pipelined exchange of 3 chunks.
The exchange logic of ep_forward across several processes is covered on CPU
with gloo ranks (tests/test_ep.py).
"""
import socket

import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
from mixture_experts_expert_moe_b200.ep import LibraryOps
from moe_inputs import CONFIGS, align_ids, make_layer, to_numpy
from parity_util import TOL_BF16, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_ep_route_bit_exact(cuda_device, R):
    ids = align_ids(2048, 256, 8, seed=7, dist="zipf")
    order, counts, local = m.ep_route(torch.from_numpy(ids).to(cuda_device), 256, R)
    torch.cuda.synchronize()
    flat = ids.reshape(-1)
    dest = flat // (256 // R)
    ref_order = np.argsort(dest, kind="stable")
    np.testing.assert_array_equal(order.cpu().numpy(), ref_order)
    np.testing.assert_array_equal(counts.cpu().numpy(), np.bincount(dest, minlength=R))
    np.testing.assert_array_equal(local.cpu().numpy(), flat[ref_order] % (256 // R))


def test_permute_and_scatter_rows(cuda_device):
    g = torch.Generator(device=cuda_device).manual_seed(3)
    x = torch.randn(300, 72, device=cuda_device, generator=g).to(torch.bfloat16)
    idx = torch.randperm(900, device=cuda_device, generator=g).to(torch.int32)
    got = m.permute_rows(x, idx, div=3)
    assert torch.equal(got, x[(idx // 3).long()])
    y = torch.randn(900, 20, device=cuda_device, generator=g)
    back = m.scatter_rows(y, idx, 900)
    ref = torch.empty_like(y)
    ref[idx.long()] = y
    assert torch.equal(back, ref)


def _split(t, counts):
    offs = np.concatenate([[0], np.cumsum(counts)])
    return [t[offs[i]:offs[i + 1]] for i in range(len(counts))]


def test_ep_forward_four_ranks_emulated(cuda_device):
    cfg = CONFIGS["tiny"]
    R, El = 4, CONFIGS["tiny"].E // 4
    d = make_layer(cfg, device=cuda_device)
    Tr = cfg.T // R
    ops = [LibraryOps(m, d["w13"][r * El:(r + 1) * El].contiguous(), d["w2"][r * El:(r + 1) * El].contiguous(),
                      cfg.k, cfg.bm, out_dtype=torch.float32) for r in range(R)]
    st = []
    for r in range(R):
        x_r, l_r = d["x"][r * Tr:(r + 1) * Tr].contiguous(), d["logits"][r * Tr:(r + 1) * Tr].contiguous()
        ids, w = ops[r].gate(l_r)
        order, counts, local = ops[r].route(ids, cfg.E, R)
        c = counts.cpu().numpy()
        st.append(dict(w=w, order=order, counts=c, rows=_split(ops[r].permute(x_r, order, cfg.k), c),
                       lids=_split(local, c)))
    # all-to-all: destination d receives the sources' segments in rank order
    y = []
    for dst in range(R):
        rows = torch.cat([st[src]["rows"][dst] for src in range(R)]).contiguous()
        lids = torch.cat([st[src]["lids"][dst] for src in range(R)]).contiguous()
        y.append((ops[dst].expert_ffn(rows, lids), [int(st[src]["counts"][dst]) for src in range(R)]))
    outs = []
    for r in range(R):
        back = torch.cat([_split(y[dst][0], y[dst][1])[r] for dst in range(R)]).contiguous()
        y_slots = ops[r].scatter(back, st[r]["order"], Tr * cfg.k)
        outs.append(ops[r].combine(y_slots, st[r]["w"]))
    torch.cuda.synchronize()
    ref, _, _ = oracle.moe_forward(to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k, to_numpy(d["w13"]),
                                   to_numpy(d["w2"]))
    assert_close(torch.cat(outs).cpu().numpy(), ref, TOL_BF16, "4-rank EP forward (emulated)")


def test_ep_layer_one_rank_nccl(cuda_device):
    import torch.distributed as dist
    from mixture_experts_expert_moe_b200.ep import EPMoELayer
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=cuda_device)
    try:
        cfg = CONFIGS["tiny"]
        d = make_layer(cfg, device=cuda_device)
        ref, _, _ = oracle.moe_forward(to_numpy(d["x"]), to_numpy(d["logits"]), cfg.k, to_numpy(d["w13"]),
                                       to_numpy(d["w2"]))
        # one exchange, and the pipelined exchange of 3 chunks (asynchronous all-to-alls)
        for chunks in (1, 3):
            layer = EPMoELayer(d["w13"], d["w2"], cfg.E, cfg.k, cfg.bm, out_dtype=torch.float32, chunks=chunks)
            out = layer(d["x"], d["logits"])
            torch.cuda.synchronize()
            assert_close(out.cpu().numpy(), ref, TOL_BF16, f"EP layer, one NCCL rank, {chunks} chunk(s)")
    finally:
        dist.destroy_process_group()
