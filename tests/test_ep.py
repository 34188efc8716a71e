"""Expert-parallel forward (mixture_experts_expert_moe_b200/ep.py): the
exchange logic of ep_forward across 2 and 4 gloo ranks on CPU.

The per-rank steps are executed by the oracle (test infrastructure: gating,
grouping by destination rank, the local experts' FFN, combine), so what is
checked here is the exchange itself: slot counts, split sizes, the order of
the rows sent and received, the reverse exchange and the un-permute.  The
ranks' outputs must equal the single-process oracle layer on the same tokens
(float64 throughout).  The same orchestration on the library's kernels runs
on the GPU in tests/test_gpu_ep.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

T_PER_RANK, H, I, E, K = 12, 64, 32, 8, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(R):
    rng = np.random.default_rng(1234)
    T = T_PER_RANK * R
    x = rng.standard_normal((T, H))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = rng.standard_normal((E, 2 * I, H)) * 0.1
    w2 = rng.standard_normal((E, H, I)) * 0.1
    return x, logits, w13, w2


class OracleOps:
    def __init__(self, w13_local, w2_local, k):
        self.w13, self.w2, self.k = w13_local, w2_local, k

    def gate(self, logits, bias=None, bias_mode="logits"):
        import oracle
        ids, w = oracle.topk_gate(logits.numpy(), self.k)
        return torch.from_numpy(ids), torch.from_numpy(w)

    def route(self, ids, E_, R):
        flat = ids.numpy().reshape(-1)
        dest = flat // (E_ // R)
        order = np.argsort(dest, kind="stable").astype(np.int32)
        counts = np.bincount(dest, minlength=R).astype(np.int32)
        local = (flat[order] % (E_ // R)).astype(np.int32)
        return torch.from_numpy(order), torch.from_numpy(counts), torch.from_numpy(local)

    def permute(self, x, order, k):
        return x[order.long() // k].contiguous()

    def expert_ffn(self, rows, local_ids):
        import oracle
        if rows.shape[0] == 0:
            return torch.zeros(0, rows.shape[1], dtype=torch.float64)
        y = oracle.ffn_bf16(rows.numpy(), local_ids.numpy().reshape(-1, 1), self.w13, self.w2)
        return torch.from_numpy(y)

    def scatter(self, y, order, rows):
        out = torch.zeros(rows, y.shape[1], dtype=y.dtype)
        out[order.long()] = y
        return out

    def combine(self, y_slots, w):
        import oracle
        return torch.from_numpy(oracle.combine(y_slots.numpy(), w.numpy()))


def _rank(rank, R, port, q, chunks=1, sizes=None):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        from mixture_experts_expert_moe_b200.ep import ep_forward
        x, logits, w13, w2 = _layer(R)
        El = E // R
        ops = OracleOps(w13[rank * El:(rank + 1) * El], w2[rank * El:(rank + 1) * El], K)
        sizes = sizes or [T_PER_RANK] * R      # tokens of each rank (a prefix of the layer's batch)
        start = sum(sizes[:rank])
        sl = slice(start, start + sizes[rank])
        out = ep_forward(ops, torch.from_numpy(x[sl].copy()), torch.from_numpy(logits[sl].copy()), E,
                         chunks=chunks)
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


# chunks: 1 (one exchange), 3 (the pipelined exchange of 4-token chunks) and
# 16 (more chunks than the rank's 12 tokens: empty chunks on every rank)
@pytest.mark.parametrize("chunks", [1, 3, 16])
@pytest.mark.parametrize("R", [2, 4])
def test_ep_exchange_matches_single_process_layer(R, chunks):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, R, port, q, chunks)) for r in range(R)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(R))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, logits, w13, w2 = _layer(R)
    ref, _, _ = oracle.moe_forward(x, logits, K, w13, w2)
    out = np.concatenate([got[r] for r in range(R)])
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("chunks", [1, 3])
def test_ep_exchange_uneven_ranks(chunks):
    """Ranks with different token counts, one of them with none."""
    import oracle
    R, sizes = 4, [12, 7, 0, 5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, R, port, q, chunks, sizes)) for r in range(R)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(R))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, logits, w13, w2 = _layer(R)
    n = sum(sizes)
    ref, _, _ = oracle.moe_forward(x[:n], logits[:n], K, w13, w2)
    assert [got[r].shape[0] for r in range(R)] == sizes
    out = np.concatenate([got[r] for r in range(R)])
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
