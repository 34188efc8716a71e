"""Expert-parallel (EP) MoE layer forward over a torch.distributed group.

The layer's E experts are sharded over the R ranks of the group: rank r
holds experts [r*E/R, (r+1)*E/R) (``w13_local [E/R, 2I, H]``,
``w2_local [E/R, H, I]``); every rank gates its own tokens.  Sources: the
X-MoE and GC-MoE abstracts (expert-parallel dispatch and combine across
GPUs); the steps on each rank are the single-GPU layer's (MoE Align & Sort
article: gating, permute, group GEMM, unpermute).

One forward on a rank:

    ids, w          = top-k gating of the rank's tokens           (moe_topk_gate)
    order, counts   = the slots grouped by destination rank       (moe_ep_route)
    recv counts     = all-to-all of the per-rank slot counts
    send rows       = x[order // k]                               (moe_permute_rows)
    recv rows, ids  = all-to-all of the rows and their local expert ids
    y               = the local experts' FFN on the received rows (moe_align_sort +
                      moe_grouped_ffn with one slot per row)
    back            = all-to-all of y in the reverse direction
    y_slots         = back scattered to slot order                (moe_scatter_rows)
    out             = sum_j w[t, j] y_slots[t*k + j]              (moe_combine)

Every compute step runs in the library's kernels; torch.distributed (NCCL on
GPUs) carries the exchange.  The split sizes of the variable all-to-alls are
read on the host (one device-to-host copy of R counts per forward).  The
per-rank steps are gathered in ``LibraryOps`` so that the exchange logic
above is one function (``ep_forward``) whatever executes the steps.

With ``chunks`` > 1 the rank's tokens are split into that many contiguous
chunks that flow through the steps as a pipeline: the all-to-alls are
issued asynchronously, so that the exchange of chunk c + 1 (and the return
of chunk c - 1) proceed while the local experts compute chunk c (on GPUs:
NCCL's stream next to the compute stream).  The split sizes of every chunk
travel in one all-to-all up front.  Every rank must use the same number of
chunks; a chunk may be empty on some rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The per-rank steps of ``ep_forward`` on this library's kernels."""

    def __init__(self, m, w13_local, w2_local, k, block_size, out_dtype=torch.bfloat16):
        self.m, self.w13, self.w2, self.k, self.bm = m, w13_local, w2_local, k, block_size
        self.out_dtype = out_dtype

    def gate(self, logits, bias=None, bias_mode="logits"):
        return self.m.topk_gate(logits, self.k, bias=bias, bias_mode=bias_mode)

    def route(self, ids, E, R):
        return self.m.ep_route(ids, E, R)

    def permute(self, x, order, k):
        return self.m.permute_rows(x, order, div=k)

    def expert_ffn(self, rows, local_ids):
        """y [M, H] fp32 of the local experts on the received rows (one slot
        per row)."""
        M = rows.shape[0]
        if M == 0:
            return torch.empty(0, rows.shape[1], dtype=torch.float32, device=rows.device)
        ids = local_ids.view(M, 1).contiguous()
        s, b, n = self.m.align_sort(ids, self.w13.shape[0], self.bm)
        return self.m.grouped_ffn(rows, self.w13, self.w2, s, b, n, 1, self.bm)

    def scatter(self, y, order, rows):
        return self.m.scatter_rows(y, order, rows)

    def combine(self, y_slots, w):
        return self.m.combine(y_slots, w, out_dtype=self.out_dtype)


def _all_to_all(send, send_counts, recv_counts, group):
    """Variable all-to-all of the rows of ``send`` (row counts per rank)."""
    recv = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(recv, send, recv_counts, send_counts, group=group)
    return recv


def ep_forward(ops, x, logits, E, group=None, bias=None, bias_mode="logits", chunks=1):
    """One expert-parallel layer forward of this rank's tokens (module
    docstring).  Every rank of ``group`` must call it, in the same order and
    with the same ``chunks``."""
    if chunks > 1:
        return _ep_forward_pipelined(ops, x, logits, E, group, bias, bias_mode, chunks)
    R = dist.get_world_size(group)
    T, H = x.shape
    ids, w = ops.gate(logits, bias, bias_mode)
    k = ids.shape[1]
    order, counts, local_ids = ops.route(ids, E, R)
    # split sizes: this rank's slots per destination, and what every rank sends here
    send_counts = torch.as_tensor(counts, dtype=torch.int64).reshape(R)
    recv_counts_t = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts_t, send_counts.to(recv_counts_t.device), group=group)
    send_c = send_counts.cpu().tolist()
    recv_c = recv_counts_t.cpu().tolist()
    rows = _all_to_all(ops.permute(x, order, k), send_c, recv_c, group)
    rids = _all_to_all(local_ids.reshape(-1, 1), send_c, recv_c, group).reshape(-1)
    y = ops.expert_ffn(rows, rids)
    back = _all_to_all(y, recv_c, send_c, group)
    y_slots = ops.scatter(back, order, T * k)
    return ops.combine(y_slots, w)


def _ep_forward_pipelined(ops, x, logits, E, group, bias, bias_mode, chunks):
    """ep_forward over ``chunks`` contiguous token chunks, the exchanges of
    neighbouring chunks overlapping the local experts' compute."""
    R = dist.get_world_size(group)
    T, H = x.shape
    ids, w = ops.gate(logits, bias, bias_mode)
    k = ids.shape[1]
    bounds = [T * c // chunks for c in range(chunks + 1)]
    routes = [ops.route(ids[bounds[c]:bounds[c + 1]], E, R) for c in range(chunks)]
    # split sizes of every chunk in one exchange: send[r, c] slots of chunk c go to rank r
    send_dev = torch.stack([torch.as_tensor(rt[1]).to(device=x.device, dtype=torch.int64).reshape(R)
                            for rt in routes], dim=1).contiguous()
    recv_dev = torch.empty_like(send_dev)
    dist.all_to_all_single(recv_dev, send_dev, group=group)
    send_c, recv_c = send_dev.cpu().tolist(), recv_dev.cpu().tolist()

    def dispatch(c):
        order, _, local = routes[c]
        sc = [send_c[r][c] for r in range(R)]
        rc = [recv_c[r][c] for r in range(R)]
        rows_send = ops.permute(x[bounds[c]:bounds[c + 1]], order, k)
        ids_send = local.reshape(-1, 1).contiguous()
        rows = torch.empty((sum(rc), H), dtype=rows_send.dtype, device=x.device)
        rids = torch.empty((sum(rc), 1), dtype=ids_send.dtype, device=x.device)
        works = [dist.all_to_all_single(rows, rows_send, rc, sc, group=group, async_op=True),
                 dist.all_to_all_single(rids, ids_send, rc, sc, group=group, async_op=True)]
        return rows, rids, sc, rc, works, (rows_send, ids_send)

    def compute(d):
        rows, rids, sc, rc, works, _ = d
        for wk in works:
            wk.wait()
        y = ops.expert_ffn(rows, rids.reshape(-1))
        back = torch.empty((sum(sc), H), dtype=y.dtype, device=y.device)
        return back, dist.all_to_all_single(back, y.contiguous(), sc, rc, group=group, async_op=True), y

    def finish(c, b):
        back, work, _ = b
        work.wait()
        tc = bounds[c + 1] - bounds[c]
        if tc == 0:
            return None
        y_slots = ops.scatter(back, routes[c][0], tc * k)
        return ops.combine(y_slots, w[bounds[c]:bounds[c + 1]])

    sent = [None] * chunks
    back = [None] * chunks
    outs = []
    sent[0] = dispatch(0)
    if chunks > 1:
        sent[1] = dispatch(1)
    for c in range(chunks):
        back[c] = compute(sent[c])
        sent[c] = None
        if c + 2 < chunks:
            sent[c + 2] = dispatch(c + 2)
        if c >= 1:
            outs.append(finish(c - 1, back[c - 1]))
            back[c - 1] = None
    outs.append(finish(chunks - 1, back[chunks - 1]))
    outs = [o for o in outs if o is not None]
    if not outs:
        return ops.combine(torch.empty((0, H), dtype=torch.float32, device=x.device), w)
    return torch.cat(outs)


class EPMoELayer:
    """The expert-parallel layer on this library's kernels: weights of this
    rank's E/R experts (bf16), top-k of the global E logits per token.
    ``chunks`` > 1 pipelines the rank's tokens through the exchange in that
    many chunks (every rank of the group must use the same value)."""

    def __init__(self, w13_local, w2_local, E, k, block_size, group=None, out_dtype=torch.bfloat16, chunks=1):
        import mixture_experts_expert_moe_b200 as m
        R = dist.get_world_size(group)
        if E % R or w13_local.shape[0] != E // R:
            raise ValueError("the experts must split evenly: w13_local holds E / world_size experts")
        if chunks < 1:
            raise ValueError("chunks must be at least 1")
        self.E, self.group, self.chunks = E, group, chunks
        self.ops = LibraryOps(m, w13_local, w2_local, k, block_size, out_dtype)

    def __call__(self, x, logits, bias=None, bias_mode="logits"):
        return ep_forward(self.ops, x, logits, self.E, self.group, bias, bias_mode, self.chunks)
