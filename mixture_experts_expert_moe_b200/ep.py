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


def ep_forward(ops, x, logits, E, group=None, bias=None, bias_mode="logits"):
    """One expert-parallel layer forward of this rank's tokens (module
    docstring).  Every rank of ``group`` must call it, in the same order."""
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


class EPMoELayer:
    """The expert-parallel layer on this library's kernels: weights of this
    rank's E/R experts (bf16), top-k of the global E logits per token."""

    def __init__(self, w13_local, w2_local, E, k, block_size, group=None, out_dtype=torch.bfloat16):
        import mixture_experts_expert_moe_b200 as m
        R = dist.get_world_size(group)
        if E % R or w13_local.shape[0] != E // R:
            raise ValueError("the experts must split evenly: w13_local holds E / world_size experts")
        self.E, self.group = E, group
        self.ops = LibraryOps(m, w13_local, w2_local, k, block_size, out_dtype)

    def __call__(self, x, logits, bias=None, bias_mode="logits"):
        return ep_forward(self.ops, x, logits, self.E, self.group, bias, bias_mode)
