"""Row-sharded product-key memory over G ranks ("Meta AI 可扩展内存层", 9.1: the value
matrix split by rows of the product-key index, each device reading only its own rows,
the candidate indices and partial weighted sums exchanged between devices).

Rank g owns a batch of tokens and the value rows [g*R, min((g+1)*R, C1*C2)) with
R = ceil(C1/G) * C2: a range of leading sub-key indices (4.5 of the same page: row
i*|C'| + j).  Every step of the layer runs in the library's kernels (``pkm``); this
module holds only the order of the calls and the exchanges between ranks, made by an
exchange object:

* ``TorchExchange``: ``torch.distributed.all_to_all_single`` on a process group (NCCL
  on GPUs, gloo on CPUs);
* ``LocalExchange``: one rank, nothing to move.

Forward on every rank: F1-F3 for its tokens (``pkm_query``, ``pkm_subkey_scores``,
``pkm_candidate_topk``; the query network and sub-keys are replicated), then
``pkm_shard_route``; counts, triples out; ``pkm_shard_bag`` on the triples received;
partial rows back; ``pkm_shard_combine``.  Backward: ``pkm_shard_gather_dy``; dy rows
out; ``pkm_shard_value_grad`` (dV of the rank's own rows, dL/dw of the triples it
received); dL/dw back; ``pkm_shard_scatter_dw``; ``pkm_query_grad``.  The gradients of
the replicated parameters (Wq, BatchNorm, sub-keys) are per rank, for the caller's
data-parallel reduction; dV stays on the rank that owns the rows.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import pkm as P


def rows_per_shard(C1: int, C2: int, G: int) -> int:
    """R: the rows of ceil(C1 / G) leading sub-key indices."""
    return -(-C1 // G) * C2


def shard_range(g: int, G: int, C1: int, C2: int) -> tuple[int, int]:
    """Rows [start, stop) of shard g (empty for trailing shards when G > C1)."""
    R = rows_per_shard(C1, C2, G)
    K = C1 * C2
    return min(g * R, K), min((g + 1) * R, K)


class LocalExchange:
    """One rank: every all-to-all returns what the rank sent itself."""

    def all_to_all(self, x: torch.Tensor, send_splits: list[int],
                   recv_splits: list[int]) -> torch.Tensor:
        assert list(send_splits) == list(recv_splits) and len(send_splits) == 1
        return x


class TorchExchange:
    """All-to-all over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, x: torch.Tensor, send_splits: list[int],
                   recv_splits: list[int]) -> torch.Tensor:
        import torch.distributed as dist
        out = x.new_empty((sum(recv_splits),) + tuple(x.shape[1:]))
        dist.all_to_all_single(out, x.contiguous(), recv_splits, send_splits, group=self.group)
        return out


@dataclass
class ShardedContext:
    dims: P.Dims
    G: int
    rank: int
    shard_rows: int
    saved: dict
    segpos: torch.Tensor
    perm: torch.Tensor
    recv: torch.Tensor
    recv_counts: torch.Tensor
    send_tri: list[int]
    send_seg: list[int]
    recv_tri: list[int]
    recv_seg: list[int]
    owner_ws: torch.Tensor


def _bytes(n: int, device) -> torch.Tensor:
    return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)


def sharded_forward(dims: P.Dims, G: int, rank: int, x, Wq, bn, subkeys, values_shard,
                    exchange, ops=P, stream=None):
    """y [N][d_v] for this rank's N tokens; the context the backward needs."""
    dev = x.device
    R = rows_per_shard(dims.C1, dims.C2, G)
    r0, r1 = shard_range(rank, G, dims.C1, dims.C2)
    shard_rows = max(r1 - r0, 1)
    hk = dims.h * (dims.k * dims.k if dims.flags & P.PKM_F_ALL_K2 else dims.k)
    saved = ops.alloc_saved(dims, device=dev)
    ops.pkm_query(dims, x, Wq, bn, saved, stream=stream)
    ops.pkm_subkey_scores(dims, subkeys, saved, stream=stream)
    ops.pkm_candidate_topk(dims, saved, stream=stream)
    counts = torch.empty(G, 2, dtype=torch.int32, device=dev)
    segpos = torch.empty(G, max(dims.N, 1), dtype=torch.int32, device=dev)
    send = torch.empty(max(dims.N * hk, 1), 3, dtype=torch.int32, device=dev)
    perm = torch.empty(max(dims.N * hk, 1), dtype=torch.int32, device=dev)
    ws = _bytes(ops.pkm_shard_workspace_bytes(dims, G, P.PKM_SHARD_ROUTE), dev)
    ops.pkm_shard_route(dims, G, R, saved["idx"], saved["w"], counts, segpos, send, perm, ws,
                        stream=stream)
    recv_counts = exchange.all_to_all(counts, [1] * G, [1] * G)
    ch, rh = counts.cpu().tolist(), recv_counts.cpu().tolist()
    send_tri, send_seg = [c[0] for c in ch], [c[1] for c in ch]
    recv_tri, recv_seg = [c[0] for c in rh], [c[1] for c in rh]
    recv = exchange.all_to_all(send[:sum(send_tri)], send_tri, recv_tri)
    n_tri, n_seg = sum(recv_tri), sum(recv_seg)
    owner_ws = _bytes(ops.pkm_shard_workspace_bytes(dims, G, P.PKM_SHARD_OWNER, n_tri), dev)
    partial = torch.empty(max(n_seg, 1), dims.d_v, dtype=torch.float32, device=dev)
    ops.pkm_shard_bag(dims, G, shard_rows, recv_counts, n_tri, n_seg, recv, values_shard,
                      partial, owner_ws, stream=stream)
    back = exchange.all_to_all(partial[:n_seg], recv_seg, send_seg)
    y = torch.empty(dims.N, dims.d_v, dtype=torch.float32, device=dev)
    ops.pkm_shard_combine(dims, G, segpos, back, sum(send_seg), y, stream=stream)
    ctx = ShardedContext(dims, G, rank, shard_rows, saved, segpos, perm, recv, recv_counts,
                         send_tri, send_seg, recv_tri, recv_seg, owner_ws)
    return y, ctx


def sharded_backward(ctx: ShardedContext, dy, exchange, values_shard, dvalues_shard, x=None,
                     Wq=None, bn=None, subkeys=None, dx=None, dWq=None, dbn=None, dsubkeys=None,
                     query_grad: bool = True, ops=P, stream=None):
    """dV of this rank's rows (+= into dvalues_shard) and dL/dw of its own selections
    ([N][h][k], returned); with query_grad, the query-side gradients as pkm_query_grad."""
    dims, G, dev = ctx.dims, ctx.G, dy.device
    hk = ctx.saved["idx"].shape[1] * ctx.saved["idx"].shape[2]
    n_send = sum(ctx.send_seg)
    dy_send = torch.empty(max(n_send, 1), dims.d_v, dtype=torch.float32, device=dev)
    ops.pkm_shard_gather_dy(dims, G, ctx.segpos, dy, dy_send, n_send, stream=stream)
    dy_recv = exchange.all_to_all(dy_send[:n_send], ctx.send_seg, ctx.recv_seg)
    n_tri, n_seg = sum(ctx.recv_tri), sum(ctx.recv_seg)
    dw_recv = torch.empty(max(n_tri, 1), dtype=torch.float32, device=dev)
    ops.pkm_shard_value_grad(dims, G, ctx.shard_rows, ctx.recv_counts, n_tri, n_seg, ctx.recv,
                             values_shard, dy_recv, dvalues_shard, dw_recv, ctx.owner_ws,
                             stream=stream)
    dw_ret = exchange.all_to_all(dw_recv[:n_tri], ctx.recv_tri, ctx.send_tri)
    dw = torch.empty(dims.N, hk, dtype=torch.float32, device=dev)
    ops.pkm_shard_scatter_dw(dims, ctx.perm, dw_ret, dw, stream=stream)
    dw = dw.view(dims.N, ctx.saved["idx"].shape[1], ctx.saved["idx"].shape[2])
    if query_grad:
        ws = _bytes(ops.pkm_workspace_bytes(dims, P.PKM_BWD), dev)
        ops.pkm_query_grad(dims, x, Wq, bn, subkeys, ctx.saved, dw, dx, dWq, dbn, dsubkeys, ws,
                           stream=stream)
    return dw
