"""Plain statement of the row-sharded exchange (test infrastructure).

What the library's pkm_shard_* entry points compute, written as loops over tokens and
selections: routing of each selection to the shard that holds its row ("Meta AI
可扩展内存层", 9.1: value rows split over devices, candidate indices and partial
weighted sums exchanged), the owner's partial bags and value gradients, and the
source's combine.  ``CpuOps`` wraps them (and the oracle's selection) with the
signatures of the binding, so the orchestration in ``sharded.py`` can run on CPU ranks
over gloo.
"""
from __future__ import annotations

import numpy as np
import torch


def route(idx: np.ndarray, w: np.ndarray, G: int, R: int):
    """idx, w: [N][hk].  Per destination g: the selections of token 0, then token 1, ...
    in selection order, as (segment, row - g*R, w bits); a segment is one token's run
    for g, numbered from 0 per g.  segpos[g][t]: row of the combined return buffer
    (shard 0's segments first) holding t's partial from g, or -1."""
    N, hk = idx.shape
    per_dest = [[] for _ in range(G)]
    for t in range(N):
        for s in range(hk):
            per_dest[int(idx[t, s]) // R].append((t, s))
    counts = np.zeros((G, 2), np.int32)
    segpos = np.full((G, N), -1, np.int32)
    send, perm = [], []
    base = 0
    wbits = np.ascontiguousarray(w, dtype=np.float32).view(np.int32)
    for g in range(G):
        seg_of = {}
        for t, _ in per_dest[g]:
            if t not in seg_of:
                seg_of[t] = len(seg_of)
                segpos[g, t] = base + seg_of[t]
        for t, s in per_dest[g]:
            send.append((seg_of[t], int(idx[t, s]) - g * R, int(wbits[t, s])))
            perm.append(t * hk + s)
        counts[g] = (len(per_dest[g]), len(seg_of))
        base += len(seg_of)
    return (counts, segpos, np.array(send, np.int32).reshape(-1, 3),
            np.array(perm, np.int32))


def _offsets(recv_counts: np.ndarray):
    tri = np.concatenate([[0], np.cumsum(recv_counts[:, 0])])
    seg = np.concatenate([[0], np.cumsum(recv_counts[:, 1])])
    return tri, seg


def _segments(recv_counts, recv):
    """Global segment of every received triple (sources in order)."""
    tri, seg = _offsets(recv_counts)
    out = np.zeros(len(recv), np.int64)
    for s in range(len(recv_counts)):
        out[tri[s]:tri[s + 1]] = seg[s] + recv[tri[s]:tri[s + 1], 0]
    return out


def owner_bag(recv_counts, recv, values, d_v):
    n_seg = int(recv_counts[:, 1].sum())
    w = recv[:, 2].astype(np.int32).view(np.float32).astype(np.float64)
    part = np.zeros((n_seg, d_v))
    for i, j in enumerate(_segments(recv_counts, recv)):
        part[j] += w[i] * values[recv[i, 1]]
    return part


def combine(segpos, back):
    G, N = segpos.shape
    y = np.zeros((N, back.shape[1]))
    for t in range(N):
        for g in range(G):
            if segpos[g, t] >= 0:
                y[t] += back[segpos[g, t]]
    return y


def gather_dy(segpos, dy, n_rows):
    out = np.zeros((n_rows, dy.shape[1]))
    G, N = segpos.shape
    for g in range(G):
        for t in range(N):
            if segpos[g, t] >= 0:
                out[segpos[g, t]] = dy[t]
    return out


def owner_value_grad(recv_counts, recv, values, dy_recv, dV):
    w = recv[:, 2].astype(np.int32).view(np.float32).astype(np.float64)
    dw = np.zeros(len(recv))
    for i, j in enumerate(_segments(recv_counts, recv)):
        r = recv[i, 1]
        dw[i] = dy_recv[j] @ values[r]
        dV[r] += w[i] * dy_recv[j]
    return dw


def scatter_dw(perm, dw_ret, n):
    dw = np.zeros(n)
    dw[perm] = dw_ret
    return dw


class CpuOps:
    """The binding's signatures on CPU tensors: selection from the oracle's results for
    this rank's tokens [t0, t0 + N), the exchange steps from the functions above."""

    def __init__(self, of: dict, t0: int):
        self.of, self.t0 = of, t0

    # -- F1-F3: the oracle's selection of this rank's tokens
    def alloc_saved(self, dims, device="cpu"):
        ksel = dims.k
        return dict(idx=torch.zeros(dims.N, dims.h, ksel, dtype=torch.int32),
                    w=torch.zeros(dims.N, dims.h, ksel, dtype=torch.float32))

    def pkm_query(self, dims, x, Wq, bn, saved, stream=None):
        pass

    def pkm_subkey_scores(self, dims, subkeys, saved, stream=None):
        pass

    def pkm_candidate_topk(self, dims, saved, stream=None):
        sl = slice(self.t0, self.t0 + dims.N)
        saved["idx"][:] = torch.from_numpy(self.of["idx"][sl].astype(np.int32))
        saved["w"][:] = torch.from_numpy(self.of["w"][sl].astype(np.float32))

    def pkm_shard_workspace_bytes(self, dims, G, which, n_triples=0):
        return 0

    def pkm_workspace_bytes(self, dims, which):
        return 0

    # -- the exchange steps
    def pkm_shard_route(self, dims, G, R, idx, w, counts, segpos, send, perm, ws, stream=None):
        hk = idx.shape[1] * idx.shape[2]
        c, sp, snd, pm = route(idx.reshape(dims.N, hk).numpy(), w.reshape(dims.N, hk).numpy(),
                               G, R)
        counts[:] = torch.from_numpy(c)
        segpos[:, :dims.N] = torch.from_numpy(sp)
        send[:len(snd)] = torch.from_numpy(snd)
        perm[:len(pm)] = torch.from_numpy(pm)

    def pkm_shard_bag(self, dims, G, shard_rows, recv_counts, n_tri, n_seg, recv, values,
                      partial, ws, stream=None):
        if n_seg:
            partial[:n_seg] = torch.from_numpy(
                owner_bag(recv_counts.numpy(), recv.numpy(), values.double().numpy(),
                          dims.d_v)).float()

    def pkm_shard_combine(self, dims, G, segpos, back, n_rows, y, stream=None):
        y[:] = torch.from_numpy(combine(segpos[:, :dims.N].numpy(), back.double().numpy()))

    def pkm_shard_gather_dy(self, dims, G, segpos, dy, dy_send, n_rows, stream=None):
        if n_rows:
            dy_send[:n_rows] = torch.from_numpy(
                gather_dy(segpos[:, :dims.N].numpy(), dy.double().numpy(), n_rows)).float()

    def pkm_shard_value_grad(self, dims, G, shard_rows, recv_counts, n_tri, n_seg, recv, values,
                             dy_recv, dvalues, dw_recv, ws, stream=None):
        if n_tri:
            dV = dvalues.double().numpy().copy()
            dw = owner_value_grad(recv_counts.numpy(), recv.numpy(), values.double().numpy(),
                                  dy_recv.double().numpy(), dV)
            dvalues[:] = torch.from_numpy(dV).to(dvalues.dtype)
            dw_recv[:n_tri] = torch.from_numpy(dw).float()

    def pkm_shard_scatter_dw(self, dims, perm, dw_ret, dw, stream=None):
        n = dw.numel()
        dw.view(-1)[:] = torch.from_numpy(scatter_dw(perm[:n].numpy(), dw_ret.double().numpy(),
                                                     n)).float()
