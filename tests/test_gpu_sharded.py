"""Row-sharded value table on one GPU: G ranks emulated as host threads, each with its own
stream, tokens and shard of the table; the exchanges between them go through host
memory barriers (no kernel waits on another).  The routing is checked bit for bit
against its plain statement (``tests/shard_ref.py``); the layer's outputs and
gradients against the oracle of the whole layer."""
import threading

import numpy as np
import pytest
import torch

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200 import sharded as S
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs
from tests import parity as H
from tests import shard_ref as SR

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from product_key_memory_pkm_b200 import build as B
    B.build()


def _cfg(**kw):
    base = dict(name="sharded", N=256, d_in=128, h=2, dk=64, C1=48, C2=40, k=8, d_v=72,
                dtype="bf16", score_scale=0.5)
    base.update(kw)
    return PKMConfig(**base)


class LoopbackHub:
    """All-to-all among G threads of one process: each deposits its pieces, waits for
    the others, copies what is addressed to it, waits again."""

    def __init__(self, G):
        self.G = G
        self.barrier = threading.Barrier(G, timeout=120)
        self.slots = [None] * G


class LoopbackExchange:
    def __init__(self, hub, rank):
        self.hub, self.rank = hub, rank

    def all_to_all(self, x, send_splits, recv_splits):
        torch.cuda.current_stream().synchronize()
        self.hub.slots[self.rank] = list(torch.split(x, send_splits))
        self.hub.barrier.wait()
        pieces = [self.hub.slots[src][self.rank] for src in range(self.hub.G)]
        assert [p.shape[0] for p in pieces] == list(recv_splits)
        out = torch.cat(pieces) if pieces else x[:0]
        torch.cuda.current_stream().synchronize()
        self.hub.barrier.wait()
        return out


def _run(cfg, G, seed=0):
    inp = make_inputs(cfg, seed=seed, random_bn=True)
    dev = H.to_dev(inp, cfg)
    bounds = np.linspace(0, cfg.N, G + 1).astype(int)   # ragged token batches
    hub = LoopbackHub(G)
    res, errors = [None] * G, []

    def rank_main(r):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                t0, t1 = bounds[r], bounds[r + 1]
                dims = P.Dims.from_config(cfg, N=int(t1 - t0))
                r0, r1 = S.shard_range(r, G, cfg.C1, cfg.C2)
                vs = dev["values"][r0:r1]
                ex = LoopbackExchange(hub, r)
                y, ctx = S.sharded_forward(dims, G, r, dev["x"][t0:t1], dev["Wq"], dev["bn"],
                                           dev["subkeys"], vs, ex)
                dV = torch.zeros(max(r1 - r0, 1), cfg.d_v, device="cuda")
                dx = torch.empty(t1 - t0, cfg.d_in, device="cuda")
                dWq = torch.zeros_like(dev["Wq"], dtype=torch.float32)
                dbn = torch.zeros(2, cfg.h * cfg.dk, device="cuda")
                dsub = torch.zeros_like(dev["subkeys"], dtype=torch.float32)
                res[r] = dict(y=y, idx=ctx.saved["idx"], dims=dims, ctx=ctx, dV=dV, dx=dx,
                              dWq=dWq, dbn=dbn, dsub=dsub, rows=(r0, r1), tok=(t0, t1), ex=ex,
                              vs=vs)
                torch.cuda.current_stream().synchronize()
        except BaseException as e:   # let the other threads fail instead of waiting
            errors.append(e)
            hub.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errors:
        raise errors[0]
    assert P.pkm_check_status() == P.PKM_OK
    return inp, dev, res


def _backward(res, dy_full, dev, G):
    errors = []
    hub = LoopbackHub(G)

    def rank_main(r):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                d = res[r]
                t0, t1 = d["tok"]
                ex = LoopbackExchange(hub, r)
                d["dw"] = S.sharded_backward(d["ctx"], dy_full[t0:t1].contiguous(), ex, d["vs"],
                                             d["dV"], dev["x"][t0:t1], dev["Wq"], dev["bn"],
                                             dev["subkeys"], d["dx"], d["dWq"], d["dbn"],
                                             d["dsub"])
                torch.cuda.current_stream().synchronize()
        except BaseException as e:
            errors.append(e)
            hub.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errors:
        raise errors[0]
    assert P.pkm_check_status() == P.PKM_OK


@pytest.mark.parametrize("G,kw", [
    (4, {}),
    (3, dict(C1=50, C2=24, N=200, h=3, d_v=136)),     # leading ranges of 17, 17, 16
    (8, dict(C1=20, C2=32, N=300, k=16, d_v=64)),     # 3 leading sub-keys a shard, last has 2
])
def test_row_sharded_layer_matches_the_oracle(G, kw):
    cfg = _cfg(**kw)
    inp, dev, res = _run(cfg, G)
    of = O.forward(inp, cfg)
    ranked = H.oracle_gaps(of, cfg)
    idx = np.concatenate([d["idx"].cpu().numpy() for d in res])
    clean = H.check_indices(idx, of, cfg, ranked)
    assert clean.mean() > 0.5
    y = np.concatenate([d["y"].cpu().numpy() for d in res])
    H.assert_rows(y[clean], of["y"][clean], "y")
    for t in np.nonzero(~clean)[0]:
        H.assert_rows(y[t:t + 1], H.oracle_bag_at(of, cfg, idx, t, inp["values"])[None], "y tie")
    # backward with dy on the clean tokens
    dy = inp["dy"] * clean[:, None]
    _backward(res, torch.from_numpy(dy).cuda(), dev, G)
    ob = O.backward(inp, cfg, of, dy)
    dw = np.concatenate([d["dw"].cpu().numpy() for d in res])
    dwg = H.align_to(idx[clean], of["idx"][clean], dw[clean])
    H.assert_rows(dwg.reshape(-1, cfg.k), ob["dw"][clean].reshape(-1, cfg.k), "dw")
    dV = np.zeros((cfg.K, cfg.d_v), np.float32)
    for d in res:
        r0, r1 = d["rows"]
        dV[r0:r1] = d["dV"][:r1 - r0].cpu().numpy()
    H.assert_rows(dV[ob["dV_rows"]], ob["dV_vals"], "dV")
    untouched = np.ones(cfg.K, dtype=bool)
    untouched[ob["dV_rows"]] = False
    assert not dV[untouched].any()
    dx = np.concatenate([d["dx"].cpu().numpy() for d in res])
    H.assert_rows(dx, ob["dx"], "dx")
    H.assert_rows(sum(d["dWq"] for d in res).cpu().numpy(), ob["dWq"], "dWq")
    H.assert_rows(sum(d["dsub"] for d in res).cpu().numpy().reshape(-1, cfg.dk // 2),
                  ob["dsub"].reshape(-1, cfg.dk // 2), "dsub", zero_rows=True)
    H.assert_rows(sum(d["dbn"] for d in res).cpu().numpy(),
                  np.stack([ob["dgamma"], ob["dbeta"]]), "dbn",
                  zero_rows=True)


@pytest.mark.parametrize("G,R", [(4, 480), (3, 700), (5, 400), (1, 1920)])
def test_routing_is_the_plain_statement_bit_for_bit(G, R):
    cfg = _cfg()
    inp = make_inputs(cfg, seed=1)
    dev = H.to_dev(inp, cfg)
    dims, saved, _ = H.gpu_forward(cfg, dev)
    N, hk = cfg.N, cfg.h * cfg.k
    counts = torch.empty(G, 2, dtype=torch.int32, device="cuda")
    segpos = torch.empty(G, N, dtype=torch.int32, device="cuda")
    send = torch.empty(N * hk, 3, dtype=torch.int32, device="cuda")
    perm = torch.empty(N * hk, dtype=torch.int32, device="cuda")
    ws = torch.empty(P.pkm_shard_workspace_bytes(dims, G, P.PKM_SHARD_ROUTE), dtype=torch.uint8,
                     device="cuda")
    P.pkm_shard_route(dims, G, R, saved["idx"], saved["w"], counts, segpos, send, perm, ws)
    c, sp, snd, pm = SR.route(saved["idx"].cpu().numpy().reshape(N, hk),
                              saved["w"].cpu().numpy().reshape(N, hk), G, R)
    np.testing.assert_array_equal(counts.cpu().numpy(), c)
    np.testing.assert_array_equal(segpos.cpu().numpy(), sp)
    np.testing.assert_array_equal(send.cpu().numpy(), snd)
    np.testing.assert_array_equal(perm.cpu().numpy(), pm)
    assert P.pkm_check_status() == P.PKM_OK


def test_owner_steps_are_the_plain_statement():
    """Bag and value gradient of one owner on triples from three sources, against the
    plain statement (fp64), with rows of one shard hit by several sources."""
    cfg = _cfg()
    rng = np.random.default_rng(7)
    G, shard_rows, d_v = 3, 300, cfg.d_v
    counts = np.zeros((G, 2), np.int32)
    parts = []
    for s in range(G):
        nseg = int(rng.integers(1, 40))
        per = rng.integers(1, 6, nseg)
        seg = np.repeat(np.arange(nseg), per)
        rows = rng.integers(0, shard_rows, seg.size)
        w = rng.random(seg.size).astype(np.float32)
        parts.append(np.stack([seg, rows, w.view(np.int32)], 1).astype(np.int32))
        counts[s] = (seg.size, nseg)
    recv = np.concatenate(parts)
    n_tri, n_seg = len(recv), int(counts[:, 1].sum())
    values = rng.standard_normal((shard_rows, d_v)).astype(np.float32)
    vb = torch.from_numpy(values).to(torch.bfloat16)
    dims = P.Dims.from_config(cfg)
    ws = torch.empty(P.pkm_shard_workspace_bytes(dims, G, P.PKM_SHARD_OWNER, n_tri),
                     dtype=torch.uint8, device="cuda")
    rc, rv = torch.from_numpy(counts).cuda(), torch.from_numpy(recv).cuda()
    part = torch.empty(n_seg, d_v, device="cuda")
    P.pkm_shard_bag(dims, G, shard_rows, rc, n_tri, n_seg, rv, vb.cuda(), part, ws)
    vref = vb.float().numpy().astype(np.float64)
    H.assert_rows(part.cpu().numpy(), SR.owner_bag(counts, recv, vref, d_v), "partial")
    dy = rng.standard_normal((n_seg, d_v)).astype(np.float32)
    dV = torch.zeros(shard_rows, d_v, device="cuda")
    dw = torch.empty(n_tri, device="cuda")
    P.pkm_shard_value_grad(dims, G, shard_rows, rc, n_tri, n_seg, rv, vb.cuda(),
                           torch.from_numpy(dy).cuda(), dV, dw, ws)
    dV_ref = np.zeros((shard_rows, d_v))
    dw_ref = SR.owner_value_grad(counts, recv, vref, dy.astype(np.float64), dV_ref)
    H.assert_rows(dV.cpu().numpy(), dV_ref, "dV")
    np.testing.assert_allclose(dw.cpu().numpy(), dw_ref, rtol=2e-3, atol=1e-3)
    assert P.pkm_check_status() == P.PKM_OK
