"""Row-sharded value table ("Meta AI 可扩展内存层", 9.1) over gloo ranks on the CPU: the
orchestration in ``sharded.py`` with its exchanges over torch.distributed, the steps
from ``tests/shard_ref.py`` (the plain statement of what the kernels compute), checked
against the oracle of the whole layer: every rank's bag, its dL/dw and the value
gradient of the rows it owns."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200 import sharded as S
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs
from tests.shard_ref import CpuOps

# 7 leading sub-keys over the ranks: shards of 4 and 3 (two ranks), 3, 3, 1 (three)
CFG = PKMConfig("sharded", N=24, d_in=16, h=2, dk=8, C1=7, C2=5, k=3, d_v=8, dtype="f32")


def _worker(rank, world, port, out, bounds):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = make_inputs(CFG, seed=3, random_bn=True)
        of = O.forward(inp, CFG)
        t0 = bounds[rank]
        n = bounds[rank + 1] - t0
        dims = P.Dims.from_config(CFG, N=n)
        ops = CpuOps(of, t0)
        r0, r1 = S.shard_range(rank, world, CFG.C1, CFG.C2)
        values_shard = torch.from_numpy(inp["values"][r0:r1].astype(np.float64))
        ex = S.TorchExchange()
        x = torch.from_numpy(inp["x"][t0:t0 + n])
        y, ctx = S.sharded_forward(dims, world, rank, x, None, None, None, values_shard, ex,
                                   ops=ops)
        dV = torch.zeros(r1 - r0, CFG.d_v, dtype=torch.float64)
        dy = torch.from_numpy(inp["dy"][t0:t0 + n].astype(np.float64))
        dw = S.sharded_backward(ctx, dy, ex, values_shard, dV, query_grad=False, ops=ops)
        out[rank] = (y.numpy(), dw.numpy(), dV.numpy(), r0, r1, ctx.send_tri, ctx.recv_tri)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,bounds", [
    (2, (0, 12, 24)),
    (3, (0, 8, 16, 24)),
    (2, (0, 24, 24)),          # rank 1 has no tokens; it still owns rows and serves rank 0
])
def test_row_sharded_layer_over_gloo_ranks_matches_the_oracle(world, bounds):
    port = 29700 + world * 10 + bounds[1] + (os.getpid() % 500)
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out, bounds), nprocs=world, join=True)
        res = [out[r] for r in range(world)]
    inp = make_inputs(CFG, seed=3, random_bn=True)
    of = O.forward(inp, CFG)
    ob = O.backward(inp, CFG, of, inp["dy"])
    y = np.concatenate([r[0] for r in res])
    dw = np.concatenate([r[1] for r in res])
    np.testing.assert_allclose(y, of["y"], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(dw, ob["dw"], rtol=1e-5, atol=1e-6)
    dV_full = np.zeros((CFG.K, CFG.d_v))
    dV_full[ob["dV_rows"]] = ob["dV_vals"]
    for (_, _, dV, r0, r1, _, _) in res:
        np.testing.assert_allclose(dV, dV_full[r0:r1], rtol=1e-5, atol=1e-6)
    # every selection travels once, and what a rank receives is what the others sent it
    sent = np.array([r[5] for r in res])
    recv = np.array([r[6] for r in res])
    assert sent.sum() == CFG.N * CFG.h * CFG.k
    np.testing.assert_array_equal(sent.T, recv)


def test_shard_ranges_cover_the_table_once():
    for C1, C2, G in [(7, 5, 2), (7, 5, 3), (1024, 1024, 8), (5, 3, 8)]:
        rows = [S.shard_range(g, G, C1, C2) for g in range(G)]
        assert rows[0][0] == 0 and rows[-1][1] == C1 * C2
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
        assert all(r[0] % C2 == 0 for r in rows)   # whole leading sub-key ranges
