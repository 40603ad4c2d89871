"""The benchmark's multi-GPU path runs replicas: every rank the same tables and its own
tokens, timings reduced to the slowest rank.  Its host logic is exercised here with two
gloo ranks on the CPU (no GPU, no collective on the data path)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from product_key_memory_pkm_b200.inputs import PKMConfig

CFG = PKMConfig("ranks", N=12, d_in=16, h=2, dk=8, C1=6, C2=5, k=3, d_v=8, dtype="f32")


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        inp = bench.rank_batch(CFG, rank, world)
        tables = np.concatenate([np.ravel(inp[k]) for k in ("Wq", "subkeys", "values", "bn")])
        tok = np.concatenate([np.ravel(inp["x"]), np.ravel(inp["dy"])])
        gathered = [None] * world
        dist.all_gather_object(gathered, (tables.tobytes(), tok.tobytes()))
        m = bench.max_over_ranks([1.0 + rank, 5.0 - rank], dist, "cpu")
        out[rank] = (gathered, m)
    finally:
        dist.destroy_process_group()


def test_replicas_share_tables_and_split_tokens():
    port = 29500 + (os.getpid() % 2000)
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    gathered, m0 = res[0]
    _, m1 = res[1]
    assert gathered[0][0] == gathered[1][0]        # the same tables on every rank
    assert gathered[0][1] != gathered[1][1]        # each rank its own tokens
    assert m0 == m1 == [2.0, 5.0]                  # every timing is the slowest rank's


def test_single_rank_keeps_the_seed_zero_batch():
    import bench
    from product_key_memory_pkm_b200.inputs import make_inputs
    a = bench.rank_batch(CFG, 0, 1)
    b = make_inputs(CFG, seed=0)
    for k in b:
        np.testing.assert_array_equal(a[k], b[k])
    assert bench.max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]
