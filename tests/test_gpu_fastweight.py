"""Fast-weight memory, chunked read-then-write: the CUDA path (pkm_fastweight_chunks)
against the oracle's chunk loop ("Fast-weight Product Key Memory", sections 2.2 and 3).

What is compared:
  * every chunk's read y[t] (row relative error 2e-3), for tokens whose result is
    unique (below);
  * the write: V_final[r] - V_initial[r] on every written row, same tolerance;
  * rows no chunk selected: bit-identical to the initial table.

The cases are chosen so that most tokens stay comparable: with clustered queries and
many heads, one near-tie early in the sequence taints a growing share of later tokens.

Selection does not depend on the value table (queries and keys are fixed), so the
oracle's gaps over the whole sequence decide which tokens have a unique key set.  A
token with a near-tied head may select either of several valid sets (checked for
validity); its residual then differs, so the rows it writes -- by either selection --
are "tainted" from the next chunk on, and every later token that reads a tainted row is
itself left out of the direct comparison and taints the rows it writes.  Written rows
that end tainted are left out of the table comparison.
"""
import numpy as np
import pytest
import torch

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200.inputs import FASTWEIGHT, PKMConfig, make_inputs, make_targets

from . import parity as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from product_key_memory_pkm_b200 import build as B
    B.build()


def _cfg(**kw):
    base = dict(name="fw_small", N=200, d_in=64, h=1, dk=32, C1=32, C2=32, k=8, d_v=64,
                dtype="f32", clustered=8)
    base.update(kw)
    return PKMConfig(**base)


def _run(cfg, seed, chunk, lr, lookahead, select="brute", min_good=0.5, strategy=0):
    inp = make_inputs(cfg, seed=seed, with_dy=False)
    targets = None if lookahead else make_targets(cfg, seed)
    ys_o, rows_o, vals_o = O.fastweight_chunks(inp, cfg, chunk, lr, targets=targets,
                                               lookahead=lookahead, select=select)

    dev = H.to_dev(inp, cfg)
    dims = P.Dims.from_config(cfg)
    V0 = dev["values"].clone()
    y = torch.full((cfg.N, cfg.d_v), float("nan"), device="cuda")
    mode = strategy | (P.PKM_FW_LOOKAHEAD if lookahead else 0)
    ws = P.alloc_fastweight_workspace(dims, chunk, mode)
    tg = None if lookahead else torch.from_numpy(np.asarray(targets, np.float32)).cuda()
    P.pkm_fastweight_chunks(dims, chunk, lr, dev["x"], dev["Wq"], dev["bn"], dev["subkeys"],
                            dev["values"], y, targets=tg, lookahead=lookahead, strategy=strategy,
                            workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK

    # the GPU's selection (the same kernels on the whole sequence; selection does not
    # read the value table)
    _, saved, _ = H.gpu_forward(cfg, dev)
    idx_g = saved["idx"].cpu().numpy().astype(np.int64)
    of = _selection_only(inp, cfg, select)
    ranked = H.oracle_gaps(of, cfg, select=select)
    clean = H.check_indices(idx_g, of, cfg, ranked)

    # taint propagation over chunks
    good = np.ones(cfg.N, dtype=bool)
    tainted = set()
    for c0 in range(0, cfg.N, chunk):
        c1 = min(cfg.N, c0 + chunk)
        new = set()
        for t in range(c0, c1):
            rows_t = set(of["idx"][t].ravel().tolist()) | set(idx_g[t].ravel().tolist())
            if not clean[t] or (rows_t & tainted):
                good[t] = False
                new |= rows_t
        tainted |= new
    assert good.mean() >= min_good, f"only {good.mean():.2f} of tokens comparable"

    H.assert_rows(y.cpu().numpy()[good], ys_o[good], "y")
    rows_t = torch.from_numpy(rows_o).cuda()
    keep = np.array([int(r) not in tainted for r in rows_o], dtype=bool)
    dV_g = (dev["values"][rows_t].double() - V0[rows_t].double()).cpu().numpy()
    dV_o = vals_o - np.asarray(inp["values"][rows_o], dtype=np.float64)
    H.assert_rows(dV_g[keep], dV_o[keep], "V update")
    # rows no chunk selected (by either side) are untouched, bit for bit
    untouched = torch.ones(cfg.K, dtype=torch.bool, device="cuda")
    untouched[rows_t] = False
    untouched[torch.from_numpy(np.unique(idx_g)).cuda()] = False
    assert torch.equal(dev["values"][untouched], V0[untouched])
    return good


def _selection_only(inp, cfg, select):
    """The oracle's selection for a big table without reading the value table."""
    small = dict(inp, values=np.zeros((cfg.K, 1), dtype=np.float32))
    return O.forward(small, cfg, select=select)


STRATEGIES = {"chunk_sort": 0, "global_sort": P.PKM_FW_SORT_GLOBAL,
              "per_chunk": P.PKM_FW_PER_CHUNK}


@pytest.mark.parametrize("strategy", list(STRATEGIES))
def test_fastweight_explicit_targets_ragged_last_chunk(strategy):
    _run(_cfg(), seed=1, chunk=64, lr=0.5, lookahead=False, strategy=STRATEGIES[strategy])


@pytest.mark.parametrize("strategy", list(STRATEGIES))
def test_fastweight_lookahead_targets(strategy):
    _run(_cfg(), seed=2, chunk=64, lr=0.5, lookahead=True, strategy=STRATEGIES[strategy])


@pytest.mark.parametrize("strategy", list(STRATEGIES))
def test_fastweight_two_heads_duplicate_heavy(strategy):
    _run(_cfg(h=2, clustered=4, k=16), seed=3, chunk=50, lr=0.25, lookahead=False,
         strategy=STRATEGIES[strategy])


def test_fastweight_one_token_chunks():
    _run(_cfg(N=40), seed=4, chunk=1, lr=0.5, lookahead=True)


def test_fastweight_single_chunk_and_k1_rate_one():
    _run(_cfg(k=1, clustered=0, C1=64, C2=64), seed=5, chunk=1000, lr=1.0, lookahead=False)


def test_fastweight_wide_rows_unequal_halves():
    _run(_cfg(d_in=1032, d_v=1032, C1=48, C2=24, clustered=16, N=130), seed=6, chunk=64, lr=0.1,
         lookahead=True)


def test_fastweight_chunk_sort_at_its_size_limit():
    """Chunks of exactly 16384 selections (the largest sorted in shared memory: 512 tokens
    x h = 2 x k = 16), a ragged last chunk of fewer."""
    _run(_cfg(N=1100, h=2, k=16, dk=64, C1=512, C2=512, clustered=0), seed=8, chunk=512,
         lr=0.5, lookahead=True)


def _mixed(**kw):
    """bf16 x, Wq, sub-keys (tensor-core query and scoring) beside an fp32 value table."""
    base = dict(dtype="bf16", value_dtype="f32", d_in=128, dk=128, d_v=128)
    base.update(kw)
    return _cfg(**base)


def test_fastweight_bf16_inputs_fp32_values_explicit_targets():
    _run(_mixed(N=300, h=2, k=16, C1=128, C2=96, clustered=0), seed=10, chunk=96, lr=0.5,
         lookahead=False)


def test_fastweight_bf16_inputs_fp32_values_lookahead():
    """Lookahead targets read the next token's bf16 input (clustered: rows repeat)."""
    _run(_mixed(N=257, C1=64, C2=64), seed=11, chunk=64, lr=0.5, lookahead=True)


def test_fastweight_zero_tokens_is_a_no_op():
    cfg = _cfg(N=0)
    dims = P.Dims.from_config(cfg)
    z = torch.zeros(16, device="cuda")
    P.pkm_fastweight_chunks(dims, 64, 0.5, z, z, z, z, z, z, targets=z, workspace=z)


def test_fastweight_full_size_workload():
    """The 4096-token, 1M-slot fast-weight workload (8 chunks of 512, fp32 table of
    4.3 GB, 64 input clusters), whole sequence compared."""
    _run(FASTWEIGHT, seed=0, chunk=512, lr=1.0, lookahead=False, select="product", min_good=0.5)


def test_value_sgd_step_matches_the_oracle_gradient():
    """pkm_value_sgd alone: V - lr * dV, with dV the oracle's value gradient of
    sum_t dy[t] . y[t] (upstream gradient masked to tokens with a unique key set)."""
    cfg = _cfg(N=300, h=2, k=16, clustered=6)
    inp = make_inputs(cfg, seed=9)
    dev = H.to_dev(inp, cfg)
    dims, saved, _ = H.gpu_forward(cfg, dev)
    of = O.forward(inp, cfg)
    idx_g = saved["idx"].cpu().numpy().astype(np.int64)
    clean = H.check_indices(idx_g, of, cfg, H.oracle_gaps(of, cfg))
    assert clean.mean() > 0.5
    dy = inp["dy"] * clean[:, None]
    b = O.backward(inp, cfg, of, dy)
    V0 = dev["values"].clone()
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    lr = 0.75
    P.pkm_value_sgd(dims, lr, dev["values"], saved, torch.from_numpy(dy.astype(np.float32)).cuda(),
                    workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    rows = torch.from_numpy(b["dV_rows"]).cuda()
    got = (dev["values"][rows].double() - V0[rows].double()).cpu().numpy()
    H.assert_rows(got, -lr * b["dV_vals"], "V update")
    untouched = torch.ones(cfg.K, dtype=torch.bool, device="cuda")
    untouched[torch.from_numpy(np.unique(idx_g)).cuda()] = False
    assert torch.equal(dev["values"][untouched], V0[untouched])
