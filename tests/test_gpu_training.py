"""Training-time pieces on the device against the oracle: the compact value gradient
(pkm_value_grad_rows), lazy Adam on the selected rows (pkm_value_adam) and hit counts
(pkm_hit_counts) -- "Meta AI 可扩展内存层" sections 6.1, 6.3, 6.4 and 11.2.

Where a token has a near-tied head (decided from the oracle alone) its selection is not
unique: its upstream gradient is masked to zero, and the rows (and sub-keys) that either
valid selection could touch -- every key scoring within the tie tolerance of the k-th --
are left out of the row-wise comparisons.
"""
import numpy as np
import pytest
import torch

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs

from . import parity as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from product_key_memory_pkm_b200 import build as B
    B.build()


def _cfg(**kw):
    base = dict(name="train", N=300, d_in=128, h=4, dk=128, C1=64, C2=48, k=16, d_v=200,
                score_scale=0.5)
    base.update(kw)
    return PKMConfig(**base)


def _setup(cfg, seed):
    inp = make_inputs(cfg, seed=seed, random_bn=True)
    dev = H.to_dev(inp, cfg)
    dims, saved, _ = H.gpu_forward(cfg, dev)
    of = O.forward(inp, cfg)
    idx = saved["idx"].cpu().numpy().astype(np.int64)
    ranked = H.oracle_gaps(of, cfg)
    clean = H.check_indices(idx, of, cfg, ranked)
    # rows any valid selection of a near-tied head could take
    band = set()
    for t in np.nonzero(~clean)[0]:
        for hh in range(cfg.h):
            r = ranked[t, hh]
            tol = H.GAP_REL * max(abs(r[cfg.k - 1]), 1e-2)
            S = of["s1"][t, hh][:, None] + of["s2"][t, hh][None, :]
            band |= set(np.nonzero(S.ravel() >= r[cfg.k - 1] - tol)[0].tolist())
    return inp, dev, dims, saved, of, idx, clean, band


def test_value_grad_rows_matches_the_oracle_and_the_dense_form():
    cfg = _cfg()
    inp, dev, dims, saved, of, idx, clean, band = _setup(cfg, 1)
    dy = torch.from_numpy(inp["dy"] * clean[:, None]).cuda()
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    cap = min(cfg.N * cfg.h * cfg.k, cfg.K)
    rows = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    vals = torch.full((cap, cfg.d_v), float("nan"), device="cuda")
    nrows = torch.zeros(1, dtype=torch.int32, device="cuda")
    dw = torch.zeros(cfg.N, cfg.h, cfg.k, device="cuda")
    P.pkm_value_grad_rows(dims, dev["values"], saved, dy, rows, vals, nrows, dw=dw, workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    U = int(nrows.item())
    rg = rows[:U].cpu().numpy().astype(np.int64)
    vg = vals[:U].cpu().numpy()
    assert U == np.unique(idx).size and (np.diff(rg) > 0).all()
    np.testing.assert_array_equal(rg, np.unique(idx))
    # the dense form of the same stage: identical rows, zero elsewhere
    dV = torch.zeros(cfg.K, cfg.d_v, device="cuda")
    dw2 = torch.zeros_like(dw)
    P.pkm_value_grad(dims, dev["values"], saved, dy, dw2, dvalues=dV, workspace=ws)
    dVn = dV.cpu().numpy()
    np.testing.assert_array_equal(dVn[rg], vg)
    assert torch.equal(dw, dw2)
    # against the oracle on rows no near-tie can reach
    ob = O.backward(inp, cfg, of, inp["dy"] * clean[:, None])
    want = dict(zip(ob["dV_rows"].tolist(), ob["dV_vals"]))
    keep = [i for i, r in enumerate(rg) if r not in band]
    assert len(keep) > 0.5 * U
    got = vg[keep]
    exp = np.stack([want.get(int(rg[i]), np.zeros(cfg.d_v)) for i in keep])
    H.assert_rows(got, exp, "dV rows")


def test_value_adam_two_batches():
    """Two steps of lazy Adam on two different token batches (different row sets), fp32
    table and state; untouched rows and their state stay bit-identical."""
    cfg = _cfg(value_dtype="f32", N=160)
    inp1, dev1, dims, saved1, of1, idx1, clean1, band1 = _setup(cfg, 2)
    inp2, dev2, _, saved2, of2, idx2, clean2, band2 = _setup(cfg, 3)
    dev2["values"] = dev1["values"]           # one table, two batches
    inp2["values"] = inp1["values"]
    V0 = dev1["values"].clone()
    m = torch.zeros_like(V0)
    v = torch.zeros_like(V0)
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    lr, b1, b2, eps = 0.01, 0.9, 0.99, 1e-8
    Vo, Mo, So = (np.asarray(inp1["values"], np.float64), np.zeros(V0.shape),
                  np.zeros(V0.shape))
    for step, (inp, saved, of, clean) in enumerate(((inp1, saved1, of1, clean1),
                                                    (inp2, saved2, of2, clean2)), start=1):
        dyn = inp["dy"] * clean[:, None]
        P.pkm_value_adam(dims, lr, b1, b2, eps, step, dev1["values"], m, v, saved,
                         torch.from_numpy(dyn).cuda(), workspace=ws)
        assert P.pkm_check_status() == P.PKM_OK
        ob = O.backward(dict(inp, values=Vo), cfg, of, dyn)
        Vo, Mo, So = O.sparse_adam(Vo, Mo, So, ob["dV_rows"], ob["dV_vals"], lr, b1, b2, eps,
                                   step)
    band = band1 | band2
    touched = np.union1d(np.unique(idx1), np.unique(idx2))
    keep = np.array([r for r in touched if r not in band])
    assert keep.size > 0.5 * touched.size
    kt = torch.from_numpy(keep).cuda()
    for name, got, want in (("V update", dev1["values"][kt] - V0[kt], Vo[keep] - np.asarray(
            inp1["values"], np.float64)[keep]), ("m", m[kt], Mo[keep]), ("v", v[kt], So[keep])):
        H.assert_rows(got.double().cpu().numpy(), want, name)
    untouched = torch.ones(cfg.K, dtype=torch.bool, device="cuda")
    untouched[torch.from_numpy(touched).cuda()] = False
    assert torch.equal(dev1["values"][untouched], V0[untouched])
    assert not m[untouched].any() and not v[untouched].any()


def test_hit_counts_match_the_oracle_and_accumulate():
    cfg = _cfg()
    inp, dev, dims, saved, of, idx, clean, band = _setup(cfg, 4)
    slot = torch.zeros(cfg.K, dtype=torch.int32, device="cuda")
    sub = torch.zeros(cfg.h, cfg.C1 + cfg.C2, dtype=torch.int32, device="cuda")
    P.pkm_hit_counts(dims, saved["idx"], slot, sub)
    assert P.pkm_check_status() == P.PKM_OK
    sg, ug = slot.cpu().numpy(), sub.cpu().numpy()
    so, uo = O.hit_counts(of, cfg)
    assert sg.sum() == cfg.N * cfg.h * cfg.k and (ug.sum(1) == 2 * cfg.N * cfg.k).all()
    # differences only where a near-tied head could have chosen either way
    diff = np.nonzero(sg != so)[0]
    assert set(diff.tolist()) <= band
    band_sub1 = {r // cfg.C2 for r in band}
    band_sub2 = {cfg.C1 + r % cfg.C2 for r in band}
    for hh in range(cfg.h):
        bad = set(np.nonzero(ug[hh] != uo[hh])[0].tolist())
        assert bad <= band_sub1 | band_sub2
    # accumulate semantics
    P.pkm_hit_counts(dims, saved["idx"], slot, None)
    assert (slot.cpu().numpy() == 2 * sg).all()
