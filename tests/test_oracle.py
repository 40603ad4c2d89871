"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test is chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, a wrong tie-break) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200.inputs import PKMConfig, TINY_FP32, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cfg(**kw):
    base = dict(name="t", N=8, d_in=16, h=2, dk=8, C1=12, C2=9, k=4, d_v=6, dtype="f32")
    base.update(kw)
    return PKMConfig(**base)


# --------------------------------------------------------------------------- golden
def test_golden_worked_example():
    """Hand-derived case (tests/golden/worked_example_k3.json): every forward and
    backward quantity is a closed-form number."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_k3.json")))
    cfg = PKMConfig(name="golden", dtype="f32", **g["cfg"])
    inp = {k: np.array(g[k], dtype=np.float64) for k in ("x", "Wq", "bn", "subkeys", "values")}
    f = O.forward(inp, cfg)
    e = g["expect"]
    np.testing.assert_allclose(f["q"], e["q"], atol=1e-15)
    np.testing.assert_allclose(f["s1"][0, 0], e["s1"], atol=1e-15)
    np.testing.assert_allclose(f["s2"][0, 0], e["s2"], atol=1e-15)
    assert f["idx"][0, 0].tolist() == e["idx"]
    np.testing.assert_allclose(f["w"][0, 0], e["w"], atol=1e-14)
    np.testing.assert_allclose(f["y"], e["y"], atol=1e-13)
    # the product-key search reaches the same winners
    f2 = O.forward(inp, cfg, select="product")
    assert f2["idx"][0, 0].tolist() == e["idx"]
    b = O.backward(inp, cfg, f, np.array(g["dy"], dtype=np.float64))
    np.testing.assert_allclose(b["dw"][0, 0], e["dw"], atol=1e-13)
    np.testing.assert_allclose(b["dS"][0, 0], e["dS"], atol=1e-13)
    assert b["dV_rows"].tolist() == e["dV_rows"]
    np.testing.assert_allclose(b["dV_vals"], e["dV_vals"], atol=1e-14)
    ln2 = math.log(2.0)
    u = e["ln2_units"]
    np.testing.assert_allclose(b["g1"][0, 0], np.array(u["g1"]) * ln2, atol=1e-13)
    np.testing.assert_allclose(b["g2"][0, 0], np.array(u["g2"]) * ln2, atol=1e-13)
    for key in ("dq", "dsub", "dgamma", "dbeta", "dx", "dWq"):
        np.testing.assert_allclose(b[key], np.array(u[key]) * ln2, atol=1e-13, err_msg=key)


# --------------------------------------------------------------------------- selection
def _tie_heavy_scores(rng, C1, C2):
    # small integers: many equal sums and equal sub-scores
    return (rng.integers(-3, 4, C1).astype(np.float64),
            rng.integers(-3, 4, C2).astype(np.float64))


@pytest.mark.parametrize("C1,C2,k", [(8, 8, 3), (16, 9, 4), (32, 32, 8), (7, 13, 7), (64, 40, 32)])
def test_exactness_product_key_equals_brute_force(C1, C2, k):
    """The k best of s1[i]+s2[j] over all C1*C2 keys lie inside top-k(s1) x top-k(s2),
    and the product-key search returns them in the same order ("Large Memory Layers
    with Product Keys", abstract: exact search)."""
    rng = np.random.default_rng(C1 * 1000 + C2 * 10 + k)
    for trial in range(60):
        if trial % 2:
            s1, s2 = rng.standard_normal(C1), rng.standard_normal(C2)
        else:
            s1, s2 = _tie_heavy_scores(rng, C1, C2)
        bi, bj = O.brute_force_topk(s1, s2, k)
        pi, pj = O.product_key_topk(s1, s2, k)
        assert bi.tolist() == pi.tolist() and bj.tolist() == pj.tolist()


def test_brute_force_is_full_sort_prefix():
    """brute_force_topk equals the first k of a full sort of every key by the total
    order written out with Python's sort (different code, same definition)."""
    rng = np.random.default_rng(7)
    for trial in range(40):
        C1, C2, k = 40, 30, int(rng.integers(1, 31))
        s1, s2 = _tie_heavy_scores(rng, C1, C2) if trial % 2 else (
            rng.standard_normal(C1), rng.standard_normal(C2))
        keys = sorted(((-(s1[i] + s2[j]), -s1[i], -s2[j], i * C2 + j)
                       for i in range(C1) for j in range(C2)))
        want = [kk[3] for kk in keys[:k]]
        bi, bj = O.brute_force_topk(s1, s2, k)
        assert (bi * C2 + bj).tolist() == want


def test_k_equals_C_all_keys_are_candidates():
    """k = C1 = C2: the Cartesian candidate set is the whole keyspace, so the
    product-key path is brute force over all keys by construction."""
    rng = np.random.default_rng(3)
    s1, s2 = rng.standard_normal(6), rng.standard_normal(6)
    pi, pj = O.product_key_topk(s1, s2, 6)
    bi, bj = O.brute_force_topk(s1, s2, 6)
    assert (pi * 6 + pj).tolist() == (bi * 6 + bj).tolist()
    S = s1[:, None] + s2[None, :]
    assert np.allclose(np.sort(S.ravel())[::-1][:6], s1[pi] + s2[pj])


def test_k1_is_argmax_of_each_half():
    rng = np.random.default_rng(4)
    for _ in range(30):
        s1, s2 = rng.standard_normal(20), rng.standard_normal(11)
        i, j = O.brute_force_topk(s1, s2, 1)
        assert i[0] == int(np.argmax(s1)) and j[0] == int(np.argmax(s2))


def test_half_topk_order_and_ties():
    s = np.array([1.0, 3.0, 3.0, -1.0, 2.0, 3.0])
    i, v = O.half_topk(s, 4)
    assert i.tolist() == [1, 2, 5, 4] and v.tolist() == [3, 3, 3, 2]


# --------------------------------------------------------------------------- weights, bag
def test_softmax_sums_to_one_and_monotone():
    cfg = _cfg(score_scale=0.7)
    inp = make_inputs(cfg, seed=1, with_dy=False)
    f = O.forward(inp, cfg)
    np.testing.assert_allclose(f["w"].sum(-1), 1.0, atol=1e-12)
    # winners are listed best first, so the weights are non-increasing
    assert np.all(np.diff(f["w"], axis=-1) <= 1e-15)
    # ratio of weights equals exp of the score difference (closed form of softmax)
    r = f["w"][..., 0] / f["w"][..., 1]
    np.testing.assert_allclose(np.log(r), f["S"][..., 0] - f["S"][..., 1], rtol=1e-9, atol=1e-12)


def test_one_hot_value_table_reads_back_the_weights():
    """V = identity (d_v = K): y[t] is the vector of weights scattered to the chosen
    rows and summed over heads, so indices and weights are checked at once."""
    cfg = _cfg(C1=8, C2=6, d_v=48, h=2, k=5)
    inp = make_inputs(cfg, seed=2, with_dy=False)
    inp["values"] = np.eye(cfg.K)
    f = O.forward(inp, cfg)
    for t in range(cfg.N):
        want = np.zeros(cfg.K)
        for hh in range(cfg.h):
            for j in range(cfg.k):
                want[f["idx"][t, hh, j]] += f["w"][t, hh, j]
        np.testing.assert_allclose(f["y"][t], want, atol=1e-14)
        assert abs(f["y"][t].sum() - cfg.h) < 1e-12


def test_output_is_linear_in_values():
    cfg = _cfg()
    inp = make_inputs(cfg, seed=3, with_dy=False)
    rng = np.random.default_rng(0)
    V1, V2 = rng.standard_normal((cfg.K, cfg.d_v)), rng.standard_normal((cfg.K, cfg.d_v))
    ys = []
    for V in (V1, V2, 2.0 * V1 - 3.0 * V2):
        inp["values"] = V
        ys.append(O.forward(inp, cfg)["y"])
    np.testing.assert_allclose(ys[2], 2.0 * ys[0] - 3.0 * ys[1], atol=1e-12)


def test_permuting_subkeys_with_values_leaves_output_unchanged():
    """Relabel the sub-keys of each half (with the value rows moved to match): the
    layer's output must not change (no ties in continuous random data)."""
    cfg = _cfg(h=1)
    inp = make_inputs(cfg, seed=4, with_dy=False)
    y0 = O.forward(inp, cfg)["y"]
    rng = np.random.default_rng(9)
    p1, p2 = rng.permutation(cfg.C1), rng.permutation(cfg.C2)
    sub = inp["subkeys"].copy()
    sub[0, :cfg.C1] = inp["subkeys"][0, :cfg.C1][p1]
    sub[0, cfg.C1:] = inp["subkeys"][0, cfg.C1:][p2]
    # new sub-key a = old p1[a]; new row a*C2+b must hold old row p1[a]*C2+p2[b]
    V = inp["values"].reshape(cfg.C1, cfg.C2, -1)[p1][:, p2].reshape(cfg.K, -1)
    y1 = O.forward(dict(inp, subkeys=sub, values=V), cfg)["y"]
    np.testing.assert_allclose(y1, y0, atol=1e-13)


# --------------------------------------------------------------------------- query, scores
def test_query_network_matches_library_batch_norm():
    cfg = _cfg()
    inp = make_inputs(cfg, seed=5, with_dy=False, random_bn=True)
    q, _ = O.query_network(inp["x"], inp["Wq"], inp["bn"], cfg.bn_eps)
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    lin = torch.nn.functional.linear(t(inp["x"]), t(inp["Wq"]))
    bn = [t(r) for r in inp["bn"]]
    ref = torch.nn.functional.batch_norm(lin, bn[0], bn[1], bn[2], bn[3], training=False,
                                         eps=cfg.bn_eps)
    np.testing.assert_allclose(q, ref.numpy(), rtol=1e-13, atol=1e-13)


def test_subkey_scores_of_one_hot_queries_are_subkey_columns():
    cfg = _cfg(h=2, dk=8)
    rng = np.random.default_rng(6)
    sub = rng.standard_normal((cfg.h, cfg.C1 + cfg.C2, cfg.dk // 2))
    q = np.zeros((cfg.h * cfg.dk, cfg.h * cfg.dk))
    np.fill_diagonal(q, 1.0)          # token t has q = e_t
    s1, s2 = O.subkey_scores(q, sub, cfg.h, cfg.dk, cfg.C1)
    half = cfg.dk // 2
    for t in range(q.shape[0]):
        hh, r = divmod(t, cfg.dk)
        for h2 in range(cfg.h):
            if h2 != hh:
                assert not s1[t, h2].any() and not s2[t, h2].any()
        if r < half:
            np.testing.assert_array_equal(s1[t, hh], sub[hh, :cfg.C1, r])
            assert not s2[t, hh].any()
        else:
            np.testing.assert_array_equal(s2[t, hh], sub[hh, cfg.C1:, r - half])
            assert not s1[t, hh].any()


# --------------------------------------------------------------------------- backward
def _torch_loss_fixed_selection(inp, cfg, idx, dy, bn_train=False):
    """An independent forward in torch fp64 that touches only the selected keys (with
    ``bn_train`` the library's training-mode batch_norm normalises the query)."""
    t = lambda a: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)
    x, Wq, sub, V = t(inp["x"]), t(inp["Wq"]), t(inp["subkeys"]), t(inp["values"])
    mean, var = (torch.tensor(np.asarray(r, dtype=np.float64)) for r in inp["bn"][:2])
    gamma, beta = t(inp["bn"][2]), t(inp["bn"][3])
    if bn_train:
        q = torch.nn.functional.batch_norm(x @ Wq.T, None, None, gamma, beta, training=True,
                                           eps=cfg.bn_eps)
    else:
        q = (x @ Wq.T - mean) / torch.sqrt(var + cfg.bn_eps) * gamma + beta
    N = q.shape[0]
    qh = q.reshape(N, cfg.h, cfg.dk)
    half = cfg.dk // 2
    idx_t = torch.from_numpy(np.asarray(idx))
    ii, jj = idx_t // cfg.C2, idx_t % cfg.C2
    y = torch.zeros(N, V.shape[1], dtype=torch.float64)
    for hh in range(cfg.h):
        Ca = sub[hh, ii[:, hh]]                      # [N][k][half]
        Cb = sub[hh, cfg.C1 + jj[:, hh]]
        sa = (Ca * qh[:, hh, None, :half]).sum(-1)
        sb = (Cb * qh[:, hh, None, half:]).sum(-1)
        w = torch.softmax(cfg.score_scale * (sa + sb), dim=-1)
        y = y + (w[..., None] * V[idx_t[:, hh]]).sum(1)
    L = (torch.from_numpy(np.asarray(dy, dtype=np.float64)) * y).sum()
    L.backward()
    return dict(dx=x.grad.numpy(), dWq=Wq.grad.numpy(), dsub=sub.grad.numpy(),
                dV=V.grad.numpy(), dgamma=gamma.grad.numpy(), dbeta=beta.grad.numpy())


@pytest.mark.parametrize("scale,bn_train", [(1.0, False), (0.37, False), (0.6, True)])
def test_backward_matches_autograd_of_independent_forward(scale, bn_train):
    cfg = _cfg(score_scale=scale, N=10, h=2)
    inp = make_inputs(cfg, seed=8, random_bn=True)
    f = O.forward(inp, cfg, bn_train=bn_train)
    b = O.backward(inp, cfg, f, inp["dy"])
    ref = _torch_loss_fixed_selection(inp, cfg, f["idx"], inp["dy"], bn_train=bn_train)
    for key in ("dx", "dWq", "dsub", "dgamma", "dbeta"):
        np.testing.assert_allclose(b[key], ref[key], rtol=1e-10, atol=1e-12, err_msg=key)
    dV = np.zeros_like(ref["dV"])
    dV[b["dV_rows"]] = b["dV_vals"]
    np.testing.assert_allclose(dV, ref["dV"], rtol=1e-10, atol=1e-12)


def test_training_batch_norm_matches_the_library():
    """Training-mode BatchNorm: q and the running-statistics update equal the library's
    batch_norm(training=True) (biased variance to normalise, unbiased for the running
    variance); each column of q-hat has mean 0 and mean square var / (var + eps)."""
    cfg = _cfg(N=24)
    inp = make_inputs(cfg, seed=30, with_dy=False, random_bn=True)
    q, qhat, mu, var = O.query_network_train(inp["x"], inp["Wq"], inp["bn"], cfg.bn_eps)
    t = lambda a: torch.from_numpy(np.array(a, dtype=np.float64))
    rm, rv = t(inp["bn"][0]), t(inp["bn"][1])
    ref = torch.nn.functional.batch_norm(t(inp["x"]) @ t(inp["Wq"]).T, rm, rv, t(inp["bn"][2]),
                                         t(inp["bn"][3]), training=True, momentum=0.1,
                                         eps=cfg.bn_eps)
    np.testing.assert_allclose(q, ref.numpy(), rtol=1e-12, atol=1e-12)
    upd = O.running_stats_update(inp["bn"], mu, var, cfg.N, 0.1)
    np.testing.assert_allclose(upd[0], rm.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(upd[1], rv.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(upd[2:], np.asarray(inp["bn"][2:], dtype=np.float64))
    np.testing.assert_allclose(qhat.mean(0), 0.0, atol=1e-12)
    np.testing.assert_allclose((qhat ** 2).mean(0), var / (var + cfg.bn_eps), rtol=1e-12)


def test_training_batch_norm_dx_by_finite_differences():
    """Training mode couples every token through the batch statistics: central
    differences of the loss in x (any token) match the analytic dx."""
    cfg = _cfg(N=8, h=2)
    inp = make_inputs(cfg, seed=31, random_bn=True)
    inp = {k: np.asarray(v, dtype=np.float64) for k, v in inp.items()}
    f0 = O.forward(inp, cfg, bn_train=True)
    b = O.backward(inp, cfg, f0, inp["dy"])
    rng = np.random.default_rng(32)
    tested = 0
    for _ in range(30):
        ix = tuple(int(rng.integers(0, s)) for s in inp["x"].shape)
        vals, ok = [], True
        for sgn in (1, -1):
            p = {k: v.copy() for k, v in inp.items()}
            p["x"][ix] += sgn * 1e-6
            f = O.forward(p, cfg, bn_train=True)
            ok &= np.array_equal(f["idx"], f0["idx"])
            vals.append((inp["dy"] * f["y"]).sum())
        if ok:
            np.testing.assert_allclose((vals[0] - vals[1]) / 2e-6, b["dx"][ix], rtol=1e-5,
                                       atol=1e-8)
            tested += 1
    assert tested >= 20


def test_value_gradient_row_sum_closed_form():
    """sum_r dV[r] = sum_t sum_h (sum_j w) dy[t] = h * sum_t dy[t]."""
    cfg = _cfg(h=3, N=12)
    inp = make_inputs(cfg, seed=10)
    f = O.forward(inp, cfg)
    b = O.backward(inp, cfg, f, inp["dy"])
    np.testing.assert_allclose(b["dV_vals"].sum(0), cfg.h * inp["dy"].astype(np.float64).sum(0),
                               rtol=1e-12, atol=1e-12)


def test_backward_central_finite_differences_tiny_config():
    """Central differences in fp64 on the tiny workload's shapes (sampled entries),
    skipping perturbations that change the selected keys."""
    cfg = TINY_FP32.with_(N=16)
    inp = make_inputs(cfg, seed=0, random_bn=True)
    inp = {k: np.asarray(v, dtype=np.float64) for k, v in inp.items()}
    dy = inp["dy"]
    L0, f0 = O.loss(inp, cfg, dy)
    b = O.backward(inp, cfg, f0, dy)
    dV = {int(r): v for r, v in zip(b["dV_rows"], b["dV_vals"])}
    rng = np.random.default_rng(11)
    eps = 1e-6
    checks = []
    for name, shape in (("x", inp["x"].shape), ("Wq", inp["Wq"].shape),
                        ("subkeys", inp["subkeys"].shape), ("bn", inp["bn"].shape)):
        for _ in range(25):
            checks.append((name, tuple(int(rng.integers(0, s)) for s in shape)))
    for r in list(dV)[:10]:
        checks.append(("values", (r, int(rng.integers(0, cfg.d_v)))))
    checks.append(("values", (int(np.setdiff1d(np.arange(cfg.K), b["dV_rows"])[0]), 0)))
    tested = 0
    for name, ix in checks:
        if name == "bn" and ix[0] < 2:
            ix = (ix[0] + 2,) + ix[1:]           # running stats are not parameters
        vals = []
        ok = True
        for sgn in (1, -1):
            p = {k: v.copy() for k, v in inp.items()}
            p[name][ix] += sgn * eps
            L, f = O.loss(p, cfg, dy)
            ok &= np.array_equal(f["idx"], f0["idx"])
            vals.append(L)
        if not ok:
            continue
        fd = (vals[0] - vals[1]) / (2 * eps)
        if name == "x":
            an = b["dx"][ix]
        elif name == "Wq":
            an = b["dWq"][ix]
        elif name == "subkeys":
            an = b["dsub"][ix]
        elif name == "bn":
            an = (b["dgamma"] if ix[0] == 2 else b["dbeta"])[ix[1]]
        else:
            an = dV.get(ix[0], np.zeros(cfg.d_v))[ix[1]]
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, ix, fd, an)
        tested += 1
    assert tested >= 90


# --------------------------------------------------------------------------- fast weights
def _fw_cfg(**kw):
    base = dict(name="fw", N=48, d_in=6, h=1, dk=8, C1=12, C2=10, k=3, d_v=6, dtype="f32",
                clustered=4)
    base.update(kw)
    return PKMConfig(**base)


def test_fastweight_zero_rate_is_plain_forward():
    cfg = _fw_cfg()
    inp = make_inputs(cfg, seed=1)
    tg = np.random.default_rng(0).standard_normal((cfg.N, cfg.d_v))
    ys, rows, vals = O.fastweight_chunks(inp, cfg, 16, 0.0, targets=tg)
    np.testing.assert_allclose(ys, O.forward(inp, cfg)["y"], atol=1e-13)
    np.testing.assert_array_equal(vals, inp["values"][rows])


def test_fastweight_one_chunk_is_a_descent_step():
    """One chunk: the write is -lr times the gradient of the chunk's loss, whose
    gradient for row r is sum over selections of r of w * (y - target) (closed form,
    written out here per selection); only selected rows change; and for a small rate
    the loss at the same selection drops by lr * |grad|^2 to first order."""
    cfg = _fw_cfg(h=2)
    inp = make_inputs(cfg, seed=2)
    tg = np.random.default_rng(1).standard_normal((cfg.N, cfg.d_v))
    lr = 1e-4
    _, rows, vals = O.fastweight_chunks(inp, cfg, cfg.N, lr, targets=tg)
    f = O.forward(inp, cfg)
    grad = {}
    for t in range(cfg.N):
        for hh in range(cfg.h):
            for j in range(cfg.k):
                r = int(f["idx"][t, hh, j])
                grad[r] = grad.get(r, 0.0) + f["w"][t, hh, j] * (f["y"][t] - tg[t])
    assert sorted(grad) == rows.tolist()
    for r, v in zip(rows, vals):
        np.testing.assert_allclose(v, inp["values"][r] - lr * grad[int(r)], atol=1e-13)
    V1 = np.array(inp["values"], dtype=np.float64)
    V1[rows] = vals
    loss0 = 0.5 * ((f["y"] - tg) ** 2).sum()
    loss1 = 0.5 * ((O.bag(f["w"], f["idx"], V1) - tg) ** 2).sum()
    g2 = sum((g ** 2).sum() for g in grad.values())
    np.testing.assert_allclose(loss0 - loss1, lr * g2, rtol=1e-3)


def test_fastweight_later_chunks_read_earlier_writes():
    """Two chunks: the second chunk's reads differ from reading the untouched table
    exactly on tokens that select a row the first chunk wrote (selection does not
    depend on the value table)."""
    cfg = _fw_cfg(C1=16, C2=16, k=2, clustered=0)
    inp = make_inputs(cfg, seed=3)
    tg = np.random.default_rng(2).standard_normal((cfg.N, cfg.d_v))
    ys, rows, _ = O.fastweight_chunks(inp, cfg, 24, 0.5, targets=tg)
    f0 = O.forward(inp, cfg)
    first = set(np.unique(f0["idx"][:24]).tolist())
    np.testing.assert_allclose(ys[:24], f0["y"][:24], atol=1e-14)
    n_touch = 0
    for t in range(24, cfg.N):
        touches = bool(set(f0["idx"][t].ravel().tolist()) & first)
        n_touch += touches
        assert np.allclose(ys[t], f0["y"][t], atol=1e-14) == (not touches), t
    assert 0 < n_touch < cfg.N - 24


def test_fastweight_rate_one_on_a_lone_selection_reaches_the_target():
    """k = 1, one token, w = 1: the gradient of 1/2 ||V[r] - target||^2 is V[r] -
    target, so a step of rate 1 writes the target into the row exactly."""
    cfg = _fw_cfg(N=1, k=1)
    inp = make_inputs(cfg, seed=4)
    tg = np.random.default_rng(3).standard_normal((1, cfg.d_v))
    _, rows, vals = O.fastweight_chunks(inp, cfg, 1, 1.0, targets=tg)
    assert rows.size == 1
    np.testing.assert_allclose(vals[0], tg[0], atol=1e-14)


def test_fastweight_lookahead_targets_are_the_next_input():
    """Lookahead equals explicit targets x[t + 1] with the last token's target set to
    its own read (zero residual)."""
    cfg = _fw_cfg(d_in=6, d_v=6)
    inp = make_inputs(cfg, seed=5)
    ys_a, rows_a, vals_a = O.fastweight_chunks(inp, cfg, 16, 0.3, lookahead=True)
    tg = np.zeros((cfg.N, cfg.d_v))
    tg[:-1] = np.asarray(inp["x"], dtype=np.float64)[1:]
    # the last token's target: its read, which no earlier write of its own chunk changes
    tg[-1] = ys_a[-1]
    ys_b, rows_b, vals_b = O.fastweight_chunks(inp, cfg, 16, 0.3, targets=tg)
    np.testing.assert_allclose(ys_a, ys_b, atol=1e-13)
    assert rows_a.tolist() == rows_b.tolist()
    np.testing.assert_allclose(vals_a, vals_b, atol=1e-13)


# --------------------------------------------------------------------------- bf16 q scoring
def test_round_bf16_hand_cases_and_library():
    """Ties go to the even neighbour; everything else to the nearest bf16; agrees with
    the library's fp32 -> bfloat16 conversion on random values."""
    e = 2.0 ** -8
    cases = [(1.0, 1.0), (1 + e, 1.0), (1 + 3 * e, 1 + 4 * e), (1 + e + 2.0 ** -20, 1 + 2 * e),
             (-(1 + e), -1.0), (3.0, 3.0), (0.0, 0.0), (2.0 ** -130, 2.0 ** -130)]
    for a, want in cases:
        assert O.round_bf16(np.array([a]))[0] == want, (a, want)
    r = np.random.default_rng(0).standard_normal(10000) * 10.0 ** np.random.default_rng(1).integers(-6, 6, 10000)
    lib = torch.from_numpy(r.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(r), lib)


def _bf16_exact_q_case():
    """Wq = I, BN with var + eps = 1: q = x exactly, and x is bf16."""
    eps = 2.0 ** -10
    cfg = _cfg(d_in=16, h=2, dk=8, dtype="bf16", bn_eps=eps)
    inp = make_inputs(cfg, seed=11)
    inp["Wq"] = np.eye(16, dtype=np.float32)
    inp["bn"] = np.stack([np.zeros(16), np.full(16, 1 - eps), np.ones(16), np.zeros(16)])
    return cfg, inp


def test_bf16_q_variant_equals_plain_when_q_is_bf16():
    cfg, inp = _bf16_exact_q_case()
    f0, f1 = O.forward(inp, cfg), O.forward(inp, cfg, q_bf16=True)
    np.testing.assert_array_equal(f1["q_scores"], f0["q"])
    assert (f0["idx"] == f1["idx"]).all()
    np.testing.assert_array_equal(f0["y"], f1["y"])
    b0, b1 = O.backward(inp, cfg, f0, inp["dy"]), O.backward(inp, cfg, f1, inp["dy"])
    for key in ("dsub", "dx", "dWq", "dgamma", "dbeta", "dV_vals"):
        np.testing.assert_array_equal(b0[key], b1[key], err_msg=key)


def test_bf16_q_scores_within_the_rounding_bound():
    """|s_b - s| <= sum_d 2^-9 |q_d| |C_d| (half an ulp of bf16 per query coordinate),
    and the bound is not vacuous (the scores do move)."""
    cfg = _cfg(h=2, dk=16, C1=20, C2=12)
    inp = make_inputs(cfg, seed=12, random_bn=True)
    f0, f1 = O.forward(inp, cfg), O.forward(inp, cfg, q_bf16=True)
    sub = np.asarray(inp["subkeys"], dtype=np.float64)
    q1, q2 = O.split_halves(np.abs(f0["q"]), cfg.h, cfg.dk)
    b1 = 2.0 ** -9 * np.einsum("thd,hid->thi", q1, np.abs(sub[:, :cfg.C1]))
    b2 = 2.0 ** -9 * np.einsum("thd,hid->thi", q2, np.abs(sub[:, cfg.C1:]))
    assert np.all(np.abs(f1["s1"] - f0["s1"]) <= b1 * (1 + 1e-12))
    assert np.all(np.abs(f1["s2"] - f0["s2"]) <= b2 * (1 + 1e-12))
    assert np.abs(f1["s1"] - f0["s1"]).max() > 0


def test_bf16_q_subkey_gradient_by_finite_differences():
    """The sub-key gradient after a bf16-q forward is the derivative of the loss in the
    sub-keys with the rounded q (which does not depend on them): central differences."""
    cfg = _cfg(h=2, dk=8, C1=10, C2=9, k=3)
    inp = make_inputs(cfg, seed=13, random_bn=True)
    f = O.forward(inp, cfg, q_bf16=True)
    g = O.backward(inp, cfg, f, inp["dy"])["dsub"]
    sub0 = np.asarray(inp["subkeys"], dtype=np.float64)
    rng = np.random.default_rng(5)
    for _ in range(12):
        i = tuple(int(rng.integers(0, n)) for n in sub0.shape)
        h = 1e-6
        vals = []
        for sgn in (1, -1):
            s = sub0.copy()
            s[i] += sgn * h
            fs = O.forward(dict(inp, subkeys=s), cfg, q_bf16=True)
            assert (fs["idx"] == f["idx"]).all()
            vals.append((inp["dy"] * fs["y"]).sum())
        np.testing.assert_allclose((vals[0] - vals[1]) / (2 * h), g[i], rtol=1e-5, atol=1e-8)


# --------------------------------------------------------------------------- training pieces
def test_hit_counts_totals_and_argmax_case():
    """Every token contributes h*k slot hits and 2k sub-key hits per head; with k = 1 the
    sub-key hits are the per-half argmax counts."""
    cfg = _cfg(N=40, h=2, k=4)
    inp = make_inputs(cfg, seed=21)
    f = O.forward(inp, cfg)
    slot, sub = O.hit_counts(f, cfg)
    assert slot.sum() == cfg.N * cfg.h * cfg.k and slot.shape == (cfg.K,)
    assert (sub.sum(1) == 2 * cfg.N * cfg.k).all()
    assert (sub[:, :cfg.C1].sum(1) == cfg.N * cfg.k).all()
    # rows never selected have zero hits; the selected ones at least one
    assert (slot[np.unique(f["idx"])] > 0).all() and slot.sum() == f["idx"].size
    cfg1 = _cfg(N=40, h=2, k=1)
    f1 = O.forward(make_inputs(cfg1, seed=22), cfg1)
    _, sub1 = O.hit_counts(f1, cfg1)
    for hh in range(cfg1.h):
        a1 = np.bincount(np.argmax(f1["s1"][:, hh], axis=1), minlength=cfg1.C1)
        a2 = np.bincount(np.argmax(f1["s2"][:, hh], axis=1), minlength=cfg1.C2)
        np.testing.assert_array_equal(sub1[hh], np.concatenate([a1, a2]))


def test_sparse_adam_matches_the_library_optimisers():
    """Lazy Adam against two independent implementations: torch.optim.SparseAdam on
    changing row sets (it adds eps to sqrt(v) before the bias correction, so eps is made
    negligible there), and torch.optim.Adam when every row is touched at every step
    (lazy and dense Adam then coincide; this pins where eps enters)."""
    rng = np.random.default_rng(23)
    K, d = 12, 5
    V0 = rng.standard_normal((K, d))
    lr, b1, b2 = 0.05, 0.9, 0.99
    p = torch.nn.Parameter(torch.from_numpy(V0.copy()))
    opt = torch.optim.SparseAdam([p], lr=lr, betas=(b1, b2), eps=1e-30)
    V, M, S = V0.copy(), np.zeros((K, d)), np.zeros((K, d))
    for step, rows in enumerate(([1, 4, 7], [4, 5], [0, 1, 4, 11]), start=1):
        rows = np.array(rows)
        g = rng.standard_normal((rows.size, d))
        V, M, S = O.sparse_adam(V, M, S, rows, g, lr, b1, b2, 1e-30, step)
        p.grad = torch.sparse_coo_tensor(torch.from_numpy(rows)[None], torch.from_numpy(g), (K, d))
        opt.step()
    np.testing.assert_allclose(V, p.detach().numpy(), rtol=1e-12, atol=1e-12)

    eps = 1e-3
    p = torch.nn.Parameter(torch.from_numpy(V0.copy()))
    opt = torch.optim.Adam([p], lr=lr, betas=(b1, b2), eps=eps)
    V, M, S = V0.copy(), np.zeros((K, d)), np.zeros((K, d))
    for step in range(1, 4):
        g = rng.standard_normal((K, d)) * 1e-3
        V, M, S = O.sparse_adam(V, M, S, np.arange(K), g, lr, b1, b2, eps, step)
        p.grad = torch.from_numpy(g.copy())
        opt.step()
    np.testing.assert_allclose(V, p.detach().numpy(), rtol=1e-12, atol=1e-12)


def test_sparse_adam_first_step_closed_form_and_untouched_rows():
    """From zero state the first step moves a row by lr * g / (|g| + eps) elementwise;
    untouched rows and their state stay as they were."""
    rng = np.random.default_rng(24)
    V0, M0, S0 = rng.standard_normal((6, 3)), rng.standard_normal((6, 3)), rng.random((6, 3))
    M0[2] = S0[2] = 0.0
    g = rng.standard_normal((1, 3))
    V, M, S = O.sparse_adam(V0, M0, S0, np.array([2]), g, 0.1, 0.9, 0.999, 1e-8, 1)
    np.testing.assert_allclose(V[2], V0[2] - 0.1 * g[0] / (np.abs(g[0]) + 1e-8), rtol=1e-12)
    keep = np.arange(6) != 2
    np.testing.assert_array_equal(V[keep], V0[keep])
    np.testing.assert_array_equal(M[keep], M0[keep])
    np.testing.assert_array_equal(S[keep], S0[keep])


# --------------------------------------------------------------------------- all k^2 variant
def test_all_k2_with_full_halves_is_softmax_attention_over_every_key():
    """k = C1 = C2: the k x k candidates are every product key, so the variant is a dense
    softmax over all C1*C2 keys: y = softmax(scale * (s1[i] + s2[j])) @ V, written here
    with plain matrix operations."""
    cfg = _cfg(C1=6, C2=6, k=6, h=2, N=7, score_scale=0.8)
    inp = make_inputs(cfg, seed=40)
    f = O.forward(inp, cfg, all_k2=True)
    assert f["idx"].shape == (cfg.N, cfg.h, 36)
    V = np.asarray(inp["values"], dtype=np.float64)
    want = np.zeros((cfg.N, cfg.d_v))
    for hh in range(cfg.h):
        S = cfg.score_scale * (f["s1"][:, hh, :, None] + f["s2"][:, hh, None, :]).reshape(cfg.N, -1)
        P = np.exp(S - S.max(1, keepdims=True))
        want += (P / P.sum(1, keepdims=True)) @ V
    np.testing.assert_allclose(f["y"], want, rtol=1e-12, atol=1e-13)


def test_all_k2_candidates_and_gradient():
    """The variant keeps exactly top-k(s1) x top-k(s2) (a-major), its weights sum to one,
    and its backward matches central differences in the sub-keys and x (the candidate
    set held fixed)."""
    cfg = _cfg(C1=9, C2=7, k=3, h=2, N=5)
    inp = make_inputs(cfg, seed=41, random_bn=True)
    inp = {k_: np.asarray(v, dtype=np.float64) for k_, v in inp.items()}
    f = O.forward(inp, cfg, all_k2=True)
    for t in range(cfg.N):
        for hh in range(cfg.h):
            a, b = O.half_topk(f["s1"][t, hh], 3)[0], O.half_topk(f["s2"][t, hh], 3)[0]
            want = [int(i) * cfg.C2 + int(j) for i in a for j in b]
            assert f["idx"][t, hh].tolist() == want
    np.testing.assert_allclose(f["w"].sum(-1), 1.0, atol=1e-12)
    b = O.backward(inp, cfg, f, inp["dy"])
    rng = np.random.default_rng(42)
    tested = 0
    for name, key in (("subkeys", "dsub"), ("x", "dx")):
        for _ in range(12):
            ix = tuple(int(rng.integers(0, s)) for s in inp[name].shape)
            vals, ok = [], True
            for sgn in (1, -1):
                p = {k_: v.copy() for k_, v in inp.items()}
                p[name][ix] += sgn * 1e-6
                fs = O.forward(p, cfg, all_k2=True)
                ok &= np.array_equal(fs["idx"], f["idx"])
                vals.append((inp["dy"] * fs["y"]).sum())
            if ok:
                np.testing.assert_allclose((vals[0] - vals[1]) / 2e-6, b[key][ix], rtol=1e-5,
                                           atol=1e-8)
                tested += 1
    assert tested >= 16


# --------------------------------------------------------------------------- IDW scores
def test_idw_scores_closed_form():
    """With q at the origin and sub-keys at known distances, s = -log(distance); the
    softmax weights are proportional to (d1 d2)^(-scale)."""
    cfg = _cfg(N=1, h=1, dk=4, C1=3, C2=2, k=2, score_scale=1.5)
    sub = np.zeros((1, 5, 2))
    sub[0, 0] = [1.0, 0.0]     # C: distances 1, 2, 4 from the origin
    sub[0, 1] = [0.0, 2.0]
    sub[0, 2] = [4.0, 0.0]
    sub[0, 3] = [3.0, 4.0]     # C': distances 5, 0.5
    sub[0, 4] = [0.0, -0.5]
    q = np.zeros((1, 4))
    s1, s2 = O.subkey_scores_idw(q, sub, 1, 4, 3)
    np.testing.assert_allclose(s1[0, 0], -np.log([1.0, 2.0, 4.0]), atol=1e-11)
    np.testing.assert_allclose(s2[0, 0], -np.log([5.0, 0.5]), atol=1e-11)
    # the layer with these sub-keys: x = 0 and BN beta = 0 give q = 0
    inp = dict(x=np.zeros((1, 16)), Wq=np.zeros((4, 16)),
               bn=np.stack([np.zeros(4), np.ones(4), np.ones(4), np.zeros(4)]), subkeys=sub,
               values=np.eye(6))
    cfg = cfg.with_(d_in=16, d_v=6)
    f = O.forward(inp, cfg, idw=True)
    # the two closest products: (d1, d2) = (1, 0.5) and (2, 0.5), rows 0*2+1 and 1*2+1
    assert f["idx"][0, 0].tolist() == [1, 3]
    wr = (1.0 * 0.5) ** -1.5, (2.0 * 0.5) ** -1.5
    np.testing.assert_allclose(f["w"][0, 0], np.array(wr) / sum(wr), rtol=1e-10)


def test_idw_gradient_by_finite_differences():
    """The inverse-distance backward against central differences in x, the sub-keys and
    the values (selection held fixed)."""
    cfg = _cfg(N=6, h=2, dk=8, C1=9, C2=7, k=3)
    inp = make_inputs(cfg, seed=50, random_bn=True)
    inp = {k_: np.asarray(v, dtype=np.float64) for k_, v in inp.items()}
    f = O.forward(inp, cfg, idw=True)
    b = O.backward(inp, cfg, f, inp["dy"])
    rng = np.random.default_rng(51)
    tested = 0
    for name, key in (("subkeys", "dsub"), ("x", "dx"), ("Wq", "dWq")):
        for _ in range(10):
            ix = tuple(int(rng.integers(0, s)) for s in inp[name].shape)
            vals, ok = [], True
            for sgn in (1, -1):
                p = {k_: v.copy() for k_, v in inp.items()}
                p[name][ix] += sgn * 1e-6
                fs = O.forward(p, cfg, idw=True)
                ok &= np.array_equal(fs["idx"], f["idx"])
                vals.append((inp["dy"] * fs["y"]).sum())
            if ok:
                np.testing.assert_allclose((vals[0] - vals[1]) / 2e-6, b[key][ix], rtol=1e-5,
                                           atol=1e-8)
                tested += 1
    assert tested >= 24


def test_idw_product_key_search_is_exact():
    """The scores are still a sum over the two halves, so the product-key search reaches
    the brute-force winners."""
    cfg = _cfg(N=12, h=2, dk=8, C1=16, C2=12, k=5)
    inp = make_inputs(cfg, seed=52)
    fb = O.forward(inp, cfg, idw=True)
    fp = O.forward(inp, cfg, idw=True, select="product")
    np.testing.assert_array_equal(fb["idx"], fp["idx"])
