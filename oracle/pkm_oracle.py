"""CPU oracle of the product-key memory (PKM) layer, forward and backward, in fp64.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module.  The CUDA library never calls it, and it
shares no code, header, table or helper with the CUDA library.

What it computes (sources: "Large Memory Layers with Product Keys", method-details
list and abstract; "Meta AI 可扩展内存层" sections 3.2, 4.3, 4.5, 5.2, 5.3):

  1. query network      q = gamma * (x Wq^T - mean) / sqrt(var + eps) + beta
                        (Linear followed by BatchNorm with running statistics)
  2. split per head     q1 = q[h*dk : h*dk + dk/2], q2 = q[h*dk + dk/2 : (h+1)*dk]
  3. sub-key scores     s1[i] = q1 . C[h][i],  s2[j] = q2 . C'[h][j]
  4. key selection      the k best product keys (i, j) by s1[i] + s2[j] over ALL
                        C1*C2 keys (brute force: the exact nearest-neighbour result
                        the product keys are built to reach)
  5. weights            w = softmax(score_scale * (s1[i] + s2[j])) over the k winners
  6. output             y[t] = sum_h sum_winners w * V[i*C2 + j]

Readings taken where the pages are silent (each is listed in the design notes):
  * total order of keys: (s1+s2 desc, s1 desc, s2 desc, flat index asc); per
    half: (score desc, index asc).  With this order the product-key search returns
    exactly the brute-force set even with rounding ties.
  * heads each own their sub-key sets, share the value table, and their outputs
    are summed; the softmax is per head.
  * the temperature is a positive ``score_scale`` applied to the softmax only;
    selection uses the unscaled sums (a positive scale keeps the order).
  * the backward holds the selected set fixed (top-k is piecewise constant).

Every function here is pinned by a CPU test against something other than itself:
brute force vs the product-key search (exactness), a hand-derived worked example
(tests/golden), one-hot value tables, permutation and linearity invariants, the
library batch_norm, autograd of an independent forward, and central finite
differences in fp64.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------- 1
def query_network(x, Wq, bn, eps):
    """q = gamma * (x Wq^T - mean) / sqrt(var + eps) + beta, fp64.

    x [N][d_in], Wq [h*dk][d_in] (Linear weight, out x in), bn [4][h*dk] =
    (running mean, running var, gamma, beta).  BatchNorm in eval mode on the
    query ("Large Memory Layers with Product Keys", key results, BatchNorm remark).
    """
    x = np.asarray(x, dtype=np.float64)
    Wq = np.asarray(Wq, dtype=np.float64)
    mean, var, gamma, beta = (np.asarray(r, dtype=np.float64) for r in bn)
    pre = x @ Wq.T
    qhat = (pre - mean) / np.sqrt(var + eps)
    return gamma * qhat + beta, qhat


def query_network_train(x, Wq, bn, eps):
    """Training-mode BatchNorm on the query: the statistics are the batch's own, over the
    N tokens of the call (per column of x Wq^T: mean mu and the biased variance var);
    q-hat = (x Wq^T - mu) / sqrt(var + eps), q = gamma * q-hat + beta.  Returns
    (q, q-hat, mu, var).  The BatchNorm on the query is the first page's remark on
    query normalisation ("Large Memory Layers with Product Keys", key results); training
    mode is the plain reading of that layer when the batch trains it."""
    x = np.asarray(x, dtype=np.float64)
    Wq = np.asarray(Wq, dtype=np.float64)
    gamma, beta = (np.asarray(r, dtype=np.float64) for r in bn[2:4])
    pre = x @ Wq.T
    mu = pre.mean(axis=0)
    var = ((pre - mu) ** 2).mean(axis=0)
    qhat = (pre - mu) / np.sqrt(var + eps)
    return gamma * qhat + beta, qhat, mu, var


def running_stats_update(bn, mu, var, n, momentum):
    """Running statistics after a training batch of n tokens: mean <- (1 - m) mean + m mu,
    var <- (1 - m) var + m * var_batch * n / (n - 1) (the unbiased batch variance)."""
    out = np.array(bn, dtype=np.float64, copy=True)
    out[0] = (1.0 - momentum) * out[0] + momentum * mu
    out[1] = (1.0 - momentum) * out[1] + momentum * var * n / (n - 1)
    return out


def round_bf16(a):
    """Round to the nearest bfloat16 (ties to even) through fp32, returned as fp64: the
    fp32 bit pattern u becomes (u + 0x7FFF + ((u >> 16) & 1)) with the low 16 bits
    cleared (finite inputs).  Used by the single-pass scoring variant, whose scores
    take q rounded to bf16."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- 2, 3
def split_halves(q, h, dk):
    """q [N][h*dk] -> (q1, q2), each [N][h][dk/2]."""
    q = q.reshape(q.shape[0], h, dk)
    return q[:, :, : dk // 2], q[:, :, dk // 2:]


def subkey_scores(q, subkeys, h, dk, C1):
    """s1[t][h][i] = q1[t][h] . C[h][i];  s2[t][h][j] = q2[t][h] . C'[h][j]  (fp64)."""
    sub = np.asarray(subkeys, dtype=np.float64)
    q1, q2 = split_halves(q, h, dk)
    s1 = np.einsum("thd,hid->thi", q1, sub[:, :C1, :])
    s2 = np.einsum("thd,hjd->thj", q2, sub[:, C1:, :])
    return s1, s2


IDW_EPS = 1e-12


def subkey_scores_idw(q, subkeys, h, dk, C1):
    """Inverse-distance scores ("Fast-weight Product Key Memory", section 2.2, practical
    techniques: the negative log of the Euclidean distance replaces the dot product):
    s1[t][h][i] = -1/2 log(||q1[t][h] - C[h][i]||^2 + IDW_EPS), likewise s2 with C'.
    IDW_EPS only keeps a zero distance finite.  The softmax of scale * (s1 + s2) then
    weighs a key by (d1 d2)^(-scale): inverse distance weighting.  fp64."""
    sub = np.asarray(subkeys, dtype=np.float64)
    q1, q2 = split_halves(q, h, dk)
    d1 = ((q1[:, :, None, :] - sub[None, :, :C1, :]) ** 2).sum(-1)
    d2 = ((q2[:, :, None, :] - sub[None, :, C1:, :]) ** 2).sum(-1)
    return -0.5 * np.log(d1 + IDW_EPS), -0.5 * np.log(d2 + IDW_EPS)


# ----------------------------------------------------------------------------- 4
def half_topk(s, k):
    """Top-k of one half's scores s [C] by (score desc, index asc) -> (index, score)."""
    order = np.lexsort((np.arange(s.shape[0]), -s))[:k]
    return order, s[order]


def _order_candidates(S, a, b, flat):
    """Indices sorting candidates by (S desc, a desc, b desc, flat asc)."""
    return np.lexsort((flat, -b, -a, -S))


def brute_force_topk(s1, s2, k):
    """The k best keys over ALL C1*C2 product keys of one (token, head).

    The sum s1[i] + s2[j] is formed for every key; the first k under the total
    order (sum desc, s1 desc, s2 desc, flat asc) win.  Returns (i, j) of the
    winners, best first.

    Only keys whose sum reaches the k-th largest sum can be among the first k under
    an order whose first key is the sum, so the order is taken over those (all of
    them, ties included).
    """
    C1, C2 = s1.shape[0], s2.shape[0]
    S = (s1[:, None] + s2[None, :]).reshape(-1)
    flat = np.arange(C1 * C2)
    if S.shape[0] > 4 * k:
        kth = np.partition(S, S.shape[0] - k)[S.shape[0] - k]
        keep = np.nonzero(S >= kth)[0]
    else:
        keep = flat
    ii, jj = keep // C2, keep % C2
    order = _order_candidates(S[keep], s1[ii], s2[jj], keep)[:k]
    sel = keep[order]
    return sel // C2, sel % C2


def product_key_topk(s1, s2, k):
    """The product-key search for one (token, head): the top-k of each half, then the
    best k of the k x k Cartesian candidates by the same total order as
    ``brute_force_topk`` ("Large Memory Layers with Product Keys", method details;
    "Meta AI 可扩展内存层" section 4.3).  Returns (i, j), best first."""
    C2 = s2.shape[0]
    ia, va = half_topk(s1, k)
    jb, vb = half_topk(s2, k)
    S = (va[:, None] + vb[None, :]).reshape(-1)
    A = np.repeat(va, k)
    B = np.tile(vb, k)
    I = np.repeat(ia, k)
    J = np.tile(jb, k)
    order = _order_candidates(S, A, B, I * C2 + J)[:k]
    return I[order], J[order]


# ----------------------------------------------------------------------------- 5
def softmax(S):
    """Softmax over the last axis, fp64."""
    m = S.max(axis=-1, keepdims=True)
    e = np.exp(S - m)
    return e / e.sum(axis=-1, keepdims=True)


# ----------------------------------------------------------------------------- 1..6
def forward(inp, cfg, select="brute", q_bf16=False, bn_train=False, all_k2=False, idw=False):
    """The layer forward for every token of ``inp['x']``.

    ``idw``: inverse-distance sub-key scores (``subkey_scores_idw``) instead of dot
    products; selection and softmax are unchanged.

    ``all_k2``: the variant of the code snippet in "Meta AI 可扩展内存层" section 10 --
    no second top-k: every one of the k x k candidates top-k(s1) x top-k(s2) is kept
    (a-major: candidate a*k + b pairs the a-th key of the first half with the b-th of the
    second) and the softmax runs over all k^2 of them; idx, S, w are then [N][h][k*k].

    ``bn_train``: BatchNorm with the batch's statistics (``query_network_train``); the
    dict then also holds them as ``bn_batch`` = (mu, var).

    ``q_bf16``: the single-pass scoring variant -- the sub-key scores (and through them
    the selection and the weights) take q rounded to bf16 (``round_bf16``); the dict
    then also holds that q as ``q_scores``.

    Returns a dict with q [N][h*dk], qhat, s1 [N][h][C1], s2 [N][h][C2],
    sub_i/sub_s [N][h][2][k] (per-half top-k, best first), idx [N][h][k]
    (flat value rows i*C2 + j, best first), S [N][h][k] (scaled winner scores),
    w [N][h][k] (softmax weights) and y [N][d_v].
    """
    h, dk, C1, C2, k = cfg.h, cfg.dk, cfg.C1, cfg.C2, cfg.k
    if bn_train:
        q, qhat, mu, var = query_network_train(inp["x"], inp["Wq"], inp["bn"], cfg.bn_eps)
    else:
        q, qhat = query_network(inp["x"], inp["Wq"], inp["bn"], cfg.bn_eps)
    qs = round_bf16(q) if q_bf16 else q
    score = subkey_scores_idw if idw else subkey_scores
    s1, s2 = score(qs, inp["subkeys"], h, dk, C1)
    N = q.shape[0]
    pick = brute_force_topk if select == "brute" else product_key_topk
    ksel = k * k if all_k2 else k
    idx = np.zeros((N, h, ksel), dtype=np.int64)
    S = np.zeros((N, h, ksel))
    sub_i = np.zeros((N, h, 2, k), dtype=np.int64)
    sub_s = np.zeros((N, h, 2, k))
    for t in range(N):
        for hh in range(h):
            sub_i[t, hh, 0], sub_s[t, hh, 0] = half_topk(s1[t, hh], k)
            sub_i[t, hh, 1], sub_s[t, hh, 1] = half_topk(s2[t, hh], k)
            if all_k2:
                ii = np.repeat(sub_i[t, hh, 0], k)
                jj = np.tile(sub_i[t, hh, 1], k)
            else:
                ii, jj = pick(s1[t, hh], s2[t, hh], k)
            idx[t, hh] = ii * C2 + jj
            S[t, hh] = cfg.score_scale * (s1[t, hh, ii] + s2[t, hh, jj])
    w = softmax(S)
    y = bag(w, idx, inp["values"])
    out = dict(q=q, qhat=qhat, s1=s1, s2=s2, sub_i=sub_i, sub_s=sub_s, idx=idx, S=S, w=w, y=y)
    if q_bf16:
        out["q_scores"] = qs
    if bn_train:
        out["bn_batch"] = (mu, var)
    if idw:
        out["idw"] = True
    return out


def bag(w, idx, values):
    """y[t] = sum_h sum_j w[t][h][j] * V[idx[t][h][j]]  ("Meta AI 可扩展内存层" 5.3)."""
    N, h, k = idx.shape
    rows = np.asarray(values[idx.reshape(-1)], dtype=np.float64).reshape(N, h * k, -1)
    return np.einsum("tr,trd->td", w.reshape(N, h * k), rows)


# ----------------------------------------------------------------------------- backward
def backward(inp, cfg, fwd, dy):
    """Gradients of L = sum_t dy[t] . y[t] with the selected keys held fixed.
    After a ``q_bf16`` forward the sub-key gradients take the rounded q the scores
    used, and the rounding passes the query gradient through unchanged.

    Returns dict:
      dw   [N][h][k]   dL/dw            = dy[t] . V[row]
      dS   [N][h][k]   dL/d(scaled score) (softmax backward)
      g1, g2 [N][h][C1|C2]  dL/ds1, dL/ds2 (nonzero only on selected sub-keys)
      dq   [N][h*dk], dx [N][d_in], dWq [h*dk][d_in], dgamma, dbeta [h*dk]
      dsub [h][C1+C2][dk/2]
      dV_rows (sorted unique rows), dV_vals [len][d_v]  (all other rows are zero)
    """
    h, dk, C1, C2 = cfg.h, cfg.dk, cfg.C1, cfg.C2
    dy = np.asarray(dy, dtype=np.float64)
    idx, w = fwd["idx"], fwd["w"]
    N, k = idx.shape[0], idx.shape[2]      # selections per head (k, or k*k for all_k2)
    V = inp["values"]
    rows = np.asarray(V[idx.reshape(-1)], dtype=np.float64).reshape(N, h, k, -1)
    dw = np.einsum("td,thjd->thj", dy, rows)
    # softmax backward: dS_j = w_j (dw_j - sum_l w_l dw_l)
    dS = w * (dw - (w * dw).sum(axis=-1, keepdims=True))
    dsum = cfg.score_scale * dS
    g1 = np.zeros((N, h, C1))
    g2 = np.zeros((N, h, C2))
    tt = np.repeat(np.arange(N), h * k)
    hh = np.tile(np.repeat(np.arange(h), k), N)
    np.add.at(g1, (tt, hh, (idx // C2).reshape(-1)), dsum.reshape(-1))
    np.add.at(g2, (tt, hh, (idx % C2).reshape(-1)), dsum.reshape(-1))
    sub = np.asarray(inp["subkeys"], dtype=np.float64)
    q1, q2 = split_halves(fwd.get("q_scores", fwd["q"]), h, dk)
    if fwd.get("idw"):
        # s = -1/2 log(||q - c||^2 + eps): ds/dq = (c - q) / (||q - c||^2 + eps) = -ds/dc;
        # with u = g / (||q - c||^2 + eps) = g * exp(2 s):
        #   dq = sum_i u_i c_i - q sum_i u_i,  dc_i = sum_t u_ti q_t - c_i sum_t u_ti
        u1 = g1 * np.exp(2.0 * fwd["s1"])
        u2 = g2 * np.exp(2.0 * fwd["s2"])
        dq1 = np.einsum("thi,hid->thd", u1, sub[:, :C1, :]) - q1 * u1.sum(-1)[..., None]
        dq2 = np.einsum("thj,hjd->thd", u2, sub[:, C1:, :]) - q2 * u2.sum(-1)[..., None]
        dsub = np.zeros_like(sub)
        dsub[:, :C1, :] = (np.einsum("thi,thd->hid", u1, q1) -
                           sub[:, :C1, :] * u1.sum(0)[..., None])
        dsub[:, C1:, :] = (np.einsum("thj,thd->hjd", u2, q2) -
                           sub[:, C1:, :] * u2.sum(0)[..., None])
    else:
        dq1 = np.einsum("thi,hid->thd", g1, sub[:, :C1, :])
        dq2 = np.einsum("thj,hjd->thd", g2, sub[:, C1:, :])
        dsub = np.zeros_like(sub)
        dsub[:, :C1, :] = np.einsum("thi,thd->hid", g1, q1)
        dsub[:, C1:, :] = np.einsum("thj,thd->hjd", g2, q2)
    dq = np.concatenate([dq1, dq2], axis=2).reshape(N, h * dk)
    mean, var, gamma, beta = (np.asarray(r, dtype=np.float64) for r in inp["bn"])
    dgamma = (dq * fwd["qhat"]).sum(axis=0)
    dbeta = dq.sum(axis=0)
    if "bn_batch" in fwd:
        # batch statistics depend on every token: d pre = gamma / sqrt(var + eps) *
        # (dq - mean_t dq - q-hat * mean_t (dq q-hat))
        var_b = fwd["bn_batch"][1]
        n = dq.shape[0]
        dq_pre = gamma / np.sqrt(var_b + cfg.bn_eps) * (dq - dbeta / n - fwd["qhat"] * dgamma / n)
    else:
        dq_pre = dq * gamma / np.sqrt(var + cfg.bn_eps)
    x = np.asarray(inp["x"], dtype=np.float64)
    Wq = np.asarray(inp["Wq"], dtype=np.float64)
    dWq = dq_pre.T @ x
    dx = dq_pre @ Wq
    # value gradient: dV[row] += w * dy[t], summed over every (t, h, j) choosing row
    flat = idx.reshape(-1)
    contrib = (w[..., None] * dy[:, None, None, :]).reshape(N * h * k, -1)
    dV_rows, inv = np.unique(flat, return_inverse=True)
    dV_vals = np.zeros((dV_rows.shape[0], dy.shape[1]))
    np.add.at(dV_vals, inv, contrib)
    return dict(dw=dw, dS=dS, g1=g1, g2=g2, dq=dq, dq_pre=dq_pre, dx=dx, dWq=dWq,
                dgamma=dgamma, dbeta=dbeta, dsub=dsub, dV_rows=dV_rows, dV_vals=dV_vals)


def loss(inp, cfg, dy, select="brute"):
    """L = sum_t dy[t] . y[t] (the scalar whose gradient ``backward`` returns)."""
    f = forward(inp, cfg, select=select)
    return float((np.asarray(dy, dtype=np.float64) * f["y"]).sum()), f


# ----------------------------------------------------------------------------- fast weights
class _WrittenRows:
    """The value table as the fast-weight loop sees it: the initial table, with the
    rows written so far held in fp64 on top.  Indexing with an array of rows returns
    those rows as fp64 (what ``bag`` and ``backward`` read), so the loop never copies
    the whole table."""

    def __init__(self, values):
        self.base = values
        self.rows = np.zeros(0, dtype=np.int64)        # sorted
        self.vals = np.zeros((0, values.shape[1]))

    def __getitem__(self, r):
        r = np.asarray(r, dtype=np.int64)
        out = np.asarray(self.base[r], dtype=np.float64)
        if self.rows.size:
            pos = np.clip(np.searchsorted(self.rows, r), 0, self.rows.size - 1)
            hit = self.rows[pos] == r
            out[hit] = self.vals[pos[hit]]
        return out

    def sgd(self, r, g, lr):
        """rows r (unique) <- rows r - lr * g."""
        new = self[r] - lr * g
        keep = ~np.isin(self.rows, r)
        rows = np.concatenate([self.rows[keep], r])
        vals = np.concatenate([self.vals[keep], new])
        order = np.argsort(rows, kind="stable")
        self.rows, self.vals = rows[order], vals[order]


def fastweight_chunks(inp, cfg, chunk, lr, targets=None, lookahead=False, select="brute"):
    """Chunked read-then-write of the fast-weight product-key memory ("Fast-weight
    Product Key Memory", sections 2.2 and 3, test-time training).

    The token sequence is cut into consecutive chunks of ``chunk`` tokens.  Each chunk
    first READS: the layer's forward with the current value table.  Then it WRITES:
    one step of SGD with rate ``lr`` on the value rows it selected, descending the
    chunk's reconstruction loss L_c = sum_{t in chunk} 1/2 ||y_t - target_t||^2
    (only the value table is a fast weight here; queries and keys stay fixed).  The
    next chunk reads the table this chunk wrote.

    Targets: ``targets[t]`` [N][d_v], or with ``lookahead`` the next token's input,
    target_t = x[t + 1] (needs d_in = d_v); the sequence's last token then has no
    target and adds nothing to the loss.

    Returns (y [N][d_v] of every read, written rows (sorted), their final values).
    """
    N = inp["x"].shape[0]
    x = np.asarray(inp["x"], dtype=np.float64)
    if lookahead:
        assert cfg.d_in == cfg.d_v
        tg = np.zeros((N, cfg.d_v))
        tg[:-1] = x[1:]
        has_target = np.arange(N) < N - 1
    else:
        tg = np.asarray(targets, dtype=np.float64)
        has_target = np.ones(N, dtype=bool)
    table = _WrittenRows(inp["values"])
    ys = np.zeros((N, cfg.d_v))
    for c0 in range(0, N, chunk):
        c1 = min(N, c0 + chunk)
        sub = dict(inp, x=inp["x"][c0:c1], values=table)
        f = forward(sub, cfg, select=select)
        ys[c0:c1] = f["y"]
        dy = (f["y"] - tg[c0:c1]) * has_target[c0:c1, None]
        b = backward(sub, cfg, f, dy)
        table.sgd(b["dV_rows"], b["dV_vals"], lr)
    return ys, table.rows, table.vals


# ----------------------------------------------------------------------------- training pieces
def hit_counts(fwd, cfg):
    """Hit monitoring of one batch ("Meta AI 可扩展内存层" sections 6.4 and 11.2: how often
    each slot and each sub-key of each codebook is selected).

    slot [C1*C2]: number of selections (t, h, j) of each value row.
    sub [h][C1+C2]: per head, how many winners use each sub-key: entry i < C1 counts
    winners whose first-half sub-key is i, entry C1 + j those whose second-half one is j.
    """
    idx = np.asarray(fwd["idx"], dtype=np.int64)
    slot = np.bincount(idx.ravel(), minlength=cfg.K)
    sub = np.zeros((cfg.h, cfg.C1 + cfg.C2), dtype=np.int64)
    for hh in range(cfg.h):
        sub[hh] += np.bincount(idx[:, hh, :].ravel() // cfg.C2, minlength=cfg.C1 + cfg.C2)
        sub[hh, cfg.C1:] += np.bincount(idx[:, hh, :].ravel() % cfg.C2, minlength=cfg.C2)
    return slot, sub


def sparse_adam(values, m, v, rows, grads, lr, beta1, beta2, eps, step):
    """Lazy Adam on the touched value rows only ("Meta AI 可扩展内存层" section 6.3:
    optimiser state is kept and advanced only for parameters that received a gradient).

    For each touched row r with gradient g (rows unique, e.g. ``backward``'s dV_rows
    and dV_vals):  m_r <- beta1 m_r + (1 - beta1) g;  v_r <- beta2 v_r + (1 - beta2) g^2;
    V_r <- V_r - lr * (m_r / (1 - beta1^step)) / (sqrt(v_r / (1 - beta2^step)) + eps),
    with ``step`` >= 1 the caller's global step count.  Other rows and their state are
    left as they are.  Returns new (values, m, v) as fp64 copies.
    """
    V = np.array(values, dtype=np.float64, copy=True)
    M = np.array(m, dtype=np.float64, copy=True)
    S = np.array(v, dtype=np.float64, copy=True)
    g = np.asarray(grads, dtype=np.float64)
    M[rows] = beta1 * M[rows] + (1.0 - beta1) * g
    S[rows] = beta2 * S[rows] + (1.0 - beta2) * g * g
    mhat = M[rows] / (1.0 - beta1 ** step)
    vhat = S[rows] / (1.0 - beta2 ** step)
    V[rows] -= lr * mhat / (np.sqrt(vhat) + eps)
    return V, M, S
