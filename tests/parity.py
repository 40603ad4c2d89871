"""Helpers of the GPU parity tests: run the CUDA path through the C ABI binding and
compare with the CPU oracle under the agreement rules of the layer:

* indices: where the oracle's gap between the k-th and (k+1)-th product-key score
  exceeds 1e-4 relative (gap > 1e-4 * max(|S_k|, 1e-2)), the GPU's index set must equal
  the oracle's exactly, and every prefix of the ranking that the oracle separates by
  such a gap must agree as a set.  Otherwise several sets are correct: every GPU key
  must then score (in the oracle) at least S_k - tol.
* outputs and gradients: max relative error 2e-3 per row,
  max_e |got - want| / max(max_e |want|, 1e-6).
  Only the sub-key and BatchNorm gradients (dsub, dbn) take a wider floor,
  1e-3 * max |want over the tensor|, because they have rows that cancel to zero
  analytically: a sub-key shared by every winner of a head collects the sum of the
  softmax gradient over the head, which is exactly zero and which fp32 leaves as a
  ~1e-8 residue.  Every other tensor (y, w, dw, dV, dx, dWq, ...) has no such rows.
Tokens with a near-tie head (decided from the oracle alone) are left out of the direct
output comparison and have their upstream gradient masked to zero, so every compared
value is unique.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import pkm as P

GAP_REL = 1e-4
ROW_REL = 2e-3


def to_dev(inp: dict, cfg, device="cuda") -> dict:
    """Inputs on the device in their storage types."""
    st = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out = {}
    for k, v in inp.items():
        t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
        if k in ("x", "Wq", "subkeys"):
            t = t.to(st)
        elif k == "values" and cfg.vdtype == "bf16":
            t = t.to(torch.bfloat16)
        out[k] = t.to(device)
    return out


def gpu_forward(cfg, dev: dict, flags: int = 0, with_qhat: bool = True, fused: bool = False):
    """The forward through the C ABI; ``fused`` passes the few-token workspace, so the
    call runs as the single fused kernel (asserted through the launch counter)."""
    dims = P.Dims.from_config(cfg, flags=flags)
    saved = P.alloc_saved(dims, with_qhat=with_qhat)
    y = torch.empty(cfg.N, cfg.d_v, dtype=torch.float32, device="cuda")
    ws = None
    if fused:
        assert P.pkm_workspace_bytes(dims, P.PKM_FWD_FUSED) > 0
        ws = P.alloc_workspace(dims, P.PKM_FWD_FUSED)
    n0 = P.pkm_launch_count()
    P.pkm_forward(dims, dev["x"], dev["Wq"], dev["bn"], dev["subkeys"], dev["values"], y, saved,
                  workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    if fused:
        assert P.pkm_launch_count() - n0 == 1
    return dims, saved, y


def gpu_backward(cfg, dims, dev: dict, saved: dict, dy: torch.Tensor, want=("dx", "dWq", "dbn",
                                                                          "dsub", "dV", "dw")):
    z = lambda *s: torch.zeros(*s, dtype=torch.float32, device="cuda")
    g = dict(
        dx=z(cfg.N, cfg.d_in) if "dx" in want else None,
        dWq=z(cfg.h * cfg.dk, cfg.d_in) if "dWq" in want else None,
        dbn=z(2, cfg.h * cfg.dk) if "dbn" in want else None,
        dsub=z(cfg.h, cfg.C1 + cfg.C2, cfg.dk // 2) if "dsub" in want else None,
        dV=z(cfg.K, cfg.d_v) if "dV" in want else None,
        dw=z(cfg.N, cfg.h, cfg.k) if "dw" in want else None,
    )
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    P.pkm_backward(dims, dev["x"], dev["Wq"], dev["bn"], dev["subkeys"], dev["values"], saved, dy,
                   dx=g["dx"], dWq=g["dWq"], dbn=g["dbn"], dsubkeys=g["dsub"], dvalues=g["dV"],
                   dw_out=g["dw"], workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    return g


def oracle_gaps(of: dict, cfg, select: str = "brute"):
    """Per (t, h): the oracle's ranked scores of the best k+1 keys (unscaled sums).
    ``select="product"`` takes them by the product-key search (exact, and far cheaper
    over a million keys)."""
    N = of["s1"].shape[0]
    ranked = np.zeros((N, cfg.h, cfg.k + 1))
    pick = O.brute_force_topk if select == "brute" else O.product_key_topk
    for t in range(N):
        for hh in range(cfg.h):
            ii, jj = pick(of["s1"][t, hh], of["s2"][t, hh], cfg.k + 1)
            ranked[t, hh] = of["s1"][t, hh, ii] + of["s2"][t, hh, jj]
    return ranked


def check_indices(idx_gpu: np.ndarray, of: dict, cfg, ranked: np.ndarray):
    """Returns a boolean [N] array of tokens whose every head is clean (gap > tol)."""
    N = idx_gpu.shape[0]
    clean_tok = np.ones(N, dtype=bool)
    for t in range(N):
        for hh in range(cfg.h):
            r = ranked[t, hh]
            tol = GAP_REL * max(abs(r[cfg.k - 1]), 1e-2)
            g = idx_gpu[t, hh]
            o = of["idx"][t, hh]
            assert len(set(g.tolist())) == cfg.k, (t, hh, "duplicate keys")
            if r[cfg.k - 1] - r[cfg.k] > tol:
                assert set(g.tolist()) == set(o.tolist()), (t, hh, g, o)
                for j in range(cfg.k - 1):
                    if r[j] - r[j + 1] > GAP_REL * max(abs(r[j]), 1e-2):
                        assert set(g[: j + 1].tolist()) == set(o[: j + 1].tolist()), (t, hh, j)
            else:
                clean_tok[t] = False
                ii, jj = g // cfg.C2, g % cfg.C2
                sc = of["s1"][t, hh, ii] + of["s2"][t, hh, jj]
                assert np.all(sc >= r[cfg.k - 1] - tol), (t, hh, sc, r)
    return clean_tok


ABS_FLOOR = 1e-6
ZERO_ROW_FLOOR = 1e-3


def row_rel_err(got: np.ndarray, want: np.ndarray, zero_rows: bool = False) -> float:
    """Max over rows of max_e |got - want| / max(max_e |want|, floor).  The floor is
    ABS_FLOOR, or ZERO_ROW_FLOOR times the tensor's max |want| for a tensor with rows
    that are analytically zero (``zero_rows``)."""
    if np.asarray(want).size == 0:
        return 0.0
    got = np.asarray(got, dtype=np.float64).reshape(want.shape[0], -1)
    want = np.asarray(want, dtype=np.float64).reshape(want.shape[0], -1)
    err = np.abs(got - want).max(axis=1)
    floor = ABS_FLOOR
    if zero_rows:
        floor = max(floor, ZERO_ROW_FLOOR * float(np.abs(want).max()))
    den = np.maximum(np.abs(want).max(axis=1), floor)
    return float((err / den).max()) if want.shape[0] else 0.0


def assert_rows(got, want, name: str, tol: float = ROW_REL, zero_rows: bool = False):
    e = row_rel_err(got, want, zero_rows=zero_rows)
    assert e <= tol, f"{name}: max row relative error {e:.3e} > {tol}"
    return e


MAG_REL = 1e-4


def dwq_term_magnitude(inp: dict, cfg, of: dict, ob: dict):
    """Per element of dWq, the size of the terms its computation adds up (dot-product
    scores, running BatchNorm statistics), or None for other forms.

    dq[t, o] = sum_j scale w_j (dw_j - sum_l w_l dw_l) c_j[o] cancels by construction (the
    softmax gradient sums to zero over the selection), so its rounding error scales with
    A[t, o] = sum_j scale w_j (|dw_j| + sum_l w_l |dw_l|) |c_j[o]|, not with |dq[t, o]|;
    dWq[o, e] = sum_t (gamma_o / sigma_o) dq[t, o] x[t, e] carries that as
    sum_t |gamma_o / sigma_o| A[t, o] |x[t, e]|."""
    if of.get("idw") or "bn_batch" in of:
        return None
    h, dk, C1, C2 = cfg.h, cfg.dk, cfg.C1, cfg.C2
    w, idx = of["w"], of["idx"]
    adw = np.abs(ob["dw"])
    m = cfg.score_scale * w * (adw + (w * adw).sum(axis=-1, keepdims=True))   # [N][h][k]
    sub = np.abs(np.asarray(inp["subkeys"], dtype=np.float64))
    N = idx.shape[0]
    A = np.zeros((N, h, dk))
    for hh in range(h):
        c1 = sub[hh, :C1, :][idx[:, hh, :] // C2]          # [N][k][dk/2]
        c2 = sub[hh, C1:, :][idx[:, hh, :] % C2]
        A[:, hh, : dk // 2] = np.einsum("tj,tjd->td", m[:, hh, :], c1)
        A[:, hh, dk // 2:] = np.einsum("tj,tjd->td", m[:, hh, :], c2)
    mean, var, gamma, beta = (np.asarray(r, dtype=np.float64) for r in inp["bn"])
    g = np.abs(gamma) / np.sqrt(var + cfg.bn_eps)
    return (A.reshape(N, h * dk) * g).T @ np.abs(np.asarray(inp["x"], dtype=np.float64))


def assert_dwq(got, want, mag, name: str = "dWq"):
    """Row check of dWq: each row within ROW_REL of its own size, or, for rows whose
    entries cancel, within MAG_REL of the size of the terms summed into them."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if mag is None:
        return assert_rows(got, want, name)
    err = np.abs(got - want).max(axis=1)
    allow = np.maximum(ROW_REL * np.maximum(np.abs(want).max(axis=1), ABS_FLOOR),
                       MAG_REL * mag.max(axis=1))
    worst = int(np.argmax(err / allow))
    assert np.all(err <= allow), (f"{name}: row {worst} error {err[worst]:.3e} > "
                                  f"allowed {allow[worst]:.3e}")


def align_to(idx_gpu: np.ndarray, idx_ref: np.ndarray, vals_gpu: np.ndarray) -> np.ndarray:
    """Reorder per-(t, h) GPU values so that they follow the reference's key order (the
    order of near-tied neighbours is not unique).  Requires equal key sets."""
    out = np.empty_like(vals_gpu)
    for t in range(idx_gpu.shape[0]):
        for hh in range(idx_gpu.shape[1]):
            pos = {int(r): j for j, r in enumerate(idx_gpu[t, hh])}
            out[t, hh] = vals_gpu[t, hh, [pos[int(r)] for r in idx_ref[t, hh]]]
    return out


def oracle_bag_at(of: dict, cfg, idx_gpu: np.ndarray, t: int, values) -> np.ndarray:
    """Oracle output of token t evaluated at a given (valid) selection: the check of a
    non-unique case."""
    y = np.zeros(cfg.d_v)
    for hh in range(cfg.h):
        g = idx_gpu[t, hh]
        S = cfg.score_scale * (of["s1"][t, hh, g // cfg.C2] + of["s2"][t, hh, g % cfg.C2])
        w = O.softmax(S)
        y += (w[:, None] * np.asarray(values[g], dtype=np.float64)).sum(0)
    return y
