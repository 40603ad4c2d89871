"""The plain statement of the row-sharded exchange (``tests/shard_ref.py``), composed over
G ranks in one process (the all-to-alls as slicing), equals the oracle of the whole layer:
bag, dL/dw and the value gradient of every shard, with ragged token batches and with more
shards than leading sub-keys (empty shards)."""
import numpy as np
import pytest

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import sharded as S
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs
from tests import shard_ref as SR

CFG = PKMConfig("shard_ref", N=23, d_in=16, h=2, dk=8, C1=7, C2=5, k=3, d_v=8, dtype="f32")


def _a2a(send_parts):
    """send_parts[src][dst] -> recv[dst] = concatenation over src in order."""
    G = len(send_parts)
    return [np.concatenate([send_parts[s][d] for s in range(G)]) for d in range(G)]


def _split(x, splits):
    return np.split(x, np.cumsum(splits)[:-1])


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_plain_statement_composes_to_the_layer(G):
    inp = make_inputs(CFG, seed=5, random_bn=True)
    of = O.forward(inp, CFG)
    ob = O.backward(inp, CFG, of, inp["dy"])
    R = S.rows_per_shard(CFG.C1, CFG.C2, G)
    bounds = np.linspace(0, CFG.N, G + 1).astype(int)
    hk = CFG.h * CFG.k
    vals = inp["values"].astype(np.float64)
    ranks = []
    for r in range(G):
        t0, t1 = bounds[r], bounds[r + 1]
        idx = of["idx"][t0:t1].reshape(-1, hk)
        w = of["w"][t0:t1].reshape(-1, hk)
        counts, segpos, send, perm = SR.route(idx, w, G, R)
        assert counts[:, 0].sum() == (t1 - t0) * hk
        ranks.append(dict(counts=counts, segpos=segpos, send=send, perm=perm, t=(t0, t1)))
    # counts and triples to the owners
    recv_counts = _a2a([[rk["counts"][d:d + 1] for d in range(G)] for rk in ranks])
    recv = _a2a([_split(rk["send"], rk["counts"][:, 0]) for rk in ranks])
    partial = [SR.owner_bag(recv_counts[g], recv[g], vals[g * R:(g + 1) * R], CFG.d_v)
               for g in range(G)]
    back = _a2a([_split(partial[g], recv_counts[g][:, 1]) for g in range(G)])
    y = np.concatenate([SR.combine(rk["segpos"], back[r]) for r, rk in enumerate(ranks)])
    np.testing.assert_allclose(y, of["y"], rtol=1e-6, atol=1e-7)
    # backward
    dy_send = [SR.gather_dy(rk["segpos"], inp["dy"][rk["t"][0]:rk["t"][1]].astype(np.float64),
                            int(rk["counts"][:, 1].sum())) for rk in ranks]
    dy_recv = _a2a([_split(dy_send[r], ranks[r]["counts"][:, 1]) for r in range(G)])
    dV = np.zeros((CFG.K, CFG.d_v))
    dw_recv = []
    for g in range(G):
        r0, r1 = S.shard_range(g, G, CFG.C1, CFG.C2)
        dVg = np.zeros((max(r1 - r0, 1), CFG.d_v))
        dw_recv.append(SR.owner_value_grad(recv_counts[g], recv[g], vals[r0:max(r1, r0 + 1)],
                                           dy_recv[g], dVg) if len(recv[g]) else np.zeros(0))
        dV[r0:r1] = dVg[:r1 - r0]
    dw_back = _a2a([_split(dw_recv[g], recv_counts[g][:, 0]) for g in range(G)])
    dw = np.concatenate([SR.scatter_dw(rk["perm"], dw_back[r], (rk["t"][1] - rk["t"][0]) * hk)
                         for r, rk in enumerate(ranks)])
    np.testing.assert_allclose(dw, ob["dw"].reshape(-1), rtol=1e-6, atol=1e-7)
    dV_full = np.zeros((CFG.K, CFG.d_v))
    dV_full[ob["dV_rows"]] = ob["dV_vals"]
    np.testing.assert_allclose(dV, dV_full, rtol=1e-6, atol=1e-7)


def test_route_layout_on_a_hand_example():
    """Two tokens, three selections each, two shards of 10 rows."""
    idx = np.array([[12, 3, 15], [4, 5, 19]])
    w = np.array([[0.5, 0.25, 0.25], [0.6, 0.3, 0.1]], np.float32)
    counts, segpos, send, perm = SR.route(idx, w, 2, 10)
    np.testing.assert_array_equal(counts, [[3, 2], [3, 2]])
    np.testing.assert_array_equal(segpos, [[0, 1], [2, 3]])
    # shard 0: token 0's row 3 (segment 0), token 1's rows 4, 5 (segment 1)
    np.testing.assert_array_equal(send[:, :2], [[0, 3], [1, 4], [1, 5], [0, 2], [0, 5], [1, 9]])
    np.testing.assert_array_equal(perm, [1, 3, 4, 0, 2, 5])
    np.testing.assert_array_equal(send[:, 2].view(np.float32),
                                  np.float32([0.25, 0.6, 0.3, 0.5, 0.25, 0.1]))
