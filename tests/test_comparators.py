"""The parity comparators themselves, exercised on the CPU with oracle values and planted
errors (no GPU needed)."""
import numpy as np
import pytest

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs
from tests import parity as H


def _one_token_case(seed):
    cfg = PKMConfig(name="one_token", N=1, d_in=32, h=2, dk=16, C1=20, C2=14, k=6, d_v=12,
                    dtype="f32", score_scale=0.5)
    inp = make_inputs(cfg, seed=seed, random_bn=True)
    of = O.forward(inp, cfg)
    ob = O.backward(inp, cfg, of, inp["dy"])
    return cfg, inp, of, ob


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dwq_term_magnitude_bounds_the_gradient(seed):
    """Triangle inequality: every entry of dWq is at most the size of its terms, and the
    bound is tight for some entry (a term dropped from the bound would break one)."""
    cfg, inp, of, ob = _one_token_case(seed)
    mag = H.dwq_term_magnitude(inp, cfg, of, ob)
    assert mag.shape == ob["dWq"].shape
    assert np.all(np.abs(ob["dWq"]) <= mag * (1 + 1e-12) + 1e-300)
    assert (np.abs(ob["dWq"]) / np.maximum(mag, 1e-300)).max() > 0.05


@pytest.mark.parametrize("seed", [0, 1])
def test_dwq_comparator_rejects_planted_errors(seed):
    """An error of 1e-3 of an entry's term size fails the check; 1e-7 of it passes."""
    cfg, inp, of, ob = _one_token_case(seed)
    want = ob["dWq"]
    mag = H.dwq_term_magnitude(inp, cfg, of, ob)
    o, e = np.unravel_index(np.argmax(mag), mag.shape)
    ok = want.copy()
    ok[o, e] += 1e-7 * mag[o, e]
    H.assert_dwq(ok, want, mag)
    bad = want.copy()
    bad[o, e] += 1e-3 * mag[o, e]
    with pytest.raises(AssertionError):
        H.assert_dwq(bad, want, mag)


def test_dwq_comparator_without_magnitude_is_the_row_check():
    cfg, inp, of, ob = _one_token_case(0)
    want = ob["dWq"]
    bad = want.copy()
    r = int(np.argmax(np.abs(want).max(axis=1)))
    bad[r, 0] += 1e-2 * np.abs(want[r]).max()
    with pytest.raises(AssertionError):
        H.assert_dwq(bad, want, None)
    H.assert_dwq(want.copy(), want, None)
