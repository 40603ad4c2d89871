"""The value-gradient entry point that allocates nothing (pkm_value_grad_noalloc).

It serves callers that cannot allocate device memory -- code running during a CUDA
graph capture, or a plugin whose host framework owns every device allocation -- by
keeping its scratch in a fixed array inside the library.  These tests check that it
returns what the workspace-taking pkm_value_grad returns, on two calls in a row (the
array is shared and reused), and that a problem too large for the array is refused on
the host before any device work.  The file name sorts last so that a run stopping at
the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs

CFG = PKMConfig("noalloc_case", N=2048, d_in=128, h=4, dk=128, C1=128, C2=128, k=32, d_v=256)


def test_too_large_for_the_fixed_scratch_is_refused_on_the_host():
    P.load()
    d = P.Dims(N=16384, d_in=1600, h=4, dk=512, C1=1024, C2=1024, k=32, d_v=1600)
    fake = 1 << 20
    saved = P._saved_c({f: fake for f in P.SAVED_FIELDS})
    rc = P.load().pkm_value_grad_noalloc(ctypes.byref(d.c()), fake, ctypes.byref(saved), fake,
                                         fake, fake, None)
    assert rc == P.PKM_ERR_WORKSPACE


@pytest.mark.gpu
def test_value_grad_noalloc_matches_the_workspace_entry_point_twice():
    from tests import parity as H
    from product_key_memory_pkm_b200 import build as B
    B.build()
    inp = make_inputs(CFG, seed=4)
    dev = H.to_dev(inp, CFG)
    dims, saved, _ = H.gpu_forward(CFG, dev)
    dy = dev["dy"]

    # reference: the entry point that takes a caller-allocated workspace
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    dV_ref = torch.zeros(CFG.K, CFG.d_v, device="cuda")
    dw_ref = torch.zeros(CFG.N, CFG.h, CFG.k, device="cuda")
    P.pkm_value_grad(dims, dev["values"], saved, dy, dw_ref, dvalues=dV_ref, workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK

    for _ in range(2):      # the second call reuses the array the first one left behind
        dV = torch.zeros(CFG.K, CFG.d_v, device="cuda")
        dw = torch.full((CFG.N, CFG.h, CFG.k), float("nan"), device="cuda")
        P.pkm_value_grad_noalloc(dims, dev["values"], saved, dy, dw, dvalues=dV)
        assert P.pkm_check_status() == P.PKM_OK
        H.assert_rows(dw.cpu().numpy().reshape(-1, CFG.k),
                      dw_ref.cpu().numpy().reshape(-1, CFG.k), "dw")
        rows = np.unique(saved["idx"].cpu().numpy())
        H.assert_rows(dV.cpu().numpy()[rows], dV_ref.cpu().numpy()[rows], "dV")
        untouched = torch.ones(CFG.K, dtype=torch.bool, device="cuda")
        untouched[torch.from_numpy(rows).cuda()] = False
        assert not torch.any(dV[untouched])
