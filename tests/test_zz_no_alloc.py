"""The value-gradient entry point that allocates nothing (pkm_value_grad_noalloc).

Some callers cannot allocate device memory, so they cannot pass a workspace.  One is a
plugin whose host framework owns every device allocation.  Another is a latency-bound
loop that must not call cudaMalloc, which can synchronise the device.  This entry
point keeps its scratch in a fixed array inside the library.  These tests check that
it returns what the workspace-taking pkm_value_grad returns, on two calls in a row
(the array is shared and reused).  They also check that a problem one selection too
large for the array is refused on the host before any CUDA call, and that the largest
problem that fits runs and matches.  The file name sorts last so that a run stopping
at the first failure has run every other test first.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from product_key_memory_pkm_b200 import build as B
from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200.inputs import PKMConfig, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = PKMConfig("noalloc_case", N=2048, d_in=128, h=4, dk=128, C1=128, C2=128, k=32, d_v=256)
# one head, one key per token: N counts the selections one by one
LIMIT_SHAPE = dict(d_in=8, h=1, dk=32, C1=256, C2=256, k=1, d_v=8)


def _noalloc_rc_with_fake_pointers(d: "P.Dims") -> int:
    """Return code of a call whose pointers are fake (aligned, never dereferenced).
    Only safe where the call cannot reach a launch: a refused size, or a process
    that sees no GPU (the call then stops at its first CUDA call)."""
    fake = 1 << 20
    saved = P._saved_c({f: fake for f in P.SAVED_FIELDS})
    return P.load().pkm_value_grad_noalloc(ctypes.byref(d.c()), fake, ctypes.byref(saved), fake,
                                           fake, fake, None)


_PROBE = r"""
import sys
sys.path.insert(0, sys.argv[1])
from product_key_memory_pkm_b200 import pkm as P
from tests.test_zz_no_alloc import LIMIT_SHAPE, _noalloc_rc_with_fake_pointers
lo, hi = 1, 1 << 26          # lo fits, hi does not
assert _noalloc_rc_with_fake_pointers(P.Dims(N=hi, **LIMIT_SHAPE)) == P.PKM_ERR_WORKSPACE
assert _noalloc_rc_with_fake_pointers(P.Dims(N=lo, **LIMIT_SHAPE)) == P.PKM_ERR_CUDA
while hi - lo > 1:
    mid = (lo + hi) // 2
    rc = _noalloc_rc_with_fake_pointers(P.Dims(N=mid, **LIMIT_SHAPE))
    assert rc in (P.PKM_ERR_WORKSPACE, P.PKM_ERR_CUDA), rc
    if rc == P.PKM_ERR_WORKSPACE:
        hi = mid
    else:
        lo = mid
print(lo)
"""


def _largest_fitting_selections() -> int:
    """Largest N (one selection per token) the fixed scratch accepts, found by
    bisection on the host-side size check in a child process that sees no GPU: there a
    call that passes the check stops at its first CUDA call with PKM_ERR_CUDA, so no
    fake pointer ever reaches a kernel."""
    B.build()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "-c", _PROBE, ROOT], env=env, cwd=ROOT,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    return int(out.stdout.strip().splitlines()[-1])


def test_too_large_for_the_fixed_scratch_is_refused_on_the_host():
    B.build()
    d = P.Dims(N=16384, d_in=1600, h=4, dk=512, C1=1024, C2=1024, k=32, d_v=1600)
    assert _noalloc_rc_with_fake_pointers(d) == P.PKM_ERR_WORKSPACE


def test_the_size_limit_is_about_53_bytes_per_selection():
    n = _largest_fitting_selections()
    # the documented limit: about 53 bytes per selection in 64 MiB
    assert 0.95 * (64 << 20) / 53 < n < 1.05 * (64 << 20) / 53, n
    assert _noalloc_rc_with_fake_pointers(P.Dims(N=n + 1, **LIMIT_SHAPE)) == P.PKM_ERR_WORKSPACE


def _compare_with_workspace_entry_point(dims, values, saved, dy, K, d_v, calls=2):
    from tests import parity as H
    n_sel = saved["idx"].numel()
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    dV_ref = torch.zeros(K, d_v, device="cuda")
    dw_ref = torch.zeros(n_sel, device="cuda")
    P.pkm_value_grad(dims, values, saved, dy, dw_ref, dvalues=dV_ref, workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    del ws
    rows = np.unique(saved["idx"].cpu().numpy())
    for _ in range(calls):   # later calls reuse the array the previous one left behind
        dV = torch.zeros(K, d_v, device="cuda")
        dw = torch.full((n_sel,), float("nan"), device="cuda")
        P.pkm_value_grad_noalloc(dims, values, saved, dy, dw, dvalues=dV)
        assert P.pkm_check_status() == P.PKM_OK
        H.assert_rows(dw.cpu().numpy().reshape(-1, 1), dw_ref.cpu().numpy().reshape(-1, 1), "dw")
        H.assert_rows(dV.cpu().numpy()[rows], dV_ref.cpu().numpy()[rows], "dV")
        untouched = torch.ones(K, dtype=torch.bool, device="cuda")
        untouched[torch.from_numpy(rows).cuda()] = False
        assert not torch.any(dV[untouched])


@pytest.mark.gpu
def test_value_grad_noalloc_matches_the_workspace_entry_point_twice():
    from tests import parity as H
    B.build()
    inp = make_inputs(CFG, seed=4)
    dev = H.to_dev(inp, CFG)
    dims, saved, _ = H.gpu_forward(CFG, dev)
    _compare_with_workspace_entry_point(dims, dev["values"], saved, dev["dy"], CFG.K, CFG.d_v)


@pytest.mark.gpu
def test_value_grad_noalloc_at_the_size_limit():
    n = _largest_fitting_selections()
    sh = LIMIT_SHAPE
    K = sh["C1"] * sh["C2"]
    g = torch.Generator().manual_seed(11)
    idx = torch.randint(0, K, (n, 1, 1), generator=g, dtype=torch.int32).cuda()
    w = torch.rand(n, 1, 1, generator=g).cuda()
    dy = torch.randn(n, sh["d_v"], generator=g).cuda()
    values = (torch.randn(K, sh["d_v"], generator=g) / 8).to(torch.bfloat16).cuda()
    saved = {"idx": idx, "w": w}
    # one selection over the limit: refused on the host, real buffers untouched
    over = P.Dims(N=n + 1, **sh)
    with pytest.raises(RuntimeError, match="PKM_ERR_WORKSPACE"):
        P.pkm_value_grad_noalloc(over, values, saved, dy, torch.zeros(n + 1, device="cuda"))
    _compare_with_workspace_entry_point(P.Dims(N=n, **sh), values, saved, dy, K, sh["d_v"])
