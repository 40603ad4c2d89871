"""The C ABI library loads, exports every symbol ``include/pkm.h`` declares, and its
host-side validation rejects bad arguments before any device work (no GPU needed)."""
import ctypes
import os
import re

import pytest

from product_key_memory_pkm_b200 import build as B
from product_key_memory_pkm_b200 import pkm as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return P.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pkm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkm_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(P.EXPORTED)


def test_build_targets_sm100a_only():
    assert B.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_struct_layout_matches_header():
    assert ctypes.sizeof(P.pkm_dims) == 48
    assert ctypes.sizeof(P.pkm_saved) == 7 * ctypes.sizeof(ctypes.c_void_p)


def test_status_strings(lib):
    for code in range(7):
        s = P.status_string(code)
        assert s.startswith("PKM_")
    assert "UNKNOWN" in P.status_string(99)


def _dims(**kw):
    base = dict(N=64, d_in=64, h=2, dk=64, C1=32, C2=32, k=8, d_v=64)
    base.update(kw)
    return P.Dims(**base)


def test_workspace_and_saved_sizes(lib):
    d = _dims()
    assert P.pkm_workspace_bytes(d, P.PKM_FWD) == 0
    assert P.pkm_workspace_bytes(d, P.PKM_BWD) > 0
    assert P.pkm_saved_bytes(d, "q") == 2 * 2 * 64 * 128
    assert P.pkm_saved_bytes(d, "idx") == 4 * 64 * 2 * 8
    assert P.pkm_saved_bytes(d, "sub_i") == 4 * 64 * 2 * 2 * 8
    d32 = _dims(flags=P.PKM_F_FP32)
    assert P.pkm_saved_bytes(d32, "q") == 4 * 64 * 128
    assert P.pkm_saved_bytes(_dims(k=40, C1=32), "q") == 0      # invalid dims -> 0
    assert P.pkm_workspace_bytes(_dims(N=0), P.PKM_BWD) == 0


FAKE = 1 << 20          # a 16-byte-aligned address that is never dereferenced


def _fwd(d, **over):
    args = dict(x=FAKE, Wq=FAKE, bn=FAKE, subkeys=FAKE, values=FAKE, y=FAKE)
    args.update(over)
    saved = {f: FAKE for f in P.SAVED_FIELDS}
    saved.update(over.pop("saved", {}) if "saved" in over else {})
    return P.load().pkm_forward(ctypes.byref(d.c()), args["x"], args["Wq"], args["bn"],
                                args["subkeys"], args["values"], args["y"],
                                ctypes.byref(P._saved_c(saved)), None, 0, None)


@pytest.mark.parametrize("over,code", [
    (dict(k=65, C1=80, C2=80), P.PKM_ERR_UNSUPPORTED),
    (dict(k=9, C1=8), P.PKM_ERR_INVALID_ARG),
    (dict(dk=48), P.PKM_ERR_INVALID_ARG),            # bf16 needs dk % 32 == 0
    (dict(d_in=60), P.PKM_ERR_INVALID_ARG),
    (dict(d_v=12), P.PKM_ERR_INVALID_ARG),
    (dict(bn_eps=0.0), P.PKM_ERR_INVALID_ARG),
    (dict(score_scale=-1.0), P.PKM_ERR_INVALID_ARG),
    (dict(flags=0x80), P.PKM_ERR_INVALID_ARG),
    (dict(flags=P.PKM_F_BF16_Q | P.PKM_F_FP32), P.PKM_ERR_INVALID_ARG),   # no q planes
    (dict(N=-1), P.PKM_ERR_INVALID_ARG),
    (dict(C1=65536, C2=65536), P.PKM_ERR_INVALID_ARG),
])
def test_forward_rejects_bad_dims(lib, over, code):
    assert _fwd(_dims(**over)) == code


def test_k_up_to_64_passes_validation(lib):
    """k from 33 to 64 is within the boundary's limits (the host-side size queries
    accept it); k = 65 is outside them."""
    for k in (33, 48, 64):
        d = _dims(k=k, C1=64, C2=80)
        assert P.pkm_saved_bytes(d, "idx") == 4 * 64 * 2 * k
        assert P.pkm_saved_bytes(d, "sub_s") == 4 * 64 * 2 * 2 * k
        assert P.pkm_workspace_bytes(d, P.PKM_BWD) > 0
    assert P.pkm_saved_bytes(_dims(k=65, C1=80, C2=80), "idx") == 0


def test_forward_rejects_null_and_misaligned_pointers(lib):
    d = _dims()
    assert _fwd(d, x=None) == P.PKM_ERR_INVALID_ARG
    assert _fwd(d, values=FAKE + 8) == P.PKM_ERR_INVALID_ARG
    saved = {f: FAKE for f in P.SAVED_FIELDS}
    saved["idx"] = None
    rc = P.load().pkm_forward(ctypes.byref(d.c()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              ctypes.byref(P._saved_c(saved)), None, 0, None)
    assert rc == P.PKM_ERR_INVALID_ARG


def test_zero_tokens_is_a_noop(lib):
    assert _fwd(_dims(N=0)) == P.PKM_OK
    assert _fwd(_dims(N=0), x=None) == P.PKM_OK


def test_backward_checks_workspace_and_qhat(lib):
    d = _dims()
    saved = {f: FAKE for f in P.SAVED_FIELDS}
    S = ctypes.byref(P._saved_c(saved))
    L = P.load()
    need = P.pkm_workspace_bytes(d, P.PKM_BWD)
    args = (ctypes.byref(d.c()), FAKE, FAKE, FAKE, FAKE, FAKE, S, FAKE, FAKE, FAKE, FAKE, FAKE,
            FAKE, None)
    assert L.pkm_backward(*args, None, 0, None) == P.PKM_ERR_WORKSPACE
    assert L.pkm_backward(*args, FAKE, need - 1, None) == P.PKM_ERR_WORKSPACE
    assert L.pkm_backward(*args, FAKE + 16, need, None) == P.PKM_ERR_WORKSPACE  # not 256-aligned
    saved["qhat"] = None
    S2 = ctypes.byref(P._saved_c(saved))
    rc = L.pkm_backward(ctypes.byref(d.c()), FAKE, FAKE, FAKE, FAKE, FAKE, S2, FAKE, None, None,
                        FAKE, None, None, None, FAKE, need, None)
    assert rc == P.PKM_ERR_INVALID_ARG      # d gamma needs qhat


def test_fastweight_validation(lib):
    """Host-side checks of the chunked fast-weight entry point."""
    L = P.load()
    d = _dims(flags=P.PKM_F_FP32)
    need = P.pkm_fastweight_workspace_bytes(d, 16)
    assert need > 0
    ws = lambda dd, ch, m=0: P.pkm_fastweight_workspace_bytes(dd, ch, m)
    # the whole sequence is selected and sorted up front: space grows with N ...
    assert ws(_dims(N=640, flags=P.PKM_F_FP32), 16) > need
    # ... except for the per-chunk steps: one chunk's worth whatever N is
    per = P.PKM_FW_PER_CHUNK
    assert ws(_dims(N=3000, flags=P.PKM_F_FP32), 16, per) == ws(d, 16, per)
    # the global sort falls back to the per-chunk steps when (chunks x K) overflows 31 bits
    big = dict(C1=1024, C2=1024, flags=P.PKM_F_FP32)
    glob = P.PKM_FW_SORT_GLOBAL
    assert ws(_dims(N=3000, **big), 1, glob) == ws(_dims(N=3000, **big), 1, per)
    assert ws(_dims(N=2000, **big), 1, glob) > ws(_dims(N=2000, **big), 1, per)
    assert ws(d, 0) == 0

    def call(dd=d, chunk=16, lr=0.5, mode=0, targets=FAKE, ws=FAKE, wsb=need, values=FAKE):
        return L.pkm_fastweight_chunks(ctypes.byref(dd.c()), chunk, lr, mode, FAKE, FAKE, FAKE,
                                       FAKE, values, targets, FAKE, ws, wsb, None)

    assert call(dd=_dims()) == P.PKM_ERR_UNSUPPORTED              # bf16 tables
    # bf16 inputs beside an fp32 table pass validation (then the workspace check)
    assert call(dd=_dims(flags=P.PKM_F_VALUES_FP32), ws=None) == P.PKM_ERR_WORKSPACE
    assert call(chunk=0) == P.PKM_ERR_INVALID_ARG
    assert call(lr=float("nan")) == P.PKM_ERR_INVALID_ARG
    assert call(mode=0x8) == P.PKM_ERR_INVALID_ARG
    assert call(targets=None) == P.PKM_ERR_INVALID_ARG             # explicit targets needed
    assert call(dd=_dims(d_v=72, flags=P.PKM_F_FP32), mode=P.PKM_FW_LOOKAHEAD,
                targets=None) == P.PKM_ERR_INVALID_ARG             # lookahead needs d_in == d_v
    assert call(values=FAKE + 4) == P.PKM_ERR_INVALID_ARG
    assert call(ws=None) == P.PKM_ERR_WORKSPACE
    assert call(wsb=need - 1) == P.PKM_ERR_WORKSPACE
    assert call(dd=_dims(N=0, flags=P.PKM_F_FP32), ws=None, wsb=0) == P.PKM_OK
    # the write step alone
    S = ctypes.byref(P._saved_c({f: FAKE for f in P.SAVED_FIELDS}))
    nb = P.pkm_workspace_bytes(d, P.PKM_BWD)
    assert L.pkm_value_sgd(ctypes.byref(_dims().c()), 0.5, FAKE, S, FAKE, FAKE, nb,
                           None) == P.PKM_ERR_UNSUPPORTED
    assert L.pkm_value_sgd(ctypes.byref(d.c()), float("inf"), FAKE, S, FAKE, FAKE, nb,
                           None) == P.PKM_ERR_INVALID_ARG
    assert L.pkm_value_sgd(ctypes.byref(d.c()), 0.5, FAKE, S, None, FAKE, nb,
                           None) == P.PKM_ERR_INVALID_ARG
    assert L.pkm_value_sgd(ctypes.byref(d.c()), 0.5, FAKE, S, FAKE, FAKE, nb - 1,
                           None) == P.PKM_ERR_WORKSPACE


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.reload(P)
    try:
        mod._lib = None
        with pytest.raises(ImportError):
            mod.load(str(tmp_path / "missing.so"))
    finally:
        importlib.reload(P)


def test_training_batch_norm_validation(lib):
    L = P.load()
    d = _dims(flags=P.PKM_F_BN_TRAIN)
    saved = {f: FAKE for f in P.SAVED_FIELDS}
    for missing in ("qhat", "bn_batch"):
        s = dict(saved, **{missing: None})
        rc = L.pkm_forward(ctypes.byref(d.c()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                           ctypes.byref(P._saved_c(s)), None, 0, None)
        assert rc == P.PKM_ERR_INVALID_ARG, missing
    upd = lambda dd, m: L.pkm_bn_running_update(ctypes.byref(dd.c()), FAKE, FAKE, m, None)
    assert upd(_dims(N=1), 0.1) == P.PKM_ERR_INVALID_ARG        # unbiased variance needs N >= 2
    assert upd(d, 1.5) == P.PKM_ERR_INVALID_ARG
    fw = _dims(flags=P.PKM_F_BN_TRAIN | P.PKM_F_FP32)
    rc = L.pkm_fastweight_chunks(ctypes.byref(fw.c()), 16, 0.5, 0, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, 1 << 30, None)
    assert rc == P.PKM_ERR_INVALID_ARG                          # the loop's BatchNorm is eval


def test_training_pieces_validation(lib):
    L = P.load()
    d = _dims()
    d32 = _dims(flags=P.PKM_F_VALUES_FP32)
    S = ctypes.byref(P._saved_c({f: FAKE for f in P.SAVED_FIELDS}))
    nb = P.pkm_workspace_bytes(d, P.PKM_BWD)
    # compact value gradient
    rows = lambda **kw: L.pkm_value_grad_rows(
        ctypes.byref(kw.get("d", d).c()), FAKE, S, FAKE, kw.get("dw", None), kw.get("ro", FAKE),
        kw.get("dvr", FAKE), kw.get("nr", FAKE), FAKE, kw.get("nb", nb), None)
    assert rows(ro=None) == P.PKM_ERR_INVALID_ARG
    assert rows(nr=None) == P.PKM_ERR_INVALID_ARG
    assert rows(dvr=FAKE + 4) == P.PKM_ERR_INVALID_ARG
    assert rows(nb=nb - 1) == P.PKM_ERR_WORKSPACE
    assert rows(d=_dims(N=0), ro=None) == P.PKM_OK
    # lazy Adam
    adam = lambda **kw: L.pkm_value_adam(
        ctypes.byref(kw.get("d", d32).c()), 0.01, kw.get("b1", 0.9), kw.get("b2", 0.99),
        kw.get("eps", 1e-8), kw.get("step", 1), FAKE, FAKE, kw.get("v", FAKE), S, FAKE, FAKE,
        nb, None)
    assert adam(d=d) == P.PKM_ERR_UNSUPPORTED          # bf16 table
    assert adam(b1=1.0) == P.PKM_ERR_INVALID_ARG
    assert adam(b2=-0.1) == P.PKM_ERR_INVALID_ARG
    assert adam(eps=0.0) == P.PKM_ERR_INVALID_ARG
    assert adam(step=0) == P.PKM_ERR_INVALID_ARG
    assert adam(v=None) == P.PKM_ERR_INVALID_ARG
    # hit counts
    hits = lambda **kw: L.pkm_hit_counts(ctypes.byref(kw.get("d", d).c()), kw.get("idx", FAKE),
                                         kw.get("slot", FAKE), kw.get("sub", FAKE), None)
    assert hits(idx=None) == P.PKM_ERR_INVALID_ARG
    assert hits(slot=FAKE + 2) == P.PKM_ERR_INVALID_ARG
    assert hits(idx=None, slot=None, sub=None) == P.PKM_OK    # nothing asked


def test_all_k2_sizes(lib):
    """The all-k^2 variant keeps k*k selections per head: idx and w grow, the per-half
    lists do not."""
    d, d2 = _dims(), _dims(flags=P.PKM_F_ALL_K2)
    assert P.pkm_saved_bytes(d2, "idx") == d.k * P.pkm_saved_bytes(d, "idx")
    assert P.pkm_saved_bytes(d2, "w") == d.k * P.pkm_saved_bytes(d, "w")
    assert P.pkm_saved_bytes(d2, "sub_i") == P.pkm_saved_bytes(d, "sub_i")
    assert P.pkm_workspace_bytes(d2, P.PKM_BWD) > P.pkm_workspace_bytes(d, P.PKM_BWD)
    big = _dims(N=1 << 18, k=32, h=4, flags=P.PKM_F_ALL_K2)       # 2^18*4*1024*2 = 2^31
    assert _fwd(big) == P.PKM_ERR_UNSUPPORTED


def test_shard_validation(lib):
    """Row-sharded entry points: shard count, shard size, sizes of what was received and
    the workspace are checked on the host."""
    L = P.load()
    d = _dims()                                    # 32 x 32 = 1024 rows
    c = ctypes.byref(d.c())
    nb = P.pkm_shard_workspace_bytes(d, 4, P.PKM_SHARD_ROUTE)
    assert nb >= 3 * 4 * 4 * d.N                   # three [G][N] int32 tables
    assert P.pkm_shard_workspace_bytes(d, 0, P.PKM_SHARD_ROUTE) == 0
    assert P.pkm_shard_workspace_bytes(d, P.PKM_MAX_SHARDS + 1, P.PKM_SHARD_ROUTE) == 0
    assert P.pkm_shard_workspace_bytes(d, 4, 7) == 0
    own = P.pkm_shard_workspace_bytes(d, 4, P.PKM_SHARD_OWNER, 10)
    assert P.pkm_shard_workspace_bytes(d, 4, P.PKM_SHARD_OWNER, 1000) > own > 0
    route = lambda **kw: L.pkm_shard_route(
        ctypes.byref(kw.get("d", d).c()), kw.get("G", 4), kw.get("R", 256), FAKE, FAKE,
        kw.get("counts", FAKE), FAKE, kw.get("send", FAKE), FAKE, FAKE, kw.get("nb", nb), None)
    assert route(G=0) == P.PKM_ERR_INVALID_ARG
    assert route(G=P.PKM_MAX_SHARDS + 1) == P.PKM_ERR_INVALID_ARG
    assert route(R=255) == P.PKM_ERR_INVALID_ARG   # 4 shards of 255 rows miss the last rows
    assert route(R=0) == P.PKM_ERR_INVALID_ARG
    assert route(counts=None) == P.PKM_ERR_INVALID_ARG
    assert route(send=FAKE + 4) == P.PKM_ERR_INVALID_ARG
    assert route(nb=nb - 1) == P.PKM_ERR_WORKSPACE
    assert route(d=_dims(N=1 << 28), G=8, nb=1 << 40) == P.PKM_ERR_UNSUPPORTED   # G*N >= 2^31
    bag = lambda **kw: L.pkm_shard_bag(c, 4, kw.get("rows", 256), FAKE, kw.get("nt", 10),
                                       kw.get("ns", 4), FAKE, FAKE, kw.get("part", FAKE), FAKE,
                                       kw.get("nb", own), None)
    assert bag(ns=11) == P.PKM_ERR_INVALID_ARG     # more segments than triples
    assert bag(ns=0) == P.PKM_ERR_INVALID_ARG      # triples without a segment
    assert bag(rows=0) == P.PKM_ERR_INVALID_ARG
    assert bag(part=None) == P.PKM_ERR_INVALID_ARG
    assert bag(nb=own - 1) == P.PKM_ERR_WORKSPACE
    assert bag(nt=0, ns=0) == P.PKM_OK             # nothing received
    vg = lambda **kw: L.pkm_shard_value_grad(c, 4, 256, FAKE, kw.get("nt", 10), kw.get("ns", 4),
                                             FAKE, FAKE, FAKE, kw.get("dv", FAKE), FAKE, FAKE,
                                             kw.get("nb", own), None)
    assert vg(ns=11) == P.PKM_ERR_INVALID_ARG
    assert vg(dv=None) == P.PKM_ERR_INVALID_ARG
    assert vg(nb=own - 1) == P.PKM_ERR_WORKSPACE
    assert vg(nt=0, ns=0) == P.PKM_OK
    assert L.pkm_shard_combine(c, 4, FAKE, FAKE, -1, FAKE, None) == P.PKM_ERR_INVALID_ARG
    assert L.pkm_shard_combine(c, 4, None, FAKE, 10, FAKE, None) == P.PKM_ERR_INVALID_ARG
    assert L.pkm_shard_gather_dy(c, 4, FAKE, None, FAKE, 10, None) == P.PKM_ERR_INVALID_ARG
    assert L.pkm_shard_gather_dy(c, 4, None, None, None, 0, None) == P.PKM_OK
    assert L.pkm_shard_scatter_dw(c, None, FAKE, FAKE, None) == P.PKM_ERR_INVALID_ARG
