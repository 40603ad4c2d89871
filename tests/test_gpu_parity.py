"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle."""
import numpy as np
import pytest
import torch

from oracle import pkm_oracle as O
from product_key_memory_pkm_b200 import pkm as P
from product_key_memory_pkm_b200.inputs import (FULL_K1024, FWD_K512, TINY_FP32, PKMConfig,
                                                make_inputs)
from tests import parity as H

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from product_key_memory_pkm_b200 import build as B
    B.build()


def _cfg(**kw):
    base = dict(name="case", N=300, d_in=128, h=4, dk=128, C1=64, C2=48, k=16, d_v=200,
                dtype="bf16", score_scale=0.5)
    base.update(kw)
    return PKMConfig(**base)


CASES = {
    "tiny_fp32": TINY_FP32,
    "tiny_bf16": TINY_FP32.with_(name="tiny_bf16", dtype="bf16"),
    "ragged_multihead_bf16": _cfg(),
    "ragged_multihead_fp32": _cfg(name="r32", dtype="f32", dk=40),
    "k_equals_C": _cfg(N=100, h=2, C1=32, C2=32, k=32, d_v=64),
    "simt_shape_dk64": _cfg(N=200, dk=64),
    "many_chunks_C700": _cfg(N=260, h=2, C1=700, C2=300, k=32, d_v=64, d_in=256),
    "k1": _cfg(N=77, k=1, h=2),
    "one_token": _cfg(N=1),
    "two_tokens_k12": _cfg(N=2, h=2, C1=70, C2=65, k=12, d_v=40),
    "duplicate_heavy": _cfg(N=512, d_in=64, h=1, C1=64, C2=64, k=8, d_v=128, clustered=8),
    "unequal_C_wide_dv": _cfg(N=130, h=1, dk=128, C1=96, C2=40, k=24, d_v=2056),
    "fp32_values_bf16_rest": _cfg(N=211, value_dtype="f32", d_v=136),
    # few tokens (N <= 16): CUDA-core query and cluster-split scoring and bag
    "few_tokens_unequal_C_k8": _cfg(N=13, h=2, dk=64, C1=96, C2=40, k=8),
    "few_tokens_k32_small_C": _cfg(N=16, h=3, k=32, C1=40, C2=33, d_v=72),
    "split_bag_37_tokens": _cfg(N=37, h=2, dk=64, C1=96, C2=40, k=8),
    "two_tokens_k16": _cfg(N=2, h=3, dk=64, C1=96, C2=40, k=16),
    # k above 32: two candidate rows per lane, 64-key scoring lists
    "k48": _cfg(N=150, h=2, C1=96, C2=72, k=48),
    "k64": _cfg(N=150, h=2, C1=128, C2=64, k=64, d_v=136),
    "k64_fp32": _cfg(name="k64f", N=90, h=2, dtype="f32", dk=40, C1=80, C2=64, k=64),
    "few_tokens_k64": _cfg(N=5, h=2, dk=64, C1=96, C2=70, k=64),
}


def _full_check(cfg, seed=0, flags=0, inp=None, q_bf16=False, bn_train=False, idw=False,
                fused=False):
    if inp is None:
        inp = make_inputs(cfg, seed=seed, random_bn=True)
    dev = H.to_dev(inp, cfg)
    dims, saved, y = H.gpu_forward(cfg, dev, flags=flags, fused=fused)
    of = O.forward(inp, cfg, q_bf16=q_bf16, bn_train=bn_train, idw=idw)
    if bn_train:   # the batch statistics the forward recorded
        H.assert_rows(saved["bn_batch"].cpu().numpy(), np.stack(of["bn_batch"]), "bn_batch")
    ranked = H.oracle_gaps(of, cfg)
    idx = saved["idx"].cpu().numpy()
    clean = H.check_indices(idx, of, cfg, ranked)
    yg = y.cpu().numpy()
    H.assert_rows(yg[clean], of["y"][clean], "y")
    for t in np.nonzero(~clean)[0]:
        H.assert_rows(yg[t:t + 1], H.oracle_bag_at(of, cfg, idx, t, inp["values"])[None], "y tie")
    # softmax weights of clean heads
    wg = H.align_to(idx[clean], of["idx"][clean], saved["w"].cpu().numpy()[clean])
    H.assert_rows(wg.reshape(-1, cfg.k), of["w"][clean].reshape(-1, cfg.k), "w")
    # backward with dy masked to the clean tokens
    dy = inp["dy"] * clean[:, None]
    g = H.gpu_backward(cfg, dims, dev, saved, torch.from_numpy(dy).cuda())
    ob = O.backward(inp, cfg, of, dy)
    H.assert_rows(g["dx"].cpu().numpy(), ob["dx"], "dx")
    H.assert_dwq(g["dWq"].cpu().numpy(), ob["dWq"], H.dwq_term_magnitude(inp, cfg, of, ob))
    H.assert_rows(g["dbn"].cpu().numpy(), np.stack([ob["dgamma"], ob["dbeta"]]), "dbn",
                  zero_rows=True)
    H.assert_rows(g["dsub"].cpu().numpy().reshape(-1, cfg.dk // 2),
                  ob["dsub"].reshape(-1, cfg.dk // 2), "dsub", zero_rows=True)
    dV = g["dV"].cpu().numpy()
    H.assert_rows(dV[ob["dV_rows"]], ob["dV_vals"], "dV")
    untouched = np.ones(cfg.K, dtype=bool)
    untouched[ob["dV_rows"]] = False
    assert not dV[untouched].any()
    dwg = H.align_to(idx[clean], of["idx"][clean], g["dw"].cpu().numpy()[clean])
    H.assert_rows(dwg.reshape(-1, cfg.k), ob["dw"][clean].reshape(-1, cfg.k), "dw")
    return clean


@pytest.mark.parametrize("name", list(CASES))
def test_end_to_end_parity(name):
    clean = _full_check(CASES[name])
    assert clean.mean() > 0.5      # most tokens have no near-tie head


def test_simt_flag_path_matches_oracle():
    _full_check(CASES["ragged_multihead_bf16"], flags=P.PKM_F_SIMT)


def _exact_query_inputs(cfg, seed):
    """x and Wq with few significant bits and an identity BatchNorm (var + eps = 1):
    every product and partial sum of q = x Wq^T is exact in fp32, so the device and the
    oracle hold the same q and round it to bf16 the same way."""
    inp = make_inputs(cfg, seed=seed)
    rng = np.random.default_rng(seed + 100)
    inp["x"] = (rng.integers(-8, 9, (cfg.N, cfg.d_in)) / 8).astype(np.float32)
    inp["Wq"] = (rng.integers(-64, 65, (cfg.h * cfg.dk, cfg.d_in)) / 64).astype(np.float32)
    eps = 2.0 ** -10
    hq = cfg.h * cfg.dk
    inp["bn"] = np.stack([np.zeros(hq), np.full(hq, 1 - eps), np.ones(hq),
                          np.zeros(hq)]).astype(np.float32)
    return inp, cfg.with_(bn_eps=eps)


@pytest.mark.parametrize("simt,n", [(False, 300), (True, 300), (False, 12)])
def test_single_pass_bf16_q_scoring(simt, n):
    """PKM_F_BF16_Q: scores from q rounded to bf16 (one tensor-core pass, the CUDA-core
    kernel, or the few-token kernel dropping the lo plane), the sub-key gradient from the
    same rounded q, the query gradient straight through -- against the oracle's bf16-q
    variant."""
    cfg = _cfg(N=n)
    inp, cfg = _exact_query_inputs(cfg, 5)
    # the variant is visible: its scores move well beyond the index tolerance
    f0, f1 = O.forward(inp, cfg), O.forward(inp, cfg, q_bf16=True)
    assert np.abs(f1["s1"] - f0["s1"]).max() > 1e-3 * np.abs(f0["s1"]).max()
    flags = P.PKM_F_BF16_Q | (P.PKM_F_SIMT if simt else 0)
    clean = _full_check(cfg, flags=flags, inp=inp, q_bf16=True)
    assert clean.mean() > 0.5


@pytest.mark.parametrize("case", ["tensor_core", "simt", "fp32", "few_tokens"])
def test_training_mode_batch_norm(case):
    """PKM_F_BN_TRAIN: the query normalised with the batch's statistics, the backward
    through them (every token's dx depends on all tokens), and the running-statistics
    update -- against the oracle's training-mode BatchNorm."""
    cfg, flags = {
        "tensor_core": (_cfg(N=300), 0),
        "simt": (_cfg(N=300), P.PKM_F_SIMT),
        "fp32": (_cfg(N=200, dtype="f32", dk=40), 0),
        "few_tokens": (_cfg(N=12), 0),
    }[case]
    inp = make_inputs(cfg, seed=12, random_bn=True)
    clean = _full_check(cfg, flags=flags | P.PKM_F_BN_TRAIN, inp=inp, bn_train=True)
    assert clean.mean() > 0.5
    # running statistics: fold the batch into bn
    dims = P.Dims.from_config(cfg, flags=flags | P.PKM_F_BN_TRAIN)
    dev = H.to_dev(inp, cfg)
    saved = P.alloc_saved(dims)
    y = torch.empty(cfg.N, cfg.d_v, device="cuda")
    P.pkm_forward(dims, dev["x"], dev["Wq"], dev["bn"], dev["subkeys"], dev["values"], y, saved)
    bn = dev["bn"].clone()
    P.pkm_bn_running_update(dims, bn, saved["bn_batch"], 0.1)
    assert P.pkm_check_status() == P.PKM_OK
    of = O.forward(inp, cfg, bn_train=True)
    want = O.running_stats_update(inp["bn"], *of["bn_batch"], cfg.N, 0.1)
    H.assert_rows(bn.cpu().numpy(), want, "running statistics")


@pytest.mark.parametrize("k", [16, 32, 48, 64])
def test_stagewise_scores_given_oracle_query(k):
    """F2 alone: fed the oracle's q (as its hi/lo split), the per-half lists match the
    oracle's per-half top-k computed from the same q."""
    cfg = _cfg(N=257, C1=96, C2=72, k=k)
    inp = make_inputs(cfg, seed=3, random_bn=True)
    of = O.forward(inp, cfg)
    q32 = torch.from_numpy(of["q"].astype(np.float32))
    hi = q32.to(torch.bfloat16)
    lo = (q32 - hi.float()).to(torch.bfloat16)
    qrep = (hi.double() + lo.double()).numpy()
    s1, s2 = O.subkey_scores(qrep, inp["subkeys"], cfg.h, cfg.dk, cfg.C1)
    dims = P.Dims.from_config(cfg)
    saved = P.alloc_saved(dims)
    saved["q"].copy_(torch.stack([hi, lo]).cuda())
    sub = torch.from_numpy(inp["subkeys"]).to(torch.bfloat16).cuda()
    P.pkm_subkey_scores(dims, sub, saved)
    assert P.pkm_check_status() == P.PKM_OK
    gi = saved["sub_i"].cpu().numpy()
    gs = saved["sub_s"].cpu().numpy()
    for t in range(cfg.N):
        for hh in range(cfg.h):
            for half, s in ((0, s1[t, hh]), (1, s2[t, hh])):
                ii, vv = O.half_topk(s, cfg.k + 1)
                tol = H.GAP_REL * max(abs(vv[cfg.k - 1]), 1e-2)
                if vv[cfg.k - 1] - vv[cfg.k] > tol:
                    assert set(gi[t, hh, half].tolist()) == set(ii[:cfg.k].tolist())
                np.testing.assert_allclose(gs[t, hh, half], s[gi[t, hh, half]], rtol=1e-5,
                                           atol=1e-5)


@pytest.mark.parametrize("k", [32, 48, 64])
def test_stagewise_candidates_given_oracle_lists(k):
    """F3 alone: fed per-half lists (fp32), the winners and weights match the oracle's
    product-key combine of the same lists."""
    cfg = _cfg(N=500 if k == 32 else 200, k=k, C1=80, C2=72)   # k + 1 <= C for the gaps
    rng = np.random.default_rng(5)
    N, h, k = cfg.N, cfg.h, cfg.k
    s1 = rng.standard_normal((N, h, cfg.C1)).astype(np.float32)
    s2 = rng.standard_normal((N, h, cfg.C2)).astype(np.float32)
    s1[:7] = np.round(s1[:7])      # exact ties in a few tokens
    s2[:7] = np.round(s2[:7])
    sub_i = np.zeros((N, h, 2, k), dtype=np.int32)
    sub_s = np.zeros((N, h, 2, k), dtype=np.float32)
    for t in range(N):
        for hh in range(h):
            for half, s in ((0, s1[t, hh].astype(np.float64)), (1, s2[t, hh].astype(np.float64))):
                ii, vv = O.half_topk(s, k)
                sub_i[t, hh, half], sub_s[t, hh, half] = ii, vv
    dims = P.Dims.from_config(cfg)
    saved = P.alloc_saved(dims)
    saved["sub_s"].copy_(torch.from_numpy(sub_s))
    saved["sub_i"].copy_(torch.from_numpy(sub_i))
    P.pkm_candidate_topk(dims, saved)
    assert P.pkm_check_status() == P.PKM_OK
    gidx = saved["idx"].cpu().numpy()
    gw = saved["w"].cpu().numpy()
    for t in range(N):
        for hh in range(h):
            a, b = s1[t, hh].astype(np.float64), s2[t, hh].astype(np.float64)
            ii, jj = O.product_key_topk(a, b, k + 1)
            S = a[ii] + b[jj]
            tol = H.GAP_REL * max(abs(S[k - 1]), 1e-2)
            if S[k - 1] - S[k] > tol:
                assert set(gidx[t, hh].tolist()) == set((ii[:k] * cfg.C2 + jj[:k]).tolist())
                w = O.softmax(cfg.score_scale * S[:k])
                np.testing.assert_allclose(gw[t, hh], w, rtol=2e-3, atol=1e-6)
            if t < 7:
                # integer scores: fp32 sums are exact, so the order is the oracle's order
                assert gidx[t, hh].tolist() == (ii[:k] * cfg.C2 + jj[:k]).tolist()


def test_stagewise_gather_given_oracle_selection():
    cfg = _cfg(N=333, d_v=1032)
    inp = make_inputs(cfg, seed=6, with_dy=False)
    of = O.forward(inp, cfg)
    dims = P.Dims.from_config(cfg)
    V = torch.from_numpy(inp["values"]).to(torch.bfloat16).cuda()
    idx = torch.from_numpy(of["idx"].astype(np.int32)).cuda()
    w32 = of["w"].astype(np.float32)
    y = torch.empty(cfg.N, cfg.d_v, device="cuda")
    P.pkm_gather_bag(dims, V, idx, torch.from_numpy(w32).cuda(), y)
    assert P.pkm_check_status() == P.PKM_OK
    want = O.bag(w32.astype(np.float64), of["idx"], inp["values"])
    H.assert_rows(y.cpu().numpy(), want, "y", tol=1e-5)


def test_value_gradient_is_deterministic_under_duplicates():
    cfg = CASES["duplicate_heavy"]
    inp = make_inputs(cfg, seed=2)
    dev = H.to_dev(inp, cfg)
    dims, saved, _ = H.gpu_forward(cfg, dev)
    idx = saved["idx"].cpu().numpy().ravel()
    assert np.unique(idx).size < 0.5 * idx.size      # the clustered recipe duplicates rows
    dy = torch.from_numpy(inp["dy"]).cuda()
    g1 = H.gpu_backward(cfg, dims, dev, saved, dy)
    g2 = H.gpu_backward(cfg, dims, dev, saved, dy)
    for k in ("dV", "dsub", "dWq", "dx", "dbn", "dw"):
        assert torch.equal(g1[k], g2[k]), k


@pytest.mark.parametrize("case", ["duplicate_heavy", "ragged_multihead_bf16"])
def test_value_stage_in_two_parts_equals_the_whole(case):
    """pkm_value_sort then pkm_value_rows (another stream's work in between, the workspace
    left alone) gives pkm_value_grad's dV and dw bit for bit."""
    cfg = CASES[case]
    inp = make_inputs(cfg, seed=4)
    dev = H.to_dev(inp, cfg)
    dims, saved, _ = H.gpu_forward(cfg, dev)
    dy = torch.from_numpy(inp["dy"]).cuda()
    V = dev["values"]
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    dV1 = torch.zeros(cfg.K, cfg.d_v, device="cuda")
    dw1 = torch.empty(cfg.N, cfg.h, cfg.k, device="cuda")
    P.pkm_value_grad(dims, V, saved, dy, dw1, dvalues=dV1, workspace=ws)
    dV2 = torch.zeros_like(dV1)
    dw2 = torch.full_like(dw1, float("nan"))
    ws.fill_(0xA5)  # stale contents must not matter to the sort
    P.pkm_value_sort(dims, saved, workspace=ws)
    torch.cuda.synchronize()
    P.pkm_value_rows(dims, V, dy, dw2, dvalues=dV2, workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    assert torch.equal(dV1, dV2)
    assert torch.equal(dw1, dw2)


def test_gradients_accumulate_into_caller_buffers():
    cfg = CASES["tiny_bf16"]
    inp = make_inputs(cfg, seed=1)
    dev = H.to_dev(inp, cfg)
    dims, saved, _ = H.gpu_forward(cfg, dev)
    dy = torch.from_numpy(inp["dy"]).cuda()
    g1 = H.gpu_backward(cfg, dims, dev, saved, dy)
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    acc = {k: v.clone() for k, v in g1.items()}
    P.pkm_backward(dims, dev["x"], dev["Wq"], dev["bn"], dev["subkeys"], dev["values"], saved, dy,
                   dx=acc["dx"], dWq=acc["dWq"], dbn=acc["dbn"], dsubkeys=acc["dsub"],
                   dvalues=acc["dV"], dw_out=acc["dw"], workspace=ws)
    torch.cuda.synchronize()
    for k in ("dWq", "dbn", "dsub", "dV"):
        torch.testing.assert_close(acc[k], 2 * g1[k], rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(acc["dx"], g1["dx"], rtol=0, atol=0)      # overwritten


def test_zero_tokens_noop_on_device():
    cfg = _cfg(N=0)
    dims = P.Dims.from_config(cfg)
    y = torch.full((1, cfg.d_v), 7.0, device="cuda")
    saved = P.alloc_saved(P.Dims.from_config(cfg.with_(N=1)))
    dummy = torch.zeros(1024, device="cuda")
    P.pkm_forward(dims, dummy, dummy, dummy, dummy, dummy, y, saved)
    assert P.pkm_check_status() == P.PKM_OK
    assert torch.all(y == 7.0)


def _sampled_full_size(cfg, n_sample, seed=0, backward=True, fused=False):
    inp = make_inputs(cfg, seed=seed, random_bn=False)
    dev = H.to_dev(inp, cfg)
    dims, saved, y = H.gpu_forward(cfg, dev, fused=fused)
    rng = np.random.default_rng(123)
    n_sample = min(n_sample, cfg.N)
    sample = np.sort(rng.choice(cfg.N, size=n_sample, replace=False))
    sample[0], sample[-1] = 0, cfg.N - 1
    sub_inp = dict(inp, x=inp["x"][sample], dy=inp["dy"][sample])
    # the product-key search selects exactly what brute force does (pinned on the CPU)
    # at a fraction of its cost over a million keys per head
    of = O.forward(sub_inp, cfg, select="product")
    ranked = H.oracle_gaps(of, cfg, select="product")
    idx = saved["idx"][torch.from_numpy(sample).cuda()].cpu().numpy()
    clean = H.check_indices(idx, of, cfg, ranked)
    yg = y[torch.from_numpy(sample).cuda()].cpu().numpy()
    H.assert_rows(yg[clean], of["y"][clean], "y")
    if not backward:
        return
    dy_s = sub_inp["dy"] * clean[:, None]
    dy = torch.zeros(cfg.N, cfg.d_v, device="cuda")
    dy[torch.from_numpy(sample).cuda()] = torch.from_numpy(dy_s).cuda()
    del dev["dy"]
    g = H.gpu_backward(cfg, dims, dev, saved, dy)
    ob = O.backward(sub_inp, cfg, of, dy_s)
    dx = g["dx"]
    H.assert_rows(dx[torch.from_numpy(sample).cuda()].cpu().numpy(), ob["dx"], "dx")
    mask = torch.ones(cfg.N, dtype=torch.bool, device="cuda")
    mask[torch.from_numpy(sample).cuda()] = False
    assert not torch.any(dx[mask])
    H.assert_dwq(g["dWq"].cpu().numpy(), ob["dWq"], H.dwq_term_magnitude(sub_inp, cfg, of, ob))
    H.assert_rows(g["dsub"].cpu().numpy().reshape(-1, cfg.dk // 2),
                  ob["dsub"].reshape(-1, cfg.dk // 2), "dsub", zero_rows=True)
    H.assert_rows(g["dbn"].cpu().numpy(), np.stack([ob["dgamma"], ob["dbeta"]]), "dbn",
                  zero_rows=True)
    rows = torch.from_numpy(ob["dV_rows"]).cuda()
    H.assert_rows(g["dV"][rows].cpu().numpy(), ob["dV_vals"], "dV")
    assert int((g["dV"].abs().sum(1) > 0).sum()) <= len(ob["dV_rows"])


def test_forward_K512_full_size_sampled():
    _sampled_full_size(FWD_K512, 256, backward=False)


def test_fwd_bwd_K1024_full_size_sampled():
    _sampled_full_size(FULL_K1024, 128)


def test_fwd_bwd_K512_sampled():
    """4096 tokens, |K| = 512^2, d_in = 1024: the backward at the second workload's size,
    sampled tokens against the oracle."""
    _sampled_full_size(FWD_K512, 256)


def test_bounded_wait_expires_with_status_and_context_survives():
    """A wait on a barrier that nothing completes gives up after its budget, records
    PKM_ERR_DEVICE_TIMEOUT, and the next call on the same context works."""
    assert P.pkm_check_status() == P.PKM_OK
    P.pkm_selftest_wait_timeout(2_000_000)          # ~1 ms at B200 clocks
    assert P.pkm_check_status() == P.PKM_ERR_DEVICE_TIMEOUT
    assert P.pkm_check_status() == P.PKM_OK         # read-and-clear
    _full_check(CASES["tiny_bf16"])                 # the context is still usable


@pytest.mark.parametrize("n_tok", [1, 8, 64])
def test_decode_shaped_calls_on_the_full_table(n_tok):
    """Decode-sized batches (N = 1, 8, 64 tokens) against the full 1024^2 x 1600 bf16
    table: forward and backward parity for every token."""
    _sampled_full_size(FULL_K1024.with_(name=f"decode_N{n_tok}", N=n_tok), n_tok)


FUSED_CASES = {
    "one_token": _cfg(N=1),
    "two_tokens_k12": _cfg(N=2, h=2, C1=70, C2=65, k=12, d_v=40),
    "five_tokens_unequal_C_ragged": _cfg(N=5, h=3, dk=64, C1=96, C2=40, k=8, d_v=72),
    "sixteen_tokens_k32": _cfg(N=16, h=2, C1=200, C2=130, k=32, d_v=264),
    "k_equals_C": _cfg(N=3, h=2, C1=32, C2=32, k=32, d_v=64),
    "k1_single_pass_q": _cfg(N=7, h=2, k=1),
    # 64 block lists in the first half (the most the merge takes: six levels), a ragged last
    # block, and an odd list count in the second half
    "C4096_six_merge_levels": _cfg(N=2, h=1, dk=64, C1=4096, C2=200, k=8, d_v=16),
    "sixteen_tokens_wide_input": _cfg(N=16, d_in=2048, h=2, dk=256, C1=130, C2=96, k=16,
                                      d_v=40),
}


@pytest.mark.parametrize("name", list(FUSED_CASES))
def test_fused_decode_forward_and_its_saved_state(name):
    """The few-token forward as one kernel: outputs against the oracle, and the saved
    state it writes (q planes, per-half lists, selections, weights) carries the
    backward to oracle parity."""
    cfg = FUSED_CASES[name]
    flags = P.PKM_F_BF16_Q if name.endswith("single_pass_q") else 0
    _full_check(cfg, flags=flags, q_bf16=bool(flags), fused=True)


def test_fused_decode_lists_match_the_separate_kernels():
    """Per-half lists and selections of the fused kernel against the separate-kernel path
    on the same inputs (same order wherever scores are separated)."""
    cfg = _cfg(N=9, h=4, C1=256, C2=192, k=32, d_v=128)
    inp = make_inputs(cfg, seed=8, random_bn=True)
    dev = H.to_dev(inp, cfg)
    _, sf, yf = H.gpu_forward(cfg, dev, fused=True)
    _, ss, ys = H.gpu_forward(cfg, dev)
    gap = (sf["sub_s"][..., :-1] - sf["sub_s"][..., 1:]).abs()
    tied = (gap < 1e-6).any(-1)
    agree = (sf["sub_i"] == ss["sub_i"]).all(-1)
    assert torch.all(agree | tied)
    torch.testing.assert_close(sf["sub_s"], ss["sub_s"], rtol=1e-5, atol=1e-5)
    same = (sf["idx"] == ss["idx"]).all(-1).all(-1)
    assert same.float().mean() > 0.9
    torch.testing.assert_close(yf[same], ys[same], rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("n_tok", [1, 8, 16])
def test_fused_decode_on_the_full_table(n_tok):
    """The fused decode kernel at the full 1024^2 x 1600 table: forward and backward
    parity for every token."""
    _sampled_full_size(FULL_K1024.with_(name=f"decode_fused_N{n_tok}", N=n_tok), n_tok,
                       fused=True)


def test_fused_decode_is_repeatable_bit_for_bit():
    """Two fused calls on the same inputs (different barrier slots) write identical outputs
    and saved state: every reduction runs in a fixed order."""
    cfg = _cfg(N=11, h=3, C1=200, C2=130, k=32, d_v=264)
    inp = make_inputs(cfg, seed=21, random_bn=True)
    dev = H.to_dev(inp, cfg)
    _, s1, y1 = H.gpu_forward(cfg, dev, fused=True)
    _, s2, y2 = H.gpu_forward(cfg, dev, fused=True)
    assert torch.equal(y1, y2)
    for f in ("q", "qhat", "sub_s", "sub_i", "idx", "w"):
        assert torch.equal(s1[f], s2[f]), f


def test_forward_k64_on_the_full_table_sampled():
    """k = 64 (the boundary's largest; the CUDA-core scorers keep 64-key lists) on the full
    1024^2 x 1600 table, 2048 tokens: sampled forward parity."""
    _sampled_full_size(FULL_K1024.with_(name="k64_full_table", N=2048, k=64), 128,
                       backward=False)


def test_fast_weight_chunk_shape_fp32_values_duplicates():
    """One 512-token-class chunk of the fast-weight workload (fp32 values, h = 1, k = 8,
    |K| = 1024^2, d = 1024, queries around 64 centres, so value rows repeat)."""
    from product_key_memory_pkm_b200.inputs import FASTWEIGHT
    cfg = FASTWEIGHT.with_(N=192)
    inp = make_inputs(cfg, seed=0)
    dev = H.to_dev(inp, cfg)
    dims, saved, y = H.gpu_forward(cfg, dev)
    idx = saved["idx"].cpu().numpy()
    assert np.unique(idx).size < idx.size      # clustered queries share value rows
    of = O.forward(inp, cfg)
    ranked = H.oracle_gaps(of, cfg)
    clean = H.check_indices(idx, of, cfg, ranked)
    H.assert_rows(y.cpu().numpy()[clean], of["y"][clean], "y")
    dy = inp["dy"] * clean[:, None]
    g = H.gpu_backward(cfg, dims, dev, saved, torch.from_numpy(dy).cuda(), want=("dV", "dw"))
    ob = O.backward(inp, cfg, of, dy)
    H.assert_rows(g["dV"].cpu().numpy()[ob["dV_rows"]], ob["dV_vals"], "dV")


@pytest.mark.parametrize("n", [200, 12])
def test_all_k2_variant(n):
    """PKM_F_ALL_K2: every candidate of top-k(s1) x top-k(s2) is kept and the softmax runs
    over all k^2 of them.  A head's candidate set is unique where both halves separate
    their k-th from their (k+1)-th sub-key by more than the tolerance; other tokens are
    left out of the output comparison and their upstream gradient is masked."""
    cfg = _cfg(N=n, h=2, k=8, C1=64, C2=48)
    inp = make_inputs(cfg, seed=13, random_bn=True)
    dev = H.to_dev(inp, cfg)
    dims, saved, y = H.gpu_forward(cfg, dev, flags=P.PKM_F_ALL_K2)
    of = O.forward(inp, cfg, all_k2=True)
    k, kk = cfg.k, cfg.k * cfg.k
    idx = saved["idx"].cpu().numpy()
    assert idx.shape == (cfg.N, cfg.h, kk)
    clean = np.ones(cfg.N, dtype=bool)
    for t in range(cfg.N):
        for hh in range(cfg.h):
            for s in (of["s1"][t, hh], of["s2"][t, hh]):
                r = np.sort(s)[::-1]
                if r[k - 1] - r[k] <= H.GAP_REL * max(abs(r[k - 1]), 1e-2):
                    clean[t] = False
            if clean[t]:
                assert set(idx[t, hh].tolist()) == set(of["idx"][t, hh].tolist()), (t, hh)
    assert clean.mean() > 0.5
    H.assert_rows(y.cpu().numpy()[clean], of["y"][clean], "y")
    wg = H.align_to(idx[clean], of["idx"][clean], saved["w"].cpu().numpy()[clean])
    H.assert_rows(wg.reshape(-1, kk), of["w"][clean].reshape(-1, kk), "w")
    dy = inp["dy"] * clean[:, None]
    z = lambda *s: torch.zeros(*s, dtype=torch.float32, device="cuda")
    g = dict(dx=z(cfg.N, cfg.d_in), dWq=z(cfg.h * cfg.dk, cfg.d_in), dbn=z(2, cfg.h * cfg.dk),
             dsub=z(cfg.h, cfg.C1 + cfg.C2, cfg.dk // 2), dV=z(cfg.K, cfg.d_v),
             dw=z(cfg.N, cfg.h, kk))
    ws = P.alloc_workspace(dims, P.PKM_BWD)
    P.pkm_backward(dims, dev["x"], dev["Wq"], dev["bn"], dev["subkeys"], dev["values"], saved,
                   torch.from_numpy(dy).cuda(), dx=g["dx"], dWq=g["dWq"], dbn=g["dbn"],
                   dsubkeys=g["dsub"], dvalues=g["dV"], dw_out=g["dw"], workspace=ws)
    assert P.pkm_check_status() == P.PKM_OK
    ob = O.backward(inp, cfg, of, dy)
    H.assert_rows(g["dx"].cpu().numpy(), ob["dx"], "dx")
    H.assert_dwq(g["dWq"].cpu().numpy(), ob["dWq"], H.dwq_term_magnitude(inp, cfg, of, ob))
    H.assert_rows(g["dbn"].cpu().numpy(), np.stack([ob["dgamma"], ob["dbeta"]]), "dbn",
                  zero_rows=True)
    H.assert_rows(g["dsub"].cpu().numpy().reshape(-1, cfg.dk // 2),
                  ob["dsub"].reshape(-1, cfg.dk // 2), "dsub", zero_rows=True)
    H.assert_rows(g["dV"].cpu().numpy()[ob["dV_rows"]], ob["dV_vals"], "dV")
    dwg = H.align_to(idx[clean], of["idx"][clean], g["dw"].cpu().numpy()[clean])
    H.assert_rows(dwg.reshape(-1, kk), ob["dw"][clean].reshape(-1, kk), "dw")


@pytest.mark.parametrize("case", ["bf16", "fp32", "few_tokens"])
def test_inverse_distance_scores(case):
    """PKM_F_IDW: sub-key scores -1/2 log(||q_half - c||^2 + eps), on the CUDA-core and the
    few-token kernels, and their backward (u = g / d^2 corrections) -- against the oracle's
    inverse-distance scorer.  Sub-keys ~ N(0, 1), at the queries' scale, so that distances
    differ across keys."""
    cfg = {"bf16": _cfg(N=200, h=2, dk=64, C1=64, C2=48, k=16, d_v=64),
           "fp32": _cfg(N=200, h=2, dk=64, C1=64, C2=48, k=16, d_v=64, dtype="f32"),
           "few_tokens": _cfg(N=14, h=2, dk=64, C1=64, C2=48, k=16, d_v=64)}[case]
    inp = make_inputs(cfg, seed=14, random_bn=True)
    rng = np.random.default_rng(99)
    sub = rng.standard_normal(inp["subkeys"].shape).astype(np.float32)
    if cfg.dtype == "bf16":
        sub = torch.from_numpy(sub).bfloat16().float().numpy()
    inp["subkeys"] = sub
    clean = _full_check(cfg, flags=P.PKM_F_IDW, inp=inp, idw=True)
    assert clean.mean() > 0.5
