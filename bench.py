"""Benchmark of the product-key memory layer (forward + sparse backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--no-e2e] [--no-cpu-baseline] [--stage S] [--decode]

Default: the full-scale forward + backward workload (16384 tokens, |K| = 1024², h = 4,
k = 32, d = 1600).  --workload fwpkm_chunk512_K1024x1024_h1_k8_d1024 times the
fast-weight chunked read-then-write over a 4096-token sequence; --decode times
decode-shaped forward calls (N = 1, 8, 64); --stage times one stage alone.

One step = one pass of the whole layer over one batch of synthetic tokens: query
network, sub-key scoring with per-half top-k, candidate top-k with softmax, value
bag (forward), then the value-gradient stage and the query-gradient stage
(backward).  Inputs are resident in HBM when the timed region starts; the L2 is
flushed (a 256 MiB write) before every timed step, outside the step's events.
Timing: CUDA events on the launching stream, W warm-up steps, K timed steps
bracketed by barrier + synchronize, max over ranks.  With N > 1 (torchrun), every
rank processes its own batch against its own replica of the tables (tokens are
independent, so there is no data-path collective): weak scaling.

Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from product_key_memory_pkm_b200.inputs import (CONFIGS, FASTWEIGHT, FULL_K1024,  # noqa: E402
                                              make_inputs, make_targets)

METRIC = "PKM layer tokens/s (fwd, fwd+bwd) at |K|=1024²,h=4,k=32; gather HBM GB/s vs peak"
FW_METRIC = "FwPKM chunked read-then-write tokens/s over the sequence (8 chunks of 512)"
FW_CHUNK, FW_LR = 512, 1.0
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sus=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def _cfg_json(cfg):
    return {"workload": cfg.name, "N_tokens": cfg.N, "d_in": cfg.d_in, "h": cfg.h, "dk": cfg.dk,
            "C1": cfg.C1, "C2": cfg.C2, "K": cfg.K, "k": cfg.k, "d_v": cfg.d_v,
            "input_dtype": cfg.dtype, "value_dtype": cfg.vdtype, "l2": "flushed before every timed step (256 MiB write)"}


# ---------------------------------------------------------------- ranks
def rank_batch(cfg, rank: int, world: int, with_dy: bool = True) -> dict:
    """One replica's inputs: the same tables on every rank (seed 0), and with more than one
    rank each its own tokens (and upstream gradient) from seed 1000 + rank."""
    inp = make_inputs(cfg, seed=0, with_dy=with_dy)
    if world > 1:
        other = make_inputs(cfg, seed=1000 + rank, with_dy=with_dy)
        inp["x"] = other["x"]
        if with_dy:
            inp["dy"] = other["dy"]
    return inp


def max_over_ranks(values, dist, device) -> list:
    """Each timing as the maximum over the ranks (the slowest replica sets the step)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.uuid = gpu_uuid
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"pkm_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle timing
def _oracle_kw(variant: str) -> dict:
    return {"bf16_q": dict(q_bf16=True), "bn_train": dict(bn_train=True),
            "all_k2": dict(all_k2=True)}.get(variant, {})


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_oracle(cfg, inp, seconds: float, batch: int = 8, variant: str = "none",
                backward: bool = True, select: str = "brute"):
    """Oracle forward [+ backward] on successive token batches until ``seconds`` of host
    time have passed.  ``select`` is the oracle's key selection: "brute" (every key
    scored, the definition) or "product" (its product-key search, pinned equal to brute
    force).  Returns (tokens/s, tokens, threads)."""
    from oracle import pkm_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    done, t0 = 0, time.perf_counter()
    while True:
        sl = slice(done % cfg.N, done % cfg.N + batch)
        sub = dict(inp, x=inp["x"][sl])
        f = O.forward(sub, cfg, select=select, **_oracle_kw(variant))
        if backward:
            O.backward(sub, cfg, f, inp["dy"][sl])
        done += sub["x"].shape[0]
        el = time.perf_counter() - t0
        if el >= seconds:
            return done / el, done, threads


# ---------------------------------------------------------------- the B200 arm
def run_b200(args, cfg, rank, world, dist):
    import torch

    from product_key_memory_pkm_b200 import build as B
    from product_key_memory_pkm_b200 import pkm as P

    if not os.path.exists(B.LIB):
        if rank == 0:
            print("building libpkm_b200.so", file=sys.stderr)
        B.build()
    P.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    st = torch.cuda.current_stream()

    t_gen = time.perf_counter()
    inp = rank_batch(cfg, rank, world)
    bf = torch.bfloat16
    x = torch.from_numpy(inp["x"]).to(bf).to(dev)
    Wq = torch.from_numpy(inp["Wq"]).to(bf).to(dev)
    bn = torch.from_numpy(inp["bn"]).to(dev)
    sub = torch.from_numpy(inp["subkeys"]).to(bf).to(dev)
    # stage-only runs of the forward steps before the gather need no value table
    need_table = args.stage not in ("query", "subkey_scores", "candidate_topk")
    V = torch.from_numpy(inp["values"]).to(bf).to(dev) if need_table else None
    dy = torch.from_numpy(inp["dy"]).to(dev)
    gen_s = time.perf_counter() - t_gen

    vflags = {"none": 0, "bf16_q": P.PKM_F_BF16_Q, "bn_train": P.PKM_F_BN_TRAIN,
              "all_k2": P.PKM_F_ALL_K2}[args.variant]
    dims = P.Dims.from_config(cfg, flags=vflags)
    ksel = cfg.k * cfg.k if args.variant == "all_k2" else cfg.k
    saved = P.alloc_saved(dims, with_qhat=True)
    y = torch.empty(cfg.N, cfg.d_v, device=dev)
    dx = torch.empty(cfg.N, cfg.d_in, device=dev)
    dWq = torch.zeros(cfg.h * cfg.dk, cfg.d_in, device=dev)
    dbn = torch.zeros(2, cfg.h * cfg.dk, device=dev)
    dsub = torch.zeros(cfg.h, cfg.C1 + cfg.C2, cfg.dk // 2, device=dev)
    dV = (torch.zeros(cfg.K, cfg.d_v, device=dev)
          if args.stage in (None, "value_grad", "query_grad") else None)
    dw = torch.empty(cfg.N, cfg.h, ksel, device=dev)
    ws = P.alloc_workspace(dims, P.PKM_BWD, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    names = ["query", "subkey_scores", "candidate_topk", "gather_bag", "value_grad", "query_grad"]
    # high priority: the sort's short kernels are scheduled ahead of the bag's waiting CTAs
    side = torch.cuda.Stream(device=dev, priority=-1)
    fork_ev, join_ev = torch.cuda.Event(), torch.cuda.Event()

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(st)
        mark(0)
        P.pkm_query(dims, x, Wq, bn, saved, stream=st)
        mark(1)
        P.pkm_subkey_scores(dims, sub, saved, stream=st)
        mark(2)
        P.pkm_candidate_topk(dims, saved, stream=st)
        mark(3)
        # the value stage (pkm_value_grad) in its two parts: the sort needs only the
        # selection, so it runs on a second stream beside the bag; the row pass is timed
        # alone (any wait for the sort is in the value stage's time)
        fork_ev.record(st)
        side.wait_event(fork_ev)
        P.pkm_value_sort(dims, saved, workspace=ws, stream=side)
        join_ev.record(side)
        P.pkm_gather_bag(dims, V, saved["idx"], saved["w"], y, stream=st)
        mark(4)
        st.wait_event(join_ev)
        mark(5)
        P.pkm_value_rows(dims, V, dy, dw, dvalues=dV, workspace=ws, stream=st)
        mark(6)
        P.pkm_query_grad(dims, x, Wq, bn, sub, saved, dw, dx=dx, dWq=dWq, dbn=dbn, dsubkeys=dsub,
                         workspace=ws, stream=st)
        mark(7)

    if args.stage:
        return run_stage(args, cfg, dims, saved, P, st, step, flush, names, locals())

    clocks = ClockSampler(torch.cuda.get_device_properties(dev).uuid and
                          "GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if P.pkm_check_status(st) != P.PKM_OK:
        raise RuntimeError("device status after warm-up is not OK")
    # algorithmic bytes of the value stage need the number of distinct rows
    U = int(torch.unique(saved["idx"]).numel())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = P.pkm_launch_count()
    for s in range(args.steps):
        flush.zero_()
        step(evs[s])
    torch.cuda.synchronize()
    launches = P.pkm_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    # stage boundaries: query, scores, candidates, bag, value stage (sort + rows), query grad
    bounds = [(0, 1), (1, 2), (2, 3), (3, 4), (4, 6), (6, 7)]
    stage_ms = np.array([[evs[s][a].elapsed_time(evs[s][b]) for a, b in bounds]
                         for s in range(args.steps)])
    rows_ms = float(np.mean([evs[s][5].elapsed_time(evs[s][6]) for s in range(args.steps)]))
    step_ms = float(stage_ms.sum(1).mean())
    # the forward alone (F1-F4), timed in its own steps: in the full step the bag's interval
    # also holds the backward's sort, which runs beside it
    fwd_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for s_ in range(args.steps):
        flush.zero_()
        fwd_ev[s_][0].record(st)
        P.pkm_query(dims, x, Wq, bn, saved, stream=st)
        P.pkm_subkey_scores(dims, sub, saved, stream=st)
        P.pkm_candidate_topk(dims, saved, stream=st)
        P.pkm_gather_bag(dims, V, saved["idx"], saved["w"], y, stream=st)
        fwd_ev[s_][1].record(st)
    torch.cuda.synchronize()
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in fwd_ev]))
    if P.pkm_check_status(st) != P.PKM_OK:
        raise RuntimeError("device status after the timed steps is not OK")

    # e2e through the public API with host buffers: every step's x and dy come in from pinned
    # host memory and its y and dx go back, all inside one timed region.  The layer runs as
    # its stage entry points (pkm_query ... pkm_query_grad, what pkm_forward and pkm_backward
    # call) in the device-timed step's schedule, the value stage's sort beside the bag.  The loop prefetches
    # as a training loop's input pipeline does: while step s computes, step s+1's inputs come
    # in (copy stream) and step s's y, then dx, go out (a second copy stream) as soon as they
    # exist; device and host buffers alternate between steps, and a buffer is written again
    # only after its previous copy finished.  The first step's inputs and the last step's
    # outputs are copied inside the region too.
    e2e = None
    if not args.no_e2e:
        xh = torch.from_numpy(inp["x"]).to(bf).pin_memory()
        dyh = torch.from_numpy(inp["dy"]).pin_memory()
        yh = [torch.empty(cfg.N, cfg.d_v).pin_memory() for _ in range(2)]
        dxh = [torch.empty(cfg.N, cfg.d_in).pin_memory() for _ in range(2)]
        xd = [x, torch.empty_like(x)]
        dyd = [dy, torch.empty_like(dy)]
        yd = [y, torch.empty_like(y)]
        dxd = [dx, torch.empty_like(dx)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_run(K):
            ev = lambda: torch.cuda.Event(enable_timing=False)
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            in_ready, done, out_done = [None] * K, [None] * K, [None] * K
            start.record(st)

            def fetch(s_):
                b = s_ % 2
                with torch.cuda.stream(s_in):
                    xd[b].copy_(xh, non_blocking=True)
                    dyd[b].copy_(dyh, non_blocking=True)
                in_ready[s_] = s_in.record_event(ev())
            s_in.wait_event(start)
            fetch(0)
            for s_ in range(K):
                b = s_ % 2
                flush.zero_()
                if s_ + 1 < K:                      # buffers b^1 were last read by step s-1
                    if s_ >= 1:
                        s_in.wait_event(done[s_ - 1])
                    fetch(s_ + 1)
                st.wait_event(in_ready[s_])
                if s_ >= 2:                         # y and dx buffers b: step s-2 copied out
                    st.wait_event(out_done[s_ - 2])
                # the layer through its public stage entry points, in the device-timed step's
                # schedule: the value stage's sort on the side stream beside the bag
                P.pkm_query(dims, xd[b], Wq, bn, saved, stream=st)
                P.pkm_subkey_scores(dims, sub, saved, stream=st)
                P.pkm_candidate_topk(dims, saved, stream=st)
                side.wait_event(st.record_event(ev()))
                P.pkm_value_sort(dims, saved, workspace=ws, stream=side)
                sorted_ev = side.record_event(ev())
                P.pkm_gather_bag(dims, V, saved["idx"], saved["w"], yd[b], stream=st)
                s_out.wait_event(st.record_event(ev()))
                with torch.cuda.stream(s_out):
                    yh[b].copy_(yd[b], non_blocking=True)
                st.wait_event(sorted_ev)
                P.pkm_value_rows(dims, V, dyd[b], dw, dvalues=dV, workspace=ws, stream=st)
                P.pkm_query_grad(dims, xd[b], Wq, bn, sub, saved, dw, dx=dxd[b], dWq=dWq,
                                 dbn=dbn, dsubkeys=dsub, workspace=ws, stream=st)
                done[s_] = st.record_event(ev())
                s_out.wait_event(done[s_])
                with torch.cuda.stream(s_out):
                    dxh[b].copy_(dxd[b], non_blocking=True)
                out_done[s_] = s_out.record_event(ev())
            st.wait_stream(s_out)
            st.wait_stream(s_in)
            end.record(st)
            end.synchronize()
            return start.elapsed_time(end) / K
        e2e_run(max(2, args.warmup))
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e2e_ms = e2e_run(args.steps)
        torch.cuda.synchronize()
        e2e = dict(ms=e2e_ms,
                   h2d=x.numel() * x.element_size() + dy.numel() * dy.element_size(),
                   d2h=y.numel() * 4 + dx.numel() * 4)
    clk = clocks.stop()

    # max over ranks
    step_ms, fwd_ms, e2e_ms = max_over_ranks([step_ms, fwd_ms, e2e["ms"] if e2e else 0.0], dist,
                                             dev)
    if rank != 0:
        return None

    pk = _peaks()
    st_mean = stage_ms.mean(0)
    hk = cfg.h * ksel
    sel = cfg.N * hk
    bytes_gather = sel * cfg.d_v * 2 + cfg.N * cfg.d_v * 4 + sel * 8
    bytes_value = U * cfg.d_v * (2 + 8) + cfg.N * cfg.d_v * 4 + sel * 12
    # per kernel: the bag, and the value stage's row pass (value_rows_kernel, timed alone;
    # the stage's sort is in stage_ms["value_grad"])
    rl = {
        "gather_bag": dict(bytes=bytes_gather, ms=float(st_mean[3])),
        "value_rows": dict(bytes=bytes_value, ms=rows_ms),
    }
    dom = max(rl, key=lambda k: rl[k]["ms"])
    traffic = _ncu_traffic(dom)

    def roof(name):
        r = rl[name]
        ach = r["bytes"] / (r["ms"] * 1e-3) / 1e9
        return {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"],
                "unit": "GB/s", "frac": round(ach / pk["hbm"], 4),
                "traffic": traffic if name == dom else _ncu_traffic(name),
                "algorithmic_bytes": int(r["bytes"]), "ms": round(r["ms"], 4),
                "peak_source": pk["src"]}

    out = {
        "metric": METRIC,
        "value": round(cfg.N * world / (step_ms * 1e-3), 1),
        "unit": "tokens/s (fwd+bwd)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded; tables random-init, no trained weights)",
        "config": dict(_cfg_json(cfg), parallelism=f"replicas{world}" if world > 1 else "single",
                       variant=args.variant),
        "schedule": "the value stage's sort on a high-priority second stream beside the bag",
        "fwd": {"value": round(cfg.N * world / (fwd_ms * 1e-3), 1), "unit": "tokens/s (fwd)",
                "ms": round(fwd_ms, 4)},
        "stage_ms": {n: round(float(v), 4) for n, v in zip(names, st_mean)},
        "roofline": roof(dom),
        "roofline_other": [dict(roof(n), note="the value stage's sort runs beside this kernel "
                                              "on a high-priority second stream; this interval "
                                              "includes its share")
                           if n == "gather_bag" else roof(n) for n in rl if n != dom],
        "clocks": clk,
        "gpu_launches": int(launches),
        "input_gen_s": round(gen_s, 1),
    }
    if e2e:
        out["e2e"] = {"value": round(cfg.N * world / (e2e_ms * 1e-3), 1),
                      "unit": "tokens/s (fwd+bwd)",
                      "how": "host buffers in and out through pinned memory every step; the "
                             "copies overlap the neighbouring steps' compute; the layer through "
                             "its public stage entry points in the step's schedule (the value "
                             "sort beside the bag)",
                      "h2d_bytes_per_step": int(e2e["h2d"]), "d2h_bytes_per_step": int(e2e["d2h"]),
                      "ms": round(e2e_ms, 4)}
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_fwdbwd(cfg, inp, args.cpu_seconds, args.variant)
    return out


def cpu_baseline_fwdbwd(cfg, inp, seconds: float, variant: str = "none") -> dict:
    """The oracle on the host cores: its product-key search (two thirds of the time, in
    batches of 64 tokens) and, beside it, its brute-force definition (one third)."""
    v, n, thr = time_oracle(cfg, inp, seconds * 2 / 3, batch=64, variant=variant,
                            select="product")
    vb, nb, _ = time_oracle(cfg, inp, seconds / 3, variant=variant)
    return {"value": round(v, 3), "unit": "tokens/s (fwd+bwd)", "cores": thr, "kind": "oracle",
            "cpu": cpu_model(),
            "sample": f"{n} tokens of the same batch in batches of 64; fp64 numpy oracle with its "
                      f"product-key search (per-half top-k, then the k x k combine; selection "
                      f"pinned equal to brute force), analytic backward; "
                      f"~{seconds * 2 / 3:.0f} s of host time",
            "brute_force": {"value": round(vb, 3), "unit": "tokens/s (fwd+bwd)",
                            "sample": f"{nb} tokens; every one of the {cfg.K} keys scored per "
                                      f"head (the definition); ~{seconds / 3:.0f} s"}}


# ---------------------------------------------------------------- fast-weight workload
def time_oracle_fastweight(cfg, inp, targets, seconds: float, n: int = 32):
    """The oracle's chunk loop on successive n-token slices (one chunk each) until
    ``seconds`` of host time have passed.  Returns (tokens/s, tokens, threads)."""
    from oracle import pkm_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    done, t0 = 0, time.perf_counter()
    while True:
        sl = slice(done % cfg.N, done % cfg.N + n)
        sub = dict(inp, x=inp["x"][sl])
        O.fastweight_chunks(sub, cfg, n, FW_LR, targets=targets[sl])
        done += n
        el = time.perf_counter() - t0
        if el >= seconds:
            return done / el, done, threads


def run_fastweight(args, cfg, rank, world, dist):
    """One step = the whole chunk loop over the sequence: every chunk reads (query,
    scoring, candidates, bag + residual) and then writes (sparse SGD on its rows).
    Headline: the loop captured once into a CUDA graph and replayed; the eager loop
    and a per-stage breakdown (each stage timed alone over the 8 chunks) beside it."""
    import torch

    from product_key_memory_pkm_b200 import build as B
    from product_key_memory_pkm_b200 import pkm as P

    if not os.path.exists(B.LIB):
        B.build()
    P.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    t_gen = time.perf_counter()
    inp = rank_batch(cfg, rank, world, with_dy=False)   # each rank its own sequence
    tg_np = make_targets(cfg, seed=1000 + rank if world > 1 else 0)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
    sto = (lambda a: f32(a).to(torch.bfloat16)) if cfg.dtype == "bf16" else f32
    x, Wq, bn, sub, V, tg = (sto(inp["x"]), sto(inp["Wq"]), f32(inp["bn"]), sto(inp["subkeys"]),
                             f32(inp["values"]), f32(tg_np))
    gen_s = time.perf_counter() - t_gen
    dims = P.Dims.from_config(cfg)
    y = torch.empty(cfg.N, cfg.d_v, device=dev)
    ws = P.alloc_fastweight_workspace(dims, FW_CHUNK, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    side = torch.cuda.Stream(device=dev)

    def loop(stream, xb=x, tgb=tg, yb=y):
        P.pkm_fastweight_chunks(dims, FW_CHUNK, FW_LR, xb, Wq, bn, sub, V, yb, targets=tgb,
                                workspace=ws, stream=stream)

    clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            flush.zero_()
            loop(side)
        side.synchronize()
        if P.pkm_check_status(side) != P.PKM_OK:
            raise RuntimeError("device status after warm-up is not OK")
        l0 = P.pkm_launch_count()
        loop(side)
        side.synchronize()
        launches_per_step = P.pkm_launch_count() - l0

        def timed(fn):
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            if dist is not None:
                dist.barrier()
            torch.cuda.synchronize()
            for a, b in evs:
                flush.zero_()
                a.record(side)
                fn()
                b.record(side)
            torch.cuda.synchronize()
            if dist is not None:
                dist.barrier()
            return float(np.mean([a.elapsed_time(b) for a, b in evs]))

        eager_ms = timed(lambda: loop(side))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            loop(side)
        for _ in range(args.warmup):
            graph.replay()
        graph_ms = timed(graph.replay)
        if P.pkm_check_status(side) != P.PKM_OK:
            raise RuntimeError("device status after the timed steps is not OK")

        # per-stage view through the stage entry points, as the loop runs them: the
        # selection of the whole sequence at once (it does not read the table), then
        # per chunk the bag and the write (pkm_value_sgd sorts its own chunk)
        names = ["query", "subkey_scores", "candidate_topk", "gather_bag", "value_sgd"]
        sdims = P.Dims.from_config(cfg)
        cdims = P.Dims.from_config(cfg, N=FW_CHUNK)
        saved = P.alloc_saved(sdims, with_qhat=False)
        bws = P.alloc_workspace(cdims, P.PKM_BWD, device=dev)
        dyc = torch.empty(FW_CHUNK, cfg.d_v, device=dev)
        nch = cfg.N // FW_CHUNK
        hk = cfg.h * cfg.k
        stage_ms = np.zeros(len(names))
        U_tot = 0

        def ev_time(fn):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.zero_()
            a.record(side)
            fn()
            b.record(side)
            b.synchronize()
            return a.elapsed_time(b)
        for rep in range(args.steps):
            stage_ms[0] += ev_time(lambda: P.pkm_query(sdims, x, Wq, bn, saved, stream=side))
            stage_ms[1] += ev_time(lambda: P.pkm_subkey_scores(sdims, sub, saved, stream=side))
            stage_ms[2] += ev_time(lambda: P.pkm_candidate_topk(sdims, saved, stream=side))
            for c in range(nch):
                r0, r1 = c * FW_CHUNK, (c + 1) * FW_CHUNK
                sc = {"idx": saved["idx"][r0:r1], "w": saved["w"][r0:r1]}
                stage_ms[3] += ev_time(lambda: P.pkm_gather_bag(cdims, V, sc["idx"], sc["w"],
                                                                y[r0:r1], stream=side))
                if rep == 0:
                    torch.sub(y[r0:r1], tg[r0:r1], out=dyc)
                    U_tot += int(torch.unique(sc["idx"]).numel())
                stage_ms[4] += ev_time(lambda: P.pkm_value_sgd(cdims, FW_LR, V, sc, dyc,
                                                               workspace=bws, stream=side))
        stage_ms /= args.steps
    clk = clocks.stop()
    graph_ms, eager_ms = max_over_ranks([graph_ms, eager_ms], dist, dev)
    if rank != 0:
        return None

    pk = _peaks()
    sel = FW_CHUNK * cfg.h * cfg.k
    per_launch = {"query": 1, "subkey_scores": 1, "candidate_topk": 1, "gather_bag": nch,
                  "value_sgd": nch}
    # algorithmic bytes over the sequence (the bag and the write are HBM-bound)
    alg = {
        "gather_bag": nch * (sel * cfg.d_v * 4 + FW_CHUNK * cfg.d_v * 4 + sel * 8),
        "value_sgd": U_tot * cfg.d_v * 8 + nch * (FW_CHUNK * cfg.d_v * 4 + sel * 8),
    }
    tc = cfg.dtype == "bf16"       # tensor-core query and scoring (q as hi + lo: 2 passes)
    flops = {"query": 2.0 * cfg.N * cfg.d_in * cfg.h * cfg.dk,
             "subkey_scores": (2 if tc else 1) * 2.0 * cfg.N * cfg.h * (cfg.C1 + cfg.C2) *
             cfg.dk / 2}
    # fp32 CUDA-core peak: 148 SMs x 128 FMA lanes x 2 flops x max SM clock
    fp32_peak = 148 * 128 * 2 * (clk.get("sm_max_mhz") or 1965) * 1e6 / 1e12
    dom_i = int(np.argmax(stage_ms))
    dom = names[dom_i]
    launch_ms = stage_ms[dom_i] / per_launch[dom]
    if dom in alg:
        ach = alg[dom] / (stage_ms[dom_i] * 1e-3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"],
                "unit": "GB/s", "frac": round(ach / pk["hbm"], 4), "traffic": None,
                "algorithmic_bytes": int(alg[dom] / per_launch[dom]), "peak_source": pk["src"]}
    elif dom in flops:
        ach = flops[dom] / (stage_ms[dom_i] * 1e-3) / 1e12
        peak = pk["bf16"] if tc else round(fp32_peak, 1)
        roof = {"kernel": dom, "bound": "tensor" if tc else "alu", "achieved": round(ach, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None,
                "algorithmic_flops": flops[dom],
                "peak_source": pk["src"] if tc else "fp32 FMA lanes x max SM clock"}
    else:
        roof = {"kernel": dom, "bound": "latency", "achieved": None, "peak": None, "unit": None,
                "frac": None, "traffic": None}
    roof["ms_per_launch"] = round(float(launch_ms), 4)

    # e2e: every sequence's inputs (x, targets) in from pinned host memory and every read (y)
    # back, all inside one timed region.  Two graphs over alternating buffers: while sequence s
    # runs, the inputs of s+1 come in on a copy stream and the y of s goes out on another as
    # soon as it exists; the table is updated by the sequences in order on the compute stream.
    xh, tgh = x.cpu().pin_memory(), tg.cpu().pin_memory()
    yh = [torch.empty(cfg.N, cfg.d_v).pin_memory() for _ in range(2)]
    xs, tgs, ys = [x, torch.empty_like(x)], [tg, torch.empty_like(tg)], [y, torch.empty_like(y)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    with torch.cuda.stream(side):
        graph2 = torch.cuda.CUDAGraph()
        xs[1].copy_(x)
        tgs[1].copy_(tg)
        with torch.cuda.graph(graph2, stream=side):
            loop(side, xs[1], tgs[1], ys[1])
        graphs = [graph, graph2]

        def e2e_run(K):
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            in_ready, done, out_done = [None] * K, [None] * K, [None] * K
            start.record(side)

            def fetch(s_):
                with torch.cuda.stream(s_in):
                    xs[s_ % 2].copy_(xh, non_blocking=True)
                    tgs[s_ % 2].copy_(tgh, non_blocking=True)
                in_ready[s_] = s_in.record_event()
            s_in.wait_event(start)
            fetch(0)
            for s_ in range(K):
                b = s_ % 2
                flush.zero_()
                if s_ + 1 < K:                  # buffers b^1 were last read by sequence s-1
                    if s_ >= 1:
                        s_in.wait_event(done[s_ - 1])
                    fetch(s_ + 1)
                side.wait_event(in_ready[s_])
                if s_ >= 2:                     # y buffer b: sequence s-2's copy out finished
                    side.wait_event(out_done[s_ - 2])
                graphs[b].replay()
                done[s_] = side.record_event()
                s_out.wait_event(done[s_])
                with torch.cuda.stream(s_out):
                    yh[b].copy_(ys[b], non_blocking=True)
                out_done[s_] = s_out.record_event()
            side.wait_stream(s_out)
            side.wait_stream(s_in)
            end.record(side)
            end.synchronize()
            return start.elapsed_time(end) / K
        e2e_run(max(2, args.warmup))
        if dist is not None:
            dist.barrier()
        e2e_ms = e2e_run(args.steps)
    del graph, graph2, graphs

    out = {
        "metric": FW_METRIC,
        "value": round(cfg.N * world / (graph_ms * 1e-3), 1),
        "unit": "tokens/s (read + write, whole sequence)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(graph_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if cfg.dtype == "f32" else "bf16 inputs, f32 value table",
        "data": "synthetic (seeded; 64 input clusters, N(0,1) targets)",
        "config": dict(_cfg_json(cfg), chunk=FW_CHUNK, lr=FW_LR,
                       parallelism=f"replicas{world}" if world > 1 else "single"),
        "eager": {"ms": round(eager_ms, 4), "value": round(cfg.N * world / (eager_ms * 1e-3), 1)},
        "stage_ms_per_sequence": {n: round(float(v), 4) for n, v in zip(names, stage_ms)},
        "distinct_rows_per_chunk": round(U_tot / nch, 1),
        "roofline": roof,
        "clocks": clk,
        "gpu_launches": int(launches_per_step * args.steps),
        "input_gen_s": round(gen_s, 1),
        "e2e": {"value": round(cfg.N * world / (e2e_ms * 1e-3), 1),
                "unit": "tokens/s (host x and targets in, y out)",
                "h2d_bytes_per_step": int(xh.numel() * xh.element_size() +
                                          tgh.numel() * tgh.element_size()),
                "d2h_bytes_per_step": int(cfg.N * cfg.d_v * 4), "ms": round(e2e_ms, 4)},
    }
    if world == 1 and not args.no_cpu_baseline:
        v, n, thr = time_oracle_fastweight(cfg, inp, tg_np, args.cpu_seconds)
        out["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s (read + write)",
                               "cores": thr, "kind": "oracle",
                               "sample": f"{n} tokens, 32-token chunks of the same sequence; fp64 "
                                         f"numpy oracle, brute force over all {cfg.K} keys"}
    return out


# ---------------------------------------------------------------- decode latency
DECODE_METRIC = "PKM decode forward latency (us/call) at |K|=1024², h=4, k=32, d=1600"
SHARD_METRIC = "row-sharded PKM layer tokens/s (fwd+bwd), value rows split over the ranks"


def run_decode(args, cfg, rank, world, dist):
    """Decode-shaped forward calls (N = 1, 8, 64 tokens) against the full table: the
    four forward steps captured once per size into a CUDA graph and replayed, timed per
    call with the L2 warm (back-to-back replays) and flushed (a 256 MiB write before
    each call, outside its events); the eager call sequence beside it."""
    import torch

    from product_key_memory_pkm_b200 import build as B
    from product_key_memory_pkm_b200 import pkm as P

    if not os.path.exists(B.LIB):
        B.build()
    P.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    sizes = (1, 8, 64)
    inp = make_inputs(cfg.with_(N=max(sizes)), seed=0, with_dy=False)
    bf = torch.bfloat16
    x_all = torch.from_numpy(inp["x"]).to(bf).to(dev)
    Wq = torch.from_numpy(inp["Wq"]).to(bf).to(dev)
    bn = torch.from_numpy(inp["bn"]).to(dev)
    sub = torch.from_numpy(inp["subkeys"]).to(bf).to(dev)
    V = torch.from_numpy(inp["values"]).to(bf).to(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    side = torch.cuda.Stream(device=dev)
    reps = max(50, args.steps * 20)
    clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    res, launches = {}, 0
    with torch.cuda.stream(side):
        for n in sizes:
            dims = P.Dims.from_config(cfg, N=n)
            saved = P.alloc_saved(dims, with_qhat=False)
            x = x_all[:n].contiguous()
            y = torch.empty(n, cfg.d_v, device=dev)
            # few tokens: the optional workspace runs the forward as one fused kernel
            fused_ws = (P.alloc_workspace(dims, P.PKM_FWD_FUSED)
                        if P.pkm_workspace_bytes(dims, P.PKM_FWD_FUSED) > 0 else None)

            def call(ws=fused_ws):
                P.pkm_forward(dims, x, Wq, bn, sub, V, y, saved, workspace=ws, stream=side)

            def call_separate():
                P.pkm_forward(dims, x, Wq, bn, sub, V, y, saved, stream=side)
            for _ in range(args.warmup):
                call()
            side.synchronize()
            l0 = P.pkm_launch_count()
            call()
            side.synchronize()
            per_call = P.pkm_launch_count() - l0

            def burst(fn):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(side)
                for _ in range(reps):
                    fn()
                b.record(side)
                b.synchronize()
                return 1e3 * a.elapsed_time(b) / reps

            def cold(fn):
                out = []
                for _ in range(args.steps * 5):
                    a, b = (torch.cuda.Event(enable_timing=True),
                            torch.cuda.Event(enable_timing=True))
                    flush.zero_()
                    a.record(side)
                    fn()
                    b.record(side)
                    b.synchronize()
                    out.append(1e3 * a.elapsed_time(b))
                return float(np.median(out))
            eager_warm = burst(call)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                call()
            g.replay()
            graph_warm = burst(g.replay)
            graph_cold = cold(g.replay)
            eager_cold = cold(call)
            sep = None
            if fused_ws is not None:  # the four separate kernels, for comparison
                l1 = P.pkm_launch_count()
                call_separate()
                side.synchronize()
                launches += (P.pkm_launch_count() - l1) * (reps + args.steps * 5)
                g2 = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g2, stream=side):
                    call_separate()
                g2.replay()
                sep = {"graph_us_l2_warm": round(burst(g2.replay), 2),
                       "graph_us_l2_flushed": round(cold(g2.replay), 2)}
                del g2
            launches += per_call * (reps + args.steps * 5) * 2
            assert P.pkm_check_status(side) == P.PKM_OK
            # bytes a call must move: Wq and the sub-keys once, then n*h*k value rows
            alg = (cfg.h * cfg.dk * cfg.d_in * 2 + cfg.h * (cfg.C1 + cfg.C2) * cfg.dk // 2 * 2 +
                   n * cfg.h * cfg.k * cfg.d_v * 2 + n * (cfg.d_in * 2 + cfg.d_v * 4))
            res[n] = {"graph_us_l2_warm": round(graph_warm, 2),
                      "graph_us_l2_flushed": round(graph_cold, 2),
                      "eager_us_l2_warm": round(eager_warm, 2),
                      "eager_us_l2_flushed": round(eager_cold, 2),
                      "kernels_per_call": int(per_call), "algorithmic_bytes": int(alg),
                      **({"separate_kernels": sep} if sep else {})}
            del g
    clk = clocks.stop()
    if rank != 0:
        return None
    pk = _peaks()
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        tps, n_tok, thr = time_oracle(cfg.with_(N=max(sizes)), inp, min(args.cpu_seconds, 8.0),
                                      batch=1, backward=False)
        cpu = {"value": round(1e6 / tps, 1), "unit": "us per forward call at N=1", "cores": thr,
               "kind": "oracle",
               "sample": f"{n_tok} single-token forward calls; fp64 numpy oracle, brute force "
                         f"over all {cfg.K} keys per head"}
    top = res[max(sizes)]
    ach = top["algorithmic_bytes"] / (top["graph_us_l2_flushed"] * 1e-6) / 1e9
    return {
        "metric": DECODE_METRIC, "value": res[1]["graph_us_l2_flushed"],
        "unit": "us per forward call at N=1 (CUDA graph, L2 flushed)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(res[1]["graph_us_l2_flushed"] / 1e3, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; tables random-init)",
        "config": dict(_cfg_json(cfg), N_tokens=list(sizes), parallelism="single"),
        "per_size": {str(n): v for n, v in res.items()},
        "roofline": {"kernel": "forward call at N=64 (graph, flushed)", "bound": "hbm",
                     "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
                     "frac": round(ach / pk["hbm"], 4), "traffic": None,
                     "algorithmic_bytes": top["algorithmic_bytes"], "peak_source": pk["src"]},
        "clocks": clk, "gpu_launches": int(launches),
        **({"cpu_baseline": cpu} if cpu else {}),
    }


def run_sharded(args, cfg, rank, world, dist):
    """The row-sharded layer, fwd + bwd: every rank its own tokens and 1/world of the value
    table's rows (whole leading sub-key ranges); the exchanges between the library's calls
    go through torch.distributed (NCCL), with one rank through nothing.  Also the owner's
    partial-bag kernel alone, against the HBM roofline."""
    import torch

    from product_key_memory_pkm_b200 import build as B
    from product_key_memory_pkm_b200 import pkm as P
    from product_key_memory_pkm_b200 import sharded as S

    if not os.path.exists(B.LIB):
        B.build()
    P.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    st = torch.cuda.current_stream()
    inp = rank_batch(cfg, rank, world)
    bf = torch.bfloat16
    r0, r1 = S.shard_range(rank, world, cfg.C1, cfg.C2)
    x = torch.from_numpy(inp["x"]).to(bf).to(dev)
    Wq = torch.from_numpy(inp["Wq"]).to(bf).to(dev)
    bn = torch.from_numpy(inp["bn"]).to(dev)
    sub = torch.from_numpy(inp["subkeys"]).to(bf).to(dev)
    Vs = torch.from_numpy(inp["values"][r0:r1]).to(bf).to(dev)
    dy = torch.from_numpy(inp["dy"]).to(dev)
    ex = S.TorchExchange() if world > 1 else S.LocalExchange()
    dims = P.Dims.from_config(cfg)
    dVs = torch.zeros(max(r1 - r0, 1), cfg.d_v, device=dev)
    dx = torch.empty(cfg.N, cfg.d_in, device=dev)
    dWq = torch.zeros(cfg.h * cfg.dk, cfg.d_in, device=dev)
    dbn = torch.zeros(2, cfg.h * cfg.dk, device=dev)
    dsub = torch.zeros(cfg.h, cfg.C1 + cfg.C2, cfg.dk // 2, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(st)
        y, ctx = S.sharded_forward(dims, world, rank, x, Wq, bn, sub, Vs, ex, stream=st)
        if ev is not None:
            ev[1].record(st)
        S.sharded_backward(ctx, dy, ex, Vs, dVs, x, Wq, bn, sub, dx, dWq, dbn, dsub, stream=st)
        if ev is not None:
            ev[2].record(st)
        return ctx

    clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if P.pkm_check_status(st) != P.PKM_OK:
        raise RuntimeError("device status after warm-up is not OK")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = P.pkm_launch_count()
    for s_ in range(args.steps):
        flush.zero_()
        ctx = step(evs[s_])
    torch.cuda.synchronize()
    launches = P.pkm_launch_count() - launches0
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    # the owner's partial bag alone (the shard's HBM-bound kernel), L2 flushed before each
    n_tri, n_seg = sum(ctx.recv_tri), sum(ctx.recv_seg)
    part = torch.empty(max(n_seg, 1), cfg.d_v, device=dev)
    bag_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        P.pkm_shard_bag(dims, world, ctx.shard_rows, ctx.recv_counts, n_tri, n_seg, ctx.recv,
                        Vs, part, ctx.owner_ws, stream=st)
        b.record(st)
        b.synchronize()
        bag_ms.append(a.elapsed_time(b))
    launches += 2 * args.steps   # the bag call above: segment starts, bag
    if P.pkm_check_status(st) != P.PKM_OK:
        raise RuntimeError("device status after the timed steps is not OK")
    clk = clocks.stop()
    step_ms, fwd_ms, bwd_ms, bag = max_over_ranks(
        [fwd_ms + bwd_ms, fwd_ms, bwd_ms, float(np.mean(bag_ms))], dist, dev)
    if dist is not None:
        dist.barrier()
    if rank != 0:
        return None
    pk = _peaks()
    bag_bytes = n_tri * cfg.d_v * 2 + n_seg * cfg.d_v * 4 + n_tri * 12
    ach = bag_bytes / (bag * 1e-3) / 1e9
    out = {
        "metric": SHARD_METRIC,
        "value": round(cfg.N * world / (step_ms * 1e-3), 1),
        "unit": "tokens/s (fwd+bwd)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; tables random-init, no trained weights)",
        "config": dict(_cfg_json(cfg), parallelism=f"rowshard{world}", shard_rows=r1 - r0,
                       l2="flushed before every timed step (256 MiB write)"),
        "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
        "roofline": {"kernel": "shard_bag (owner partial bags)", "bound": "hbm",
                     "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
                     "frac": round(ach / pk["hbm"], 4), "traffic": _ncu_traffic("shard_bag"),
                     "algorithmic_bytes": int(bag_bytes), "ms": round(bag, 4),
                     "peak_source": pk["src"]},
        "clocks": clk, "gpu_launches": int(launches),
    }
    if world == 1 and not args.no_cpu_baseline:
        v, n, thr = time_oracle(cfg, inp, args.cpu_seconds)
        out["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s (fwd+bwd)", "cores": thr,
                               "kind": "oracle",
                               "sample": f"{n} tokens of the same batch, fp64 numpy oracle of the "
                                         f"whole layer (the sharding does not change the result)"}
    return out


def run_stage(args, cfg, dims, saved, P, st, step, flush, names, env):
    """Times one stage alone (after one full step has filled the saved tensors): the
    per-op view, and the launch that profiling captures target."""
    import torch
    x, Wq, bn, sub, V, y, dy, dw, ws = (env[k] for k in ("x", "Wq", "bn", "sub", "V", "y", "dy",
                                                            "dw", "ws"))
    dV, dx, dWq, dbn, dsub = (env[k] for k in ("dV", "dx", "dWq", "dbn", "dsub"))
    calls = {
        "query": lambda: P.pkm_query(dims, x, Wq, bn, saved, stream=st),
        "subkey_scores": lambda: P.pkm_subkey_scores(dims, sub, saved, stream=st),
        "candidate_topk": lambda: P.pkm_candidate_topk(dims, saved, stream=st),
        "gather_bag": lambda: P.pkm_gather_bag(dims, V, saved["idx"], saved["w"], y, stream=st),
        "value_grad": lambda: P.pkm_value_grad(dims, V, saved, dy, dw, dvalues=dV, workspace=ws,
                                               stream=st),
        "query_grad": lambda: P.pkm_query_grad(dims, x, Wq, bn, sub, saved, dw, dx=dx, dWq=dWq,
                                               dbn=dbn, dsubkeys=dsub, workspace=ws, stream=st),
    }
    order = list(calls)
    extra = {}
    if args.stage in ("value_grad_rows", "value_adam", "hit_counts"):
        # training-time stages after the forward: compact value gradient, lazy Adam on the
        # selected rows (fp32 table and state), hit histograms
        for prev in order[:4]:
            calls[prev]()
        torch.cuda.synchronize()
        U = int(torch.unique(saved["idx"]).numel())
        sel = cfg.N * cfg.h * cfg.k
        if args.stage == "value_grad_rows":
            cap = min(sel, cfg.K)
            rows = torch.empty(cap, dtype=torch.int32, device=x.device)
            dvr = torch.empty(cap, cfg.d_v, device=x.device)
            nr = torch.empty(1, dtype=torch.int32, device=x.device)
            fn = lambda: P.pkm_value_grad_rows(dims, V, saved, dy, rows, dvr, nr, dw=dw,
                                               workspace=ws, stream=st)
            alg = U * cfg.d_v * (2 + 4) + cfg.N * cfg.d_v * 4 + sel * 12
        elif args.stage == "value_adam":
            d32 = P.Dims.from_config(cfg.with_(value_dtype="f32"))
            V32, m, v = V.float(), torch.zeros(cfg.K, cfg.d_v, device=x.device), None
            v = torch.zeros_like(m)
            fn = lambda: P.pkm_value_adam(d32, 1e-3, 0.9, 0.999, 1e-8, 1, V32, m, v, saved, dy,
                                          workspace=ws, stream=st)
            alg = U * cfg.d_v * 4 * 6 + cfg.N * cfg.d_v * 4 + sel * 12
        else:
            slot = torch.zeros(cfg.K, dtype=torch.int32, device=x.device)
            subh = torch.zeros(cfg.h, cfg.C1 + cfg.C2, dtype=torch.int32, device=x.device)
            fn = lambda: P.pkm_hit_counts(dims, saved["idx"], slot, subh, stream=st)
            alg = sel * 4
        extra = {"distinct_rows": U, "algorithmic_bytes": int(alg)}
    else:
        for prev in order[: order.index(args.stage)]:   # fill the saved tensors the stage reads
            calls[prev]()
        torch.cuda.synchronize()
        fn = calls[args.stage]
        if args.stage in ("gather_bag", "value_grad"):
            # the same algorithmic bytes as the full step's roofline
            sel = cfg.N * cfg.h * cfg.k
            if args.stage == "gather_bag":
                alg = sel * cfg.d_v * 2 + cfg.N * cfg.d_v * 4 + sel * 8
                extra = {"algorithmic_bytes": int(alg)}
            else:
                U = int(torch.unique(saved["idx"]).numel())
                alg = U * cfg.d_v * (2 + 8) + cfg.N * cfg.d_v * 4 + sel * 12
                extra = {"distinct_rows": U, "algorithmic_bytes": int(alg)}
    for _ in range(args.warmup):
        flush.zero_()
        fn()
    ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        fn()
        b.record(st)
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    assert P.pkm_check_status(st) == P.PKM_OK
    out = {"stage": args.stage, "workload": cfg.name, "variant": args.variant,
           "ms_per_call": round(float(np.mean(ms)), 4), "ms_min": round(float(np.min(ms)), 4),
           "calls": args.steps}
    if extra:
        out.update(extra)
        out["GB_per_s"] = round(extra["algorithmic_bytes"] / (np.mean(ms) * 1e-3) / 1e9, 1)
    return out


def _ncu_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, when it is still current."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        j = json.load(open(p))
        ent = j.get(kernel)
        if not ent:
            return None
        import hashlib
        h = hashlib.sha256()
        for f in ent["sources"]:
            h.update(open(os.path.join(ROOT, f), "rb").read())
        if h.hexdigest() != ent["source_sha256"]:
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


# ---------------------------------------------------------------- the reference arm
def run_reference(args, cfg, rank):
    """The CPU oracle, as it stands, on a bounded sample of the workload per step: its
    product-key search (the selection pinned equal to its brute-force definition) and
    analytic backward, in fp64 numpy on the host cores."""
    if rank != 0:
        return None
    from oracle import pkm_oracle as O
    inp = make_inputs(cfg, seed=0)
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    per_step = args.ref_tokens
    times = []
    for s in range(args.warmup + args.steps):
        sl = slice((s * per_step) % cfg.N, (s * per_step) % cfg.N + per_step)
        sub = dict(inp, x=inp["x"][sl], dy=inp["dy"][sl])
        t0 = time.perf_counter()
        f = O.forward(sub, cfg, select="product")
        O.backward(sub, cfg, f, sub["dy"])
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    v = round(per_step / (ms * 1e-3), 3)
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s (fwd+bwd)",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; tables random-init, no trained weights)",
        "config": dict(_cfg_json(cfg), parallelism="single", variant="none"),
        "cpu_baseline": {"value": v, "unit": "tokens/s (fwd+bwd)", "cores": threads,
                         "kind": "oracle", "cpu": cpu_model(),
                         "sample": f"{per_step} tokens per step of the same batch; fp64 numpy "
                                   f"oracle with its product-key search over {cfg.K} keys per "
                                   f"head, analytic backward"},
        "e2e": {"value": v, "unit": "tokens/s (fwd+bwd)", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default=FULL_K1024.name, choices=sorted(CONFIGS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-tokens", type=int, default=64)
    ap.add_argument("--stage", default=None,
                    choices=["query", "subkey_scores", "candidate_topk", "gather_bag",
                             "value_grad", "query_grad", "value_grad_rows", "value_adam",
                             "hit_counts"],
                    help="time one stage alone (per-op benchmark / profiling target)")
    ap.add_argument("--tokens", type=int, default=None, help="override the token count")
    ap.add_argument("--variant", default="none", choices=["none", "bf16_q", "bn_train", "all_k2"],
                    help="layer variant for the whole step: single-pass bf16-q scoring, "
                         "training-mode BatchNorm, or the all-k^2 softmax")
    ap.add_argument("--decode", action="store_true",
                    help="decode-shaped forward latency (N = 1, 8, 64) on the workload's table")
    ap.add_argument("--sharded", action="store_true",
                    help="row-sharded value table: each rank 1/N of the rows, exchanges over "
                         "torch.distributed")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    cfg = CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.with_(N=args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        out = run_reference(args, cfg, rank)
    else:
        if world > 1:
            import datetime

            import torch
            import torch.distributed as tdist
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
            tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
            dist = tdist
        try:
            run = (run_decode if args.decode else run_sharded if args.sharded else
                   run_fastweight if cfg.name == FASTWEIGHT.name else run_b200)
            out = run(args, cfg, rank, world, dist)
        finally:
            if dist is not None:
                dist.destroy_process_group()
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
