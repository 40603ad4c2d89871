"""Seeded synthetic inputs for the product-key memory layer.

This module only draws random numbers and rounds them to the storage type.  It
holds none of the layer's arithmetic, so both the CPU oracle (``oracle/``) and
the CUDA path can take their inputs from it without sharing any computation.

Shapes and distributions follow the workloads of the product-key memory pages:
d = 1600 and h = 4 heads with k = 32 ("Large Memory Layers with Product Keys",
key results), |K| from 512^2 to 1024^2 slots (same list), queries kept near
N(0, 1) per coordinate by the batch-normalised query network (same list, the
BatchNorm remark).  Every tensor is drawn in row blocks, each block from its own
``SeedSequence([seed, tensor_id, block])``, so a block can be regenerated alone
and blocks can be drawn in parallel threads.

Layouts (row-major):
  x        [N][d_in]
  Wq       [h*dk][d_in]          (a Linear weight: out x in)
  bn       [4][h*dk]             (running mean, running var, gamma, beta)
  subkeys  [h][C1 + C2][dk/2]    (head hh: rows [0, C1) are C, rows [C1, C1+C2) are C')
  values   [C1*C2][d_v]          (row i*C2 + j belongs to the product key (i, j))
  dy       [N][d_v]
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_TENSOR_IDS = {"x": 1, "Wq": 2, "subkeys": 3, "values": 4, "dy": 5, "bn": 6,
               "centres": 7, "assign": 8, "noise": 9, "targets": 10}


@dataclasses.dataclass(frozen=True)
class PKMConfig:
    """Sizes of one product-key memory layer workload."""
    name: str
    N: int          # tokens
    d_in: int       # input width
    h: int          # heads
    dk: int         # query width per head (two halves of dk/2)
    C1: int         # |C|, first sub-key set
    C2: int         # |C'|, second sub-key set
    k: int          # top-k per half and in the final selection
    d_v: int        # value width
    dtype: str = "bf16"     # storage of x, Wq, subkeys, values: "bf16" or "f32"
    value_dtype: str = ""   # "f32": an fp32 value table beside bf16 x, Wq, subkeys
    bn_eps: float = 1e-5
    score_scale: float = 1.0
    clustered: int = 0      # >0: x drawn around this many centres (duplicate-heavy)

    @property
    def K(self) -> int:
        return self.C1 * self.C2

    @property
    def vdtype(self) -> str:
        """Storage of the value table."""
        return self.value_dtype or self.dtype

    def with_(self, **kw) -> "PKMConfig":
        return dataclasses.replace(self, **kw)


# The workloads, named by what they are.
TINY_FP32 = PKMConfig("pkm_tiny_fp32_K1024", N=64, d_in=64, h=1, dk=32, C1=32, C2=32,
                      k=8, d_v=64, dtype="f32")
FWD_K512 = PKMConfig("pkm_fwd_K512x512_h4_k32_d1024", N=4096, d_in=1024, h=4, dk=512,
                     C1=512, C2=512, k=32, d_v=1024)
FULL_K1024 = PKMConfig("pkm_fwdbwd_K1024x1024_h4_k32_d1600", N=16384, d_in=1600, h=4,
                       dk=512, C1=1024, C2=1024, k=32, d_v=1600)
FASTWEIGHT = PKMConfig("fwpkm_chunk512_K1024x1024_h1_k8_d1024", N=4096, d_in=1024, h=1,
                       dk=512, C1=1024, C2=1024, k=8, d_v=1024, value_dtype="f32",
                       clustered=64)

# the full workload with unequal sub-key sets (|C| = 2048, |C'| = 512: the same 1M slots)
FULL_K2048x512 = PKMConfig("pkm_fwdbwd_K2048x512_h4_k32_d1600", N=16384, d_in=1600, h=4,
                           dk=512, C1=2048, C2=512, k=32, d_v=1600)

CONFIGS = {c.name: c for c in (TINY_FP32, FWD_K512, FULL_K1024, FASTWEIGHT, FULL_K2048x512)}


def _round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even), returned as fp32."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _block_rng(seed: int, tensor: str, block: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed), _TENSOR_IDS[tensor], int(block)])
    return np.random.Generator(np.random.PCG64(ss))


def _draw(seed: int, tensor: str, rows: int, cols: int, kind: str, scale: float,
          rows_per_block: int, threads: int | None = None) -> np.ndarray:
    """Draw a [rows][cols] fp32 array block by block ("normal": N(0, scale^2);
    "uniform": U(-scale, scale))."""
    out = np.empty((rows, cols), dtype=np.float32)
    nblk = (rows + rows_per_block - 1) // rows_per_block

    def one(b: int) -> None:
        r0 = b * rows_per_block
        r1 = min(rows, r0 + rows_per_block)
        g = _block_rng(seed, tensor, b)
        if kind == "normal":
            blk = g.standard_normal((r1 - r0, cols), dtype=np.float32)
            blk *= np.float32(scale)
        else:
            blk = g.random((r1 - r0, cols), dtype=np.float32)
            blk = (blk * np.float32(2.0) - np.float32(1.0)) * np.float32(scale)
        out[r0:r1] = blk

    if nblk == 1:
        one(0)
    else:
        with ThreadPoolExecutor(max_workers=threads or min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(one, range(nblk)))
    return out


def _rows_per_block(cols: int) -> int:
    return max(1, (1 << 20) // max(cols, 1))


def make_inputs(cfg: PKMConfig, seed: int = 0, with_dy: bool = True,
                random_bn: bool = False) -> dict:
    """All inputs of one layer call as fp32 numpy arrays whose values are exactly
    representable in the storage type of ``cfg`` (bf16 rounding applied here).

    ``random_bn`` draws non-trivial running statistics and affine parameters, to
    exercise every term of the normalisation; by default the normalisation is the
    identity-like eval state (mean 0, var 1, gamma 1, beta 0).
    """
    hq = cfg.h * cfg.dk
    half = cfg.dk // 2
    x_scale = 1.0
    if cfg.clustered > 0:
        # x_t = mu_{c(t)} + 0.1 * noise, centres mu ~ N(0, I), c(t) uniform.
        centres = _draw(seed, "centres", cfg.clustered, cfg.d_in, "normal", 1.0,
                        _rows_per_block(cfg.d_in))
        assign = _block_rng(seed, "assign", 0).integers(0, cfg.clustered, size=cfg.N)
        noise = _draw(seed, "noise", cfg.N, cfg.d_in, "normal", 0.1,
                      _rows_per_block(cfg.d_in))
        x = centres[assign] + noise
    else:
        x = _draw(seed, "x", cfg.N, cfg.d_in, "normal", x_scale, _rows_per_block(cfg.d_in))
    Wq = _draw(seed, "Wq", hq, cfg.d_in, "normal", 1.0 / np.sqrt(cfg.d_in),
               _rows_per_block(cfg.d_in))
    sub = _draw(seed, "subkeys", cfg.h * (cfg.C1 + cfg.C2), half, "uniform",
                1.0 / np.sqrt(half), _rows_per_block(half))
    sub = sub.reshape(cfg.h, cfg.C1 + cfg.C2, half)
    V = _draw(seed, "values", cfg.K, cfg.d_v, "normal", 1.0 / np.sqrt(cfg.d_v),
              _rows_per_block(cfg.d_v))
    if random_bn:
        g = _block_rng(seed, "bn", 0)
        bn = np.stack([
            g.normal(0.0, 0.3, hq),            # running mean
            g.uniform(0.5, 2.0, hq),           # running var
            g.uniform(0.5, 1.5, hq),           # gamma
            g.normal(0.0, 0.2, hq),            # beta
        ]).astype(np.float32)
    else:
        bn = np.stack([np.zeros(hq), np.ones(hq), np.ones(hq), np.zeros(hq)]).astype(np.float32)
    if cfg.dtype == "bf16":
        x, Wq, sub = (_round_bf16(a) for a in (x, Wq, sub))
    if cfg.vdtype == "bf16":
        V = _round_bf16(V)
    out = dict(x=x, Wq=Wq, bn=bn, subkeys=sub, values=V)
    if with_dy:
        out["dy"] = _draw(seed, "dy", cfg.N, cfg.d_v, "normal", 1.0, _rows_per_block(cfg.d_v))
    return out


def make_targets(cfg: PKMConfig, seed: int = 0) -> np.ndarray:
    """Fast-weight write targets ~ N(0, 1), [N][d_v] fp32."""
    return _draw(seed, "targets", cfg.N, cfg.d_v, "normal", 1.0, _rows_per_block(cfg.d_v))
