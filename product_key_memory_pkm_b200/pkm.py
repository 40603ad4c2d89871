"""Thin Python binding of the C ABI in ``include/pkm.h`` (ctypes).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libpkm_b200.so``.  PyTorch is used for device memory and streams.  There is no
CPU fallback: loading fails loudly when the library has not been built.

The functions carry the C names (``pkm_forward``, ``pkm_backward``,
``pkm_query``, ``pkm_subkey_scores``, ``pkm_candidate_topk``,
``pkm_gather_bag``, ``pkm_check_status``, ...) and take torch tensors (device
pointers are read with ``data_ptr()``) or raw integer addresses.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
# PKM_B200_LIB overrides the library path (e.g. to compare two builds)
LIB_PATH = os.environ.get("PKM_B200_LIB") or os.path.join(HERE, "libpkm_b200.so")

PKM_OK = 0
PKM_ERR_INVALID_ARG = 1
PKM_ERR_UNSUPPORTED = 2
PKM_ERR_WORKSPACE = 3
PKM_ERR_CUDA = 4
PKM_ERR_DEVICE_TIMEOUT = 5
PKM_ERR_DEVICE_INDEX = 6

PKM_F_FP32 = 0x1
PKM_F_SIMT = 0x2
PKM_F_VALUES_FP32 = 0x4
PKM_F_BF16_Q = 0x8
PKM_F_BN_TRAIN = 0x10
PKM_F_ALL_K2 = 0x20
PKM_F_IDW = 0x40
PKM_FWD, PKM_BWD, PKM_FWD_FUSED = 0, 1, 2
PKM_FW_LOOKAHEAD = 0x1
PKM_FW_SORT_GLOBAL = 0x2
PKM_FW_PER_CHUNK = 0x4
SAVED_FIELDS = ("q", "qhat", "sub_s", "sub_i", "idx", "w", "bn_batch")
PKM_MAX_SHARDS = 1024
PKM_SHARD_ROUTE, PKM_SHARD_OWNER = 1, 2

# every symbol include/pkm.h declares
EXPORTED = ("pkm_saved_bytes", "pkm_workspace_bytes", "pkm_forward", "pkm_backward", "pkm_query",
            "pkm_subkey_scores", "pkm_candidate_topk", "pkm_gather_bag", "pkm_check_status",
            "pkm_status_string", "pkm_build_info", "pkm_value_grad", "pkm_value_sort",
            "pkm_value_rows", "pkm_query_grad",
            "pkm_launch_count", "pkm_selftest_wait_timeout", "pkm_value_grad_noalloc",
            "pkm_fastweight_workspace_bytes", "pkm_fastweight_chunks", "pkm_value_sgd",
            "pkm_value_grad_rows", "pkm_value_adam", "pkm_hit_counts", "pkm_bn_running_update",
            "pkm_shard_workspace_bytes", "pkm_shard_route", "pkm_shard_bag", "pkm_shard_combine",
            "pkm_shard_gather_dy", "pkm_shard_value_grad", "pkm_shard_scatter_dw")


class PKMError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


class pkm_dims(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("d_in", ctypes.c_int32), ("h", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("C1", ctypes.c_int32), ("C2", ctypes.c_int32),
                ("k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("bn_eps", ctypes.c_float),
                ("score_scale", ctypes.c_float), ("flags", ctypes.c_uint32)]


class pkm_saved(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in SAVED_FIELDS]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m product_key_memory_pkm_b200.build`")
    lib = ctypes.CDLL(path)
    P, S, I, U64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
    D = ctypes.POINTER(pkm_dims)
    SV = ctypes.POINTER(pkm_saved)
    sig = {
        "pkm_saved_bytes": (S, [D, I]),
        "pkm_workspace_bytes": (S, [D, I]),
        "pkm_forward": (I, [D, P, P, P, P, P, P, SV, P, S, P]),
        "pkm_backward": (I, [D, P, P, P, P, P, SV, P, P, P, P, P, P, P, P, S, P]),
        "pkm_query": (I, [D, P, P, P, SV, P]),
        "pkm_subkey_scores": (I, [D, P, SV, P]),
        "pkm_candidate_topk": (I, [D, SV, P]),
        "pkm_gather_bag": (I, [D, P, P, P, P, P]),
        "pkm_check_status": (I, [P]),
        "pkm_status_string": (ctypes.c_char_p, [I]),
        "pkm_build_info": (ctypes.c_char_p, []),
        "pkm_value_grad": (I, [D, P, SV, P, P, P, P, S, P]),
        "pkm_value_sort": (I, [D, SV, P, S, P]),
        "pkm_value_rows": (I, [D, P, P, P, P, P, S, P]),
        "pkm_query_grad": (I, [D, P, P, P, P, SV, P, P, P, P, P, P, S, P]),
        "pkm_launch_count": (ctypes.c_ulonglong, []),
        "pkm_selftest_wait_timeout": (I, [ctypes.c_uint32, P]),
        "pkm_value_grad_noalloc": (I, [D, P, SV, P, P, P, P]),
        "pkm_value_sgd": (I, [D, ctypes.c_float, P, SV, P, P, S, P]),
        "pkm_value_grad_rows": (I, [D, P, SV, P, P, P, P, P, P, S, P]),
        "pkm_value_adam": (I, [D, ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                               ctypes.c_int64, P, P, P, SV, P, P, S, P]),
        "pkm_hit_counts": (I, [D, P, P, P, P]),
        "pkm_bn_running_update": (I, [D, P, P, ctypes.c_float, P]),
        "pkm_fastweight_workspace_bytes": (S, [D, ctypes.c_int64, ctypes.c_uint32]),
        "pkm_fastweight_chunks": (I, [D, ctypes.c_int64, ctypes.c_float, ctypes.c_uint32, P, P, P,
                                      P, P, P, P, P, S, P]),
        "pkm_shard_workspace_bytes": (S, [D, ctypes.c_int32, I, ctypes.c_int64]),
        "pkm_shard_route": (I, [D, ctypes.c_int32, ctypes.c_int64, P, P, P, P, P, P, P, S, P]),
        "pkm_shard_bag": (I, [D, ctypes.c_int32, ctypes.c_int64, P, ctypes.c_int64, ctypes.c_int64,
                              P, P, P, P, S, P]),
        "pkm_shard_combine": (I, [D, ctypes.c_int32, P, P, ctypes.c_int64, P, P]),
        "pkm_shard_gather_dy": (I, [D, ctypes.c_int32, P, P, P, ctypes.c_int64, P]),
        "pkm_shard_value_grad": (I, [D, ctypes.c_int32, ctypes.c_int64, P, ctypes.c_int64,
                                     ctypes.c_int64, P, P, P, P, P, P, S, P]),
        "pkm_shard_scatter_dw": (I, [D, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    del U64
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().pkm_status_string(int(code)).decode()


# ----------------------------------------------------------------- marshalling
def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, where: str) -> None:
    if code != PKM_OK:
        raise PKMError(code, where)


@dataclass
class Dims:
    """Python mirror of ``pkm_dims``."""
    N: int
    d_in: int
    h: int
    dk: int
    C1: int
    C2: int
    k: int
    d_v: int
    bn_eps: float = 1e-5
    score_scale: float = 1.0
    flags: int = 0

    def c(self) -> pkm_dims:
        return pkm_dims(self.N, self.d_in, self.h, self.dk, self.C1, self.C2, self.k, self.d_v,
                        self.bn_eps, self.score_scale, self.flags)

    @classmethod
    def from_config(cls, cfg, flags: int = 0, N: int | None = None) -> "Dims":
        f = flags | (PKM_F_FP32 if cfg.dtype == "f32" else 0)
        if cfg.dtype != "f32" and cfg.vdtype == "f32":
            f |= PKM_F_VALUES_FP32
        return cls(cfg.N if N is None else N, cfg.d_in, cfg.h, cfg.dk, cfg.C1, cfg.C2, cfg.k,
                   cfg.d_v, cfg.bn_eps, cfg.score_scale, f)


def _saved_c(saved: dict) -> pkm_saved:
    return pkm_saved(*[_ptr(saved.get(f)) for f in SAVED_FIELDS])


def pkm_saved_bytes(dims: Dims, field: str) -> int:
    return int(load().pkm_saved_bytes(ctypes.byref(dims.c()), SAVED_FIELDS.index(field)))


def pkm_workspace_bytes(dims: Dims, which: int) -> int:
    return int(load().pkm_workspace_bytes(ctypes.byref(dims.c()), which))


def pkm_forward(dims: Dims, x, Wq, bn, subkeys, values, y, saved: dict, workspace=None,
                workspace_bytes: int = 0, stream=None) -> None:
    ws_bytes = workspace_bytes or (workspace.numel() * workspace.element_size()
                                   if workspace is not None and not isinstance(workspace, int) else 0)
    s = _saved_c(saved)
    _check(load().pkm_forward(ctypes.byref(dims.c()), _ptr(x), _ptr(Wq), _ptr(bn), _ptr(subkeys),
                              _ptr(values), _ptr(y), ctypes.byref(s), _ptr(workspace), ws_bytes,
                              _stream(stream)), "pkm_forward")


def pkm_backward(dims: Dims, x, Wq, bn, subkeys, values, saved: dict, dy, dx=None, dWq=None,
                 dbn=None, dsubkeys=None, dvalues=None, dw_out=None, workspace=None,
                 workspace_bytes: int = 0, stream=None) -> None:
    ws_bytes = workspace_bytes or (workspace.numel() * workspace.element_size()
                                   if workspace is not None and not isinstance(workspace, int) else 0)
    s = _saved_c(saved)
    _check(load().pkm_backward(ctypes.byref(dims.c()), _ptr(x), _ptr(Wq), _ptr(bn), _ptr(subkeys),
                               _ptr(values), ctypes.byref(s), _ptr(dy), _ptr(dx), _ptr(dWq),
                               _ptr(dbn), _ptr(dsubkeys), _ptr(dvalues), _ptr(dw_out),
                               _ptr(workspace), ws_bytes, _stream(stream)), "pkm_backward")


def _ws(workspace, workspace_bytes):
    if workspace_bytes:
        return workspace_bytes
    if workspace is None or isinstance(workspace, int):
        return 0
    return workspace.numel() * workspace.element_size()


def pkm_value_grad(dims: Dims, values, saved: dict, dy, dw, dvalues=None, workspace=None,
                   workspace_bytes: int = 0, stream=None) -> None:
    s = _saved_c(saved)
    _check(load().pkm_value_grad(ctypes.byref(dims.c()), _ptr(values), ctypes.byref(s), _ptr(dy),
                                 _ptr(dvalues), _ptr(dw), _ptr(workspace),
                                 _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_value_grad")


def pkm_value_sort(dims: Dims, saved: dict, workspace=None, workspace_bytes: int = 0,
                   stream=None) -> None:
    """First half of pkm_value_grad: the selections sorted by value row, into the workspace."""
    s = _saved_c(saved)
    _check(load().pkm_value_sort(ctypes.byref(dims.c()), ctypes.byref(s), _ptr(workspace),
                                 _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_value_sort")


def pkm_value_rows(dims: Dims, values, dy, dw, dvalues=None, workspace=None,
                   workspace_bytes: int = 0, stream=None) -> None:
    """Second half of pkm_value_grad: the per-row pass over what pkm_value_sort left in the
    same workspace."""
    _check(load().pkm_value_rows(ctypes.byref(dims.c()), _ptr(values), _ptr(dy), _ptr(dvalues),
                                 _ptr(dw), _ptr(workspace), _ws(workspace, workspace_bytes),
                                 _stream(stream)),
           "pkm_value_rows")


def pkm_value_grad_noalloc(dims: Dims, values, saved: dict, dy, dw, dvalues=None,
                           stream=None) -> None:
    """pkm_value_grad without a workspace argument: the scratch is a fixed device
    array inside the library (for callers that cannot allocate device memory)."""
    s = _saved_c(saved)
    _check(load().pkm_value_grad_noalloc(ctypes.byref(dims.c()), _ptr(values), ctypes.byref(s),
                                         _ptr(dy), _ptr(dvalues), _ptr(dw), _stream(stream)),
           "pkm_value_grad_noalloc")


def pkm_value_sgd(dims: Dims, lr: float, values, saved: dict, dy, workspace=None,
                  workspace_bytes: int = 0, stream=None) -> None:
    """values[r] -= lr * (sum of w * dy over the selections of r), in place (fp32)."""
    s = _saved_c(saved)
    _check(load().pkm_value_sgd(ctypes.byref(dims.c()), float(lr), _ptr(values), ctypes.byref(s),
                                _ptr(dy), _ptr(workspace), _ws(workspace, workspace_bytes),
                                _stream(stream)), "pkm_value_sgd")


def pkm_value_grad_rows(dims: Dims, values, saved: dict, dy, rows_out, dvalues_rows, num_rows,
                        dw=None, workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    """Compact value gradient: num_rows[0] = U, rows_out[:U] (ascending), dvalues_rows[:U]."""
    s = _saved_c(saved)
    _check(load().pkm_value_grad_rows(ctypes.byref(dims.c()), _ptr(values), ctypes.byref(s),
                                      _ptr(dy), _ptr(dw), _ptr(rows_out), _ptr(dvalues_rows),
                                      _ptr(num_rows), _ptr(workspace),
                                      _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_value_grad_rows")


def pkm_value_adam(dims: Dims, lr: float, beta1: float, beta2: float, eps: float, step: int,
                   values, m, v, saved: dict, dy, workspace=None, workspace_bytes: int = 0,
                   stream=None) -> None:
    """Lazy Adam on the selected value rows (values, m, v fp32, in place)."""
    s = _saved_c(saved)
    _check(load().pkm_value_adam(ctypes.byref(dims.c()), float(lr), float(beta1), float(beta2),
                                 float(eps), int(step), _ptr(values), _ptr(m), _ptr(v),
                                 ctypes.byref(s), _ptr(dy), _ptr(workspace),
                                 _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_value_adam")


def pkm_hit_counts(dims: Dims, idx, slot_hits=None, subkey_hits=None, stream=None) -> None:
    """slot_hits [C1*C2] int32 and subkey_hits [h][C1+C2] int32 accumulate (+=)."""
    _check(load().pkm_hit_counts(ctypes.byref(dims.c()), _ptr(idx), _ptr(slot_hits),
                                 _ptr(subkey_hits), _stream(stream)), "pkm_hit_counts")


def pkm_bn_running_update(dims: Dims, bn, bn_batch, momentum: float = 0.1, stream=None) -> None:
    """Fold a training-mode batch's statistics into bn's running mean and variance."""
    _check(load().pkm_bn_running_update(ctypes.byref(dims.c()), _ptr(bn), _ptr(bn_batch),
                                        float(momentum), _stream(stream)),
           "pkm_bn_running_update")


def pkm_fastweight_workspace_bytes(dims: Dims, chunk: int, mode: int = 0) -> int:
    return int(load().pkm_fastweight_workspace_bytes(ctypes.byref(dims.c()), int(chunk),
                                                     int(mode)))


def alloc_fastweight_workspace(dims: Dims, chunk: int, mode: int = 0, device="cuda"):
    import torch
    return torch.empty(max(pkm_fastweight_workspace_bytes(dims, chunk, mode), 256),
                       dtype=torch.uint8, device=device)


def pkm_fastweight_chunks(dims: Dims, chunk: int, lr: float, x, Wq, bn, subkeys, values, y,
                          targets=None, lookahead: bool = False, strategy: int = 0,
                          workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    """Chunked read-then-write of the fast-weight memory: ``values`` (fp32) is updated
    in place, ``y`` receives every chunk's read.  ``strategy``: 0, PKM_FW_SORT_GLOBAL or
    PKM_FW_PER_CHUNK (same results)."""
    mode = (PKM_FW_LOOKAHEAD if lookahead else 0) | int(strategy)
    _check(load().pkm_fastweight_chunks(ctypes.byref(dims.c()), int(chunk), float(lr), mode,
                                        _ptr(x), _ptr(Wq), _ptr(bn), _ptr(subkeys),
                                        _ptr(values), _ptr(targets), _ptr(y), _ptr(workspace),
                                        _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_fastweight_chunks")


def pkm_query_grad(dims: Dims, x, Wq, bn, subkeys, saved: dict, dw, dx=None, dWq=None, dbn=None,
                   dsubkeys=None, workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    s = _saved_c(saved)
    _check(load().pkm_query_grad(ctypes.byref(dims.c()), _ptr(x), _ptr(Wq), _ptr(bn),
                                 _ptr(subkeys), ctypes.byref(s), _ptr(dw), _ptr(dx), _ptr(dWq),
                                 _ptr(dbn), _ptr(dsubkeys), _ptr(workspace),
                                 _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_query_grad")


def pkm_selftest_wait_timeout(budget_cycles: int = 2_000_000, stream=None) -> None:
    _check(load().pkm_selftest_wait_timeout(int(budget_cycles), _stream(stream)),
           "pkm_selftest_wait_timeout")


def pkm_launch_count() -> int:
    return int(load().pkm_launch_count())


def pkm_query(dims: Dims, x, Wq, bn, saved: dict, stream=None) -> None:
    s = _saved_c(saved)
    _check(load().pkm_query(ctypes.byref(dims.c()), _ptr(x), _ptr(Wq), _ptr(bn), ctypes.byref(s),
                            _stream(stream)), "pkm_query")


def pkm_subkey_scores(dims: Dims, subkeys, saved: dict, stream=None) -> None:
    s = _saved_c(saved)
    _check(load().pkm_subkey_scores(ctypes.byref(dims.c()), _ptr(subkeys), ctypes.byref(s),
                                    _stream(stream)), "pkm_subkey_scores")


def pkm_candidate_topk(dims: Dims, saved: dict, stream=None) -> None:
    s = _saved_c(saved)
    _check(load().pkm_candidate_topk(ctypes.byref(dims.c()), ctypes.byref(s), _stream(stream)),
           "pkm_candidate_topk")


def pkm_gather_bag(dims: Dims, values, idx, w, y, stream=None) -> None:
    _check(load().pkm_gather_bag(ctypes.byref(dims.c()), _ptr(values), _ptr(idx), _ptr(w), _ptr(y),
                                 _stream(stream)), "pkm_gather_bag")


def pkm_check_status(stream=None) -> int:
    """Synchronise the stream and return the device status code (0 = PKM_OK)."""
    return int(load().pkm_check_status(_stream(stream)))


def pkm_build_info() -> str:
    return load().pkm_build_info().decode()


# ----------------------------------------------------------------- allocation helpers
def alloc_saved(dims: Dims, device="cuda", with_qhat: bool = True) -> dict:
    """Caller-owned buffers the forward writes and the backward reads (torch)."""
    import torch
    N, hq = dims.N, dims.h * dims.dk
    ksel = dims.k * dims.k if dims.flags & PKM_F_ALL_K2 else dims.k
    fp32 = bool(dims.flags & PKM_F_FP32)
    q = (torch.empty(N, hq, dtype=torch.float32, device=device) if fp32 else
         torch.empty(2, N, hq, dtype=torch.bfloat16, device=device))
    return dict(
        q=q,
        qhat=torch.empty(N, hq, dtype=torch.float32, device=device) if with_qhat else None,
        sub_s=torch.empty(N, dims.h, 2, dims.k, dtype=torch.float32, device=device),
        sub_i=torch.empty(N, dims.h, 2, dims.k, dtype=torch.int32, device=device),
        idx=torch.empty(N, dims.h, ksel, dtype=torch.int32, device=device),
        w=torch.empty(N, dims.h, ksel, dtype=torch.float32, device=device),
        bn_batch=torch.empty(2, hq, dtype=torch.float32, device=device),
    )


def alloc_workspace(dims: Dims, which: int, device="cuda"):
    import torch
    n = pkm_workspace_bytes(dims, which)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- row-sharded table
# Triples travel as int32 tensors of shape [n, 3] (segment, row, bits of the fp32 weight),
# the layout of pkm_triple.

def pkm_shard_workspace_bytes(dims: Dims, G: int, which: int, n_triples: int = 0) -> int:
    return int(load().pkm_shard_workspace_bytes(ctypes.byref(dims.c()), int(G), int(which),
                                                int(n_triples)))


def pkm_shard_route(dims: Dims, G: int, rows_per_shard: int, idx, w, counts, segpos, send, perm,
                    workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    _check(load().pkm_shard_route(ctypes.byref(dims.c()), int(G), int(rows_per_shard), _ptr(idx),
                                  _ptr(w), _ptr(counts), _ptr(segpos), _ptr(send), _ptr(perm),
                                  _ptr(workspace), _ws(workspace, workspace_bytes),
                                  _stream(stream)), "pkm_shard_route")


def pkm_shard_bag(dims: Dims, G: int, shard_rows: int, recv_counts, n_triples: int,
                  n_segments: int, recv, values, partial, workspace=None,
                  workspace_bytes: int = 0, stream=None) -> None:
    _check(load().pkm_shard_bag(ctypes.byref(dims.c()), int(G), int(shard_rows),
                                _ptr(recv_counts), int(n_triples), int(n_segments), _ptr(recv),
                                _ptr(values), _ptr(partial), _ptr(workspace),
                                _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_shard_bag")


def pkm_shard_combine(dims: Dims, G: int, segpos, partial_recv, n_rows: int, y,
                      stream=None) -> None:
    _check(load().pkm_shard_combine(ctypes.byref(dims.c()), int(G), _ptr(segpos),
                                    _ptr(partial_recv), int(n_rows), _ptr(y), _stream(stream)),
           "pkm_shard_combine")


def pkm_shard_gather_dy(dims: Dims, G: int, segpos, dy, dy_send, n_rows: int,
                        stream=None) -> None:
    _check(load().pkm_shard_gather_dy(ctypes.byref(dims.c()), int(G), _ptr(segpos), _ptr(dy),
                                      _ptr(dy_send), int(n_rows), _stream(stream)),
           "pkm_shard_gather_dy")


def pkm_shard_value_grad(dims: Dims, G: int, shard_rows: int, recv_counts, n_triples: int,
                         n_segments: int, recv, values, dy_recv, dvalues, dw_recv,
                         workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    _check(load().pkm_shard_value_grad(ctypes.byref(dims.c()), int(G), int(shard_rows),
                                       _ptr(recv_counts), int(n_triples), int(n_segments),
                                       _ptr(recv), _ptr(values), _ptr(dy_recv), _ptr(dvalues),
                                       _ptr(dw_recv), _ptr(workspace),
                                       _ws(workspace, workspace_bytes), _stream(stream)),
           "pkm_shard_value_grad")


def pkm_shard_scatter_dw(dims: Dims, perm, dw_ret, dw, stream=None) -> None:
    _check(load().pkm_shard_scatter_dw(ctypes.byref(dims.c()), _ptr(perm), _ptr(dw_ret), _ptr(dw),
                                       _stream(stream)), "pkm_shard_scatter_dw")
