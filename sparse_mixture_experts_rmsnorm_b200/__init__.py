"""Python binding of libmoe_b200.so, the B200 (sm_100a) MoE-layer forward.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are passed as device pointers (``data_ptr()``), the
stream is the current torch stream unless one is given, and every call
raises :class:`MoEError` when the library returns an error status.  There is
no fallback: importing this package fails when the library is missing.

The layer (the MoE block of the "Mixture of Experts (MoE)" lesson, AI
Engineering from Scratch, Phase 07):

    xn  = RMSNorm(h)
    out = h + sum over the top-k experts of gate_e * SwiGLU_e(xn) [+ SwiGLU_shared(xn)]

with selection on softmax score + bias and gates from the raw scores
renormalised over the k chosen experts.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT = range(6)
MOE_F32, MOE_BF16 = 0, 1

# Every entry point declared in include/moe.h, in declaration order.
ENTRY_POINTS = (
    "moe_status_string", "moe_version", "moe_workspace_size", "moe_workspace_init", "moe_route", "moe_route_hash",
    "moe_permute", "moe_permute_noalloc", "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_bias_update",
    "moe_compute_load_stats", "moe_check_device_error", "moe_set_wait_timeout_ns", "moe_set_gemm_tiling",
    "moe_selftest_wait_timeout",
)


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.moe_status_string(status).decode()}")


class MoeConfig(ctypes.Structure):
    _fields_ = [("n_tokens", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("rms_eps", ctypes.c_float), ("capacity_factor", ctypes.c_float)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("norm_w", "w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")]


class MoeRouting(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("scores", "topk_idx", "topk_gate", "counts", "offsets", "slot_row", "row_token")]


class MoeTrace(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("start", "routed", "permuted", "gate_up", "down", "shared", "combined")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python sparse_mixture_experts_rmsnorm_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    cfgp = ctypes.POINTER(MoeConfig)
    sig = {
        "moe_status_string": (ctypes.c_char_p, [I32]),
        "moe_version": (ctypes.c_char_p, []),
        "moe_workspace_size": (SZ, [cfgp]),
        "moe_workspace_init": (I32, [P, SZ, P]),
        "moe_route": (I32, [cfgp, P, P, P, P, P, P, P, P, P, P, SZ, P]),
        "moe_route_hash": (I32, [cfgp, P, P, P, P, P, P, P, P, SZ, P]),
        "moe_permute": (I32, [cfgp, P, P, P, P, P, P, P, SZ, P]),
        "moe_permute_noalloc": (I32, [cfgp, P, P, P, P, P, P, P]),
        "moe_expert_ffn": (I32, [cfgp, I32, P, I32, P, P, P, P, I32, P, P, SZ, P]),
        "moe_combine": (I32, [cfgp, P, P, P, P, P, P, P]),
        "moe_layer_forward": (I32, [cfgp, ctypes.POINTER(MoeWeights), P, P, P, ctypes.POINTER(MoeRouting),
                                    ctypes.POINTER(MoeTrace), P, SZ, P]),
        "moe_bias_update": (I32, [I32, P, F, F, P, P]),
        "moe_compute_load_stats": (I32, [cfgp, P, P, P, P]),
        "moe_check_device_error": (I32, [P, SZ, P, P]),
        "moe_set_wait_timeout_ns": (I32, [I64]),
        "moe_set_gemm_tiling": (I32, [I32]),
        "moe_selftest_wait_timeout": (I32, [P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library():
    """The loaded ctypes library (for callers that want the raw C ABI)."""
    return _lib


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _torch_stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream()
    if isinstance(stream, int):
        return torch.cuda.ExternalStream(stream)
    return stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


@dataclass
class Config:
    """Layer shape and options (mirrors ``moe_config``)."""
    n_tokens: int
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    d_ff_shared: int = 0
    dtype: str = "bf16"            # "bf16" or "f32"
    rms_eps: float = 1e-6
    capacity_factor: float = 0.0   # <= 0: no capacity limit

    def c(self) -> MoeConfig:
        return MoeConfig(self.n_tokens, self.d_model, self.n_experts, self.top_k, self.d_ff, self.d_ff_shared,
                         MOE_BF16 if self.dtype == "bf16" else MOE_F32, self.rms_eps, self.capacity_factor)


def workspace_size(cfg: Config) -> int:
    return int(_lib.moe_workspace_size(ctypes.byref(cfg.c())))


def workspace(cfg: Config, device="cuda", stream=None):
    """Allocate (through torch) and initialise a workspace for ``cfg``."""
    import torch
    n = workspace_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(_lib.moe_workspace_init(ws.data_ptr(), n, _stream(stream)), "moe_workspace_init")
    return ws


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def moe_route(cfg: Config, h, norm_w, w_router, bias, xn, scores, topk_idx, topk_gate, counts, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(cfg.c()), _ptr(h), _ptr(norm_w), _ptr(w_router), _ptr(bias), _ptr(xn),
                          _ptr(scores), _ptr(topk_idx), _ptr(topk_gate), _ptr(counts), _ptr(ws), ws.numel(),
                          _stream(stream)), "moe_route")


def moe_route_hash(cfg: Config, h, norm_w, token_ids, xn, topk_idx, topk_gate, counts, ws, stream=None):
    """RMSNorm, then routing by a SplitMix64 hash of each token id (token_ids: int64
    tensor or None for the token's position); gates 1/k."""
    _check(_lib.moe_route_hash(ctypes.byref(cfg.c()), _ptr(h), _ptr(norm_w), _ptr(token_ids), _ptr(xn),
                               _ptr(topk_idx), _ptr(topk_gate), _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_route_hash")


def moe_permute(cfg: Config, topk_idx, xn, offsets, slot_row, row_token, x_perm, ws, stream=None):
    _check(_lib.moe_permute(ctypes.byref(cfg.c()), _ptr(topk_idx), _ptr(xn), _ptr(offsets), _ptr(slot_row),
                            _ptr(row_token), _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg: Config, topk_idx, xn, offsets, slot_row, row_token, x_perm, stream=None):
    """moe_permute without a workspace (the histograms use the library's fixed
    1 MiB device array; calls that overlap on the GPU race)."""
    _check(_lib.moe_permute_noalloc(ctypes.byref(cfg.c()), _ptr(topk_idx), _ptr(xn), _ptr(offsets), _ptr(slot_row),
                                    _ptr(row_token), _ptr(x_perm), _stream(stream)), "moe_permute_noalloc")


def moe_expert_ffn(cfg: Config, n_groups: int, offsets, max_rows: int, x, w_gate, w_up, w_down, d_ff: int, y, ws,
                   stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(cfg.c()), n_groups, _ptr(offsets), max_rows, _ptr(x), _ptr(w_gate),
                               _ptr(w_up), _ptr(w_down), d_ff, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_expert_ffn")


def moe_combine(cfg: Config, h, y_perm, slot_row, topk_gate, y_shared, out, stream=None):
    _check(_lib.moe_combine(ctypes.byref(cfg.c()), _ptr(h), _ptr(y_perm), _ptr(slot_row), _ptr(topk_gate),
                            _ptr(y_shared), _ptr(out), _stream(stream)), "moe_combine")


def _weights_struct(w: dict) -> MoeWeights:
    return MoeWeights(*[_ptr(w.get(n)) for n in
                        ("norm_w", "w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")])


def moe_layer_forward(cfg: Config, weights: dict, h, bias, out, ws, routing: dict | None = None,
                      trace: dict | None = None, stream=None):
    """The whole layer on one stream.  ``routing``: optional dict of device
    output tensors (scores, topk_idx, topk_gate, counts, offsets, slot_row,
    row_token); ``trace``: optional dict of torch.cuda.Event per stage."""
    w = _weights_struct(weights)
    r = None
    if routing is not None:
        r = MoeRouting(*[_ptr(routing.get(n)) for n in
                         ("scores", "topk_idx", "topk_gate", "counts", "offsets", "slot_row", "row_token")])
    tr = None
    if trace is not None:
        handles = []
        for n in ("start", "routed", "permuted", "gate_up", "down", "shared", "combined"):
            ev = trace.get(n)
            if ev is not None and not ev.cuda_event:
                ev.record(_torch_stream(stream))  # torch creates its events lazily, on the first record
            handles.append(ev.cuda_event if ev is not None else None)
        tr = MoeTrace(*handles)
    _check(_lib.moe_layer_forward(ctypes.byref(cfg.c()), ctypes.byref(w), _ptr(h), _ptr(bias), _ptr(out),
                                  ctypes.byref(r) if r is not None else None,
                                  ctypes.byref(tr) if tr is not None else None,
                                  _ptr(ws), ws.numel(), _stream(stream)), "moe_layer_forward")


def moe_bias_update(n_experts: int, counts, target: float, gamma: float, bias, stream=None):
    _check(_lib.moe_bias_update(n_experts, _ptr(counts), target, gamma, _ptr(bias), _stream(stream)),
           "moe_bias_update")


class MoeLoadStats(ctypes.Structure):
    """Host view of one moe_load_stats (20 bytes)."""
    _fields_ = [("routed", ctypes.c_int32), ("kept", ctypes.c_int32), ("dropped", ctypes.c_int32),
                ("max_count", ctypes.c_int32), ("max_over_mean", ctypes.c_float)]


def moe_compute_load_stats(cfg: Config, counts, offsets, stats, stream=None):
    """stats: a device buffer of at least ctypes.sizeof(MoeLoadStats) bytes."""
    _check(_lib.moe_compute_load_stats(ctypes.byref(cfg.c()), _ptr(counts), _ptr(offsets), _ptr(stats),
                                       _stream(stream)), "moe_compute_load_stats")


def moe_check_device_error(ws, stream=None):
    """Synchronise, read and clear the workspace's device error record.
    Returns (status, [status, kernel id, block, wait site])."""
    info = (ctypes.c_int32 * 4)()
    st = _lib.moe_check_device_error(_ptr(ws), ws.numel(), _stream(stream), info)
    return int(st), list(info)


def moe_set_wait_timeout_ns(ns: int):
    _check(_lib.moe_set_wait_timeout_ns(int(ns)), "moe_set_wait_timeout_ns")


def moe_set_gemm_tiling(mode: int):
    """0 = automatic, 1 = single-SM 128-row tiles, 2 = SM-pair 256-row tiles,
    3 = operands swapped on SM pairs (weight rows on M, each group's rows on N)."""
    _check(_lib.moe_set_gemm_tiling(int(mode)), "moe_set_gemm_tiling")


def moe_selftest_wait_timeout(ws, stream=None):
    _check(_lib.moe_selftest_wait_timeout(_ptr(ws), ws.numel(), _stream(stream)), "moe_selftest_wait_timeout")


def version() -> str:
    return _lib.moe_version().decode()
