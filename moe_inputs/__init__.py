"""Seeded synthetic inputs for the MoE-layer forward, on the host and on the GPU.

This module is shared by the CPU oracle's tests and by the CUDA path's tests
and benchmark.  It holds none of the method's arithmetic: it only produces
the layer's inputs (hidden states, RMSNorm scale, router, bias and expert
weights) from a counter-based hash (``gen.h``), bit-identically on the host
(``libmoe_gen_host.so``, gcc + OpenMP) and on the device
(``libmoe_gen_cuda.so``).  Any slice of any tensor can be regenerated from
its element indices, so the oracle can rebuild one expert's weights without
copying them off the GPU.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

from .configs import CONFIGS, LayerConfig, TensorSpec, layer_tensor_specs  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libmoe_gen_host.so")
CUDA_LIB = os.path.join(_HERE, "libmoe_gen_cuda.so")

NORMAL, UNIFORM, CONST = 0, 1, 2
F32, BF16 = 0, 1


def build(cuda: bool = True, verbose: bool = False) -> None:
    """Compile the host generator (gcc) and, if ``cuda``, the device one (nvcc)."""
    cmds = [["gcc", "-O3", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
             "-o", HOST_LIB, os.path.join(_HERE, "gen_host.c")]]
    if cuda:
        cmds.append(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                     "-Xcompiler", "-fPIC", "-shared", "-o", CUDA_LIB,
                     os.path.join(_HERE, "gen_cuda.cu")])
    for c in cmds:
        if verbose:
            print(" ".join(c))
        subprocess.check_call(c, cwd=_HERE)


_host = None
_cuda = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            build(cuda=False)
        lib = ctypes.CDLL(HOST_LIB)
        lib.moe_gen_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int,
                                          ctypes.c_float, ctypes.c_float, ctypes.c_int]
        lib.moe_gen_fill_host.restype = None
        lib.moe_gen_hash_host.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
        lib.moe_gen_hash_host.restype = ctypes.c_uint64
        _host = lib
    return _host


def _cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(CUDA_LIB):
            raise RuntimeError(f"{CUDA_LIB} is missing: run moe_inputs.build()")
        lib = ctypes.CDLL(CUDA_LIB)
        lib.moe_gen_fill_cuda.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int,
                                          ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_void_p]
        lib.moe_gen_fill_cuda.restype = ctypes.c_int
        _cuda = lib
    return _cuda


def dist_params(dist: str, a: float = 0.0, b: float = 0.0):
    """Map a distribution description to (code, p0, p1) as fp32 values.

    ``("normal", sigma)``: p0 = fl32(sigma*sqrt(3)/65536).
    ``("uniform", lo, hi)``: p0 = lo, p1 = fl32(hi - lo).
    ``("const", value)``: p0 = value.
    """
    if dist == "normal":
        return NORMAL, float(np.float32(a * math.sqrt(3.0) / 65536.0)), 0.0
    if dist == "uniform":
        lo, hi = np.float32(a), np.float32(b)
        return UNIFORM, float(lo), float(np.float32(hi - lo))
    if dist == "const":
        return CONST, float(np.float32(a)), 0.0
    raise ValueError(dist)


def hash64(seed: int, tensor_id: int, index: int) -> int:
    return int(_host_lib().moe_gen_hash_host(seed, tensor_id, index))


def fill_host(n: int, seed: int, tensor_id: int, dist, dtype: str, start: int = 0) -> np.ndarray:
    """Generate ``n`` elements (counter indices start..start+n-1) on the host.

    Returns float32 values; for ``dtype == "bf16"`` they are the bf16-rounded
    values widened exactly to float32.
    """
    code, p0, p1 = dist_params(*dist)
    if dtype == "f32":
        out = np.empty(n, dtype=np.float32)
        _host_lib().moe_gen_fill_host(out.ctypes.data, n, start, seed, tensor_id, code, p0, p1, F32)
        return out
    bits = np.empty(n, dtype=np.uint16)
    _host_lib().moe_gen_fill_host(bits.ctypes.data, n, start, seed, tensor_id, code, p0, p1, BF16)
    return bf16_bits_to_f32(bits)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even), returned widened to float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return bf16_bits_to_f32(u.astype(np.uint16))


def fill_device(t, seed: int, tensor_id: int, dist, start: int = 0) -> None:
    """Fill a contiguous CUDA tensor (float32 or bfloat16) in place."""
    import torch

    assert t.is_cuda and t.is_contiguous()
    code, p0, p1 = dist_params(*dist)
    if t.dtype == torch.float32:
        dt = F32
    elif t.dtype == torch.bfloat16:
        dt = BF16
    else:
        raise TypeError(t.dtype)
    stream = torch.cuda.current_stream(t.device).cuda_stream
    rc = _cuda_lib().moe_gen_fill_cuda(t.data_ptr(), t.numel(), start, seed, tensor_id, code,
                                       p0, p1, dt, stream)
    if rc != 0:
        raise RuntimeError(f"moe_gen_fill_cuda failed with cudaError {rc}")


# --------------------------------------------------------------------------
# Whole-layer inputs
# --------------------------------------------------------------------------

def _spec_dtype(cfg: LayerConfig, spec: TensorSpec) -> str:
    return "f32" if spec.fp32 else cfg.dtype


def host_tensor(cfg: LayerConfig, name: str, rows: slice | None = None) -> np.ndarray:
    """One layer input on the host as float32 (bf16 values widened exactly).

    ``rows`` selects a range of the leading dimension (e.g. one expert of a
    stacked expert weight) without generating the rest.
    """
    spec = layer_tensor_specs(cfg)[name]
    shape = spec.shape
    inner = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    r0, r1 = (0, shape[0]) if rows is None else (rows.start or 0, rows.stop if rows.stop is not None else shape[0])
    out = fill_host((r1 - r0) * inner, cfg.seed, spec.tensor_id, spec.dist, _spec_dtype(cfg, spec),
                    start=r0 * inner).reshape((r1 - r0,) + tuple(shape[1:]))
    return _apply_edits_host(cfg, name, out, r0)


def _apply_edits_host(cfg: LayerConfig, name: str, arr: np.ndarray, r0: int) -> np.ndarray:
    # Load-imbalance recipe: add a constant to feature 0 of every token and a
    # matching amount to router weight [skew_expert, 0]; one fp32 add, then
    # rounding to the storage dtype, on both sides.
    if cfg.skew is None:
        return arr
    expert, a, c = cfg.skew
    rnd = f32_to_bf16_f32 if cfg.dtype == "bf16" else (lambda v: v.astype(np.float32))
    if name == "h":
        arr[:, 0] = rnd((arr[:, 0].astype(np.float32) + np.float32(a)))
    elif name == "w_router" and r0 <= expert < r0 + arr.shape[0]:
        arr[expert - r0, 0] = rnd(np.array([np.float32(arr[expert - r0, 0]) + np.float32(c / a)],
                                           dtype=np.float32))[0]
    return arr


def device_tensors(cfg: LayerConfig, device="cuda", names=None) -> dict:
    """All layer inputs generated directly on the GPU (bit-identical to host_tensor)."""
    import torch

    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}
    out = {}
    for name, spec in layer_tensor_specs(cfg).items():
        if names is not None and name not in names:
            continue
        dt = torch.float32 if spec.fp32 else tdt[cfg.dtype]
        t = torch.empty(spec.shape, dtype=dt, device=device)
        if t.numel():
            fill_device(t, cfg.seed, spec.tensor_id, spec.dist)
        out[name] = t
    if cfg.skew is not None:
        expert, a, c = cfg.skew
        if "h" in out:
            h = out["h"]
            h[:, 0] = (h[:, 0].float() + torch.tensor(a, dtype=torch.float32, device=device)).to(h.dtype)
        if "w_router" in out:
            w = out["w_router"]
            w[expert, 0] = (w[expert, 0].float() + torch.tensor(np.float32(c / a), device=device)).to(w.dtype)
    return out
