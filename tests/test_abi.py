"""The C ABI without a GPU: the library loads, exports every entry point that
include/moe.h declares, sizes workspaces and rejects bad arguments on the
host before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_rmsnorm_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    declared = _declared_functions()
    assert len(declared) >= 13
    lib = ctypes.CDLL(moe.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(moe.ENTRY_POINTS) == declared


def test_status_strings_and_version():
    lib = moe.library()
    for st in range(6):
        assert lib.moe_status_string(st).decode().startswith("MOE_")
    assert "sm_100a" in moe.version()


def _cfg(**kw):
    base = dict(n_tokens=256, d_model=64, n_experts=8, top_k=2, d_ff=128, dtype="f32")
    base.update(kw)
    return moe.Config(**base)


def test_workspace_size_grows_with_shape_and_rejects_bad_configs():
    a = moe.workspace_size(_cfg())
    assert a > 0 and a % 256 == 0
    assert moe.workspace_size(_cfg(n_tokens=512)) > a
    assert moe.workspace_size(_cfg(d_ff_shared=64)) > a
    # capacity shrinks the expert-sorted buffers
    assert moe.workspace_size(_cfg(capacity_factor=0.5)) < a
    for bad in (dict(top_k=9), dict(top_k=0), dict(n_experts=0), dict(n_experts=2000, top_k=2),
                dict(d_model=0), dict(n_tokens=-1), dict(d_ff=0), dict(top_k=33, n_experts=64)):
        assert moe.workspace_size(_cfg(**bad)) == 0, bad


def test_workspace_bytes_match_the_documented_regions():
    N, d, E, k, H, Hs = 1000, 512, 16, 4, 384, 256
    routing = N * E * 4 + 4 * N * k * 4  # logits, idx, gate, slot_row, row_token
    # bf16: xn, routing, x_perm, act, y_perm, y_shared
    c = _cfg(dtype="bf16", n_tokens=N, d_model=d, n_experts=E, top_k=k, d_ff=H, d_ff_shared=Hs)
    R = N * k  # no capacity: every slot keeps a row
    need = N * d * 2 + routing + 2 * R * d * 2 + max(R * H, N * Hs) * 2 + N * d * 2
    assert need <= moe.workspace_size(c) <= need + 64 * 1024
    # fp32: the same regions in 4-byte elements
    f = _cfg(dtype="f32", n_tokens=N, d_model=d, n_experts=E, top_k=k, d_ff=H, d_ff_shared=Hs)
    need32 = N * d * 4 + routing + 2 * R * d * 4 + max(R * H, N * Hs) * 4 + N * d * 4
    assert need32 <= moe.workspace_size(f) <= need32 + 64 * 1024
    # bf16 with a shared expert as wide as the routed ones: it is one more
    # group of N rows in act and y_perm (its input rows are read from xn), and
    # there is no separate y_shared
    g = _cfg(dtype="bf16", n_tokens=N, d_model=d, n_experts=E, top_k=k, d_ff=H, d_ff_shared=H)
    need_f = N * d * 2 + routing + R * d * 2 + (R + N) * d * 2 + (R + N) * H * 2
    assert need_f <= moe.workspace_size(g) <= need_f + 64 * 1024


def test_host_validation_before_any_launch():
    lib = moe.library()
    bad = _cfg(top_k=9).c()
    st = lib.moe_route(ctypes.byref(bad), None, None, None, None, None, None, None, None, None, None, 0, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    good = _cfg().c()
    # a workspace pointer that is not 256-byte aligned
    st = lib.moe_route(ctypes.byref(good), 16, 16, 16, None, 16, None, 16, 16, 16, 16 + 8, 1 << 30, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # a workspace smaller than moe_workspace_size
    st = lib.moe_route(ctypes.byref(good), 256, 256, 256, None, 256, None, 256, 256, 256, 256, 1024, None)
    assert st == moe.MOE_ERR_WORKSPACE
    # bf16 rows that are not whole 16-byte units
    odd = _cfg(dtype="bf16", d_model=60).c()
    st = lib.moe_permute(ctypes.byref(odd), 256, 256, 256, 256, 256, 256, 256, 1 << 30, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    # expert FFN: group count and act capacity
    st = lib.moe_expert_ffn(ctypes.byref(good), 0, None, 16, 256, 256, 256, 256, 128, 256, 256, 1 << 30, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    st = lib.moe_expert_ffn(ctypes.byref(good), 2, None, 16, 256, 256, 256, 256, 128, 256, 256, 1 << 30, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    st = lib.moe_expert_ffn(ctypes.byref(good), 1, None, 100000, 256, 256, 256, 256, 128, 256, 256, 1 << 30, None)
    assert st == moe.MOE_ERR_WORKSPACE
    assert lib.moe_bias_update(0, 256, 1.0, 1e-3, 256, None) == moe.MOE_ERR_INVALID_ARG
    # load statistics: a NULL buffer or a bad config
    assert lib.moe_compute_load_stats(ctypes.byref(good), 256, None, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_compute_load_stats(ctypes.byref(bad), 256, 256, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert ctypes.sizeof(moe.MoeLoadStats) == 20
    # combine: the expert rows are required while any slot can be kept
    st = lib.moe_combine(ctypes.byref(good), 256, None, 256, 256, None, 256, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    st = lib.moe_combine(ctypes.byref(good), None, 256, 256, 256, None, 256, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_wait_timeout_ns(-1) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_check_device_error(None, 0, None, None) == moe.MOE_ERR_INVALID_ARG
    for mode in (-1, 4, 1 << 20):
        assert lib.moe_set_gemm_tiling(mode) == moe.MOE_ERR_INVALID_ARG
    for mode in (1, 2, 3, 0):  # accepted; host state only, no launch
        assert lib.moe_set_gemm_tiling(mode) == moe.MOE_OK


def test_python_wrapper_raises_on_error_status():
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_set_wait_timeout_ns(-5)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    moe.moe_set_wait_timeout_ns(2_000_000_000)
