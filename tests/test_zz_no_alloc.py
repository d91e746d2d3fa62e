"""moe_permute_noalloc: the permute for callers that cannot give the library
scratch memory (a plugin or callback that only receives its own buffers, or
a loop that must not allocate while it runs).  Its histograms live in a
fixed device array inside the library instead of a caller workspace.

The GPU test calls it three times in a row through the C ABI, with different
routings, and checks each result against moe_permute with a workspace and
against the oracle's counting sort.  Outputs are integers and copied rows,
so they must match bit-exactly.  Every case has more than 32 chunks of 256
slots, so each one runs the multi-kernel permute whose histograms live in the
shared array; the second reuses the array after the first left its contents
there, and the third fills it to its last entry.  This file is collected
last, so a stop at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
import sparse_mixture_experts_rmsnorm_b200 as moe
from parity_helpers import capacity, expert_rows

HIST_LIMIT = 262144  # MOE_NOALLOC_HIST_INTS in include/moe.h


def _hist_ints(cfg):
    return cfg.n_experts * -(-cfg.n_tokens * cfg.top_k // 256)


def _routing(rng, n, e, k):
    # k distinct experts per token drawn with weights falling from 3 to 1
    # (Gumbel top-k), so that a capacity cut bites on the first experts
    logp = np.log(np.linspace(3.0, 1.0, e))
    keys = rng.gumbel(size=(n, e)) + logp
    return np.argsort(-keys, axis=1)[:, :k].astype(np.int32)


def _run(torch, cfg, idx_np, xn, noalloc):
    N, E, k, d = cfg.n_tokens, cfg.n_experts, cfg.top_k, cfg.d_model
    kw = dict(dtype=torch.int32, device="cuda")
    idx = torch.tensor(idx_np, **kw)
    offsets = torch.full((E + 1,), -7, **kw)
    slot_row = torch.full((N * k,), -7, **kw)
    row_token = torch.full((N * k,), -7, **kw)
    x_perm = torch.zeros(expert_rows(cfg), d, dtype=xn.dtype, device="cuda")
    if noalloc:
        moe.moe_permute_noalloc(cfg, idx, xn, offsets, slot_row, row_token, x_perm)
    else:
        ws = moe.workspace(cfg)
        moe.moe_permute(cfg, idx, xn, offsets, slot_row, row_token, x_perm, ws)
    torch.cuda.synchronize()
    R = int(offsets[-1])
    return offsets.cpu(), slot_row.cpu(), row_token[:R].cpu(), x_perm[:R].cpu()


@pytest.mark.gpu
def test_noalloc_permute_matches_workspace_permute_and_oracle_three_calls():
    import torch
    rng = np.random.default_rng(11)
    cases = [
        # DeepSeek-V3-shaped routing: 256 chunks, 65536 histogram entries
        moe.Config(n_tokens=8192, d_model=1024, n_experts=256, top_k=8, d_ff=64, dtype="bf16"),
        # a capacity cut on the multi-kernel path, after the first call filled the array
        moe.Config(n_tokens=8192, d_model=512, n_experts=64, top_k=4, d_ff=64, dtype="bf16", capacity_factor=1.1),
        # exactly at the array's size: 256 experts x 1024 chunks
        moe.Config(n_tokens=32768, d_model=64, n_experts=256, top_k=8, d_ff=64, dtype="bf16"),
    ]
    assert _hist_ints(cases[2]) == HIST_LIMIT
    for cfg in cases:
        assert -(-cfg.n_tokens * cfg.top_k // 256) > 32
        idx_np = _routing(rng, cfg.n_tokens, cfg.n_experts, cfg.top_k)
        xn = torch.randn(cfg.n_tokens, cfg.d_model, device="cuda").to(torch.bfloat16)
        got = _run(torch, cfg, idx_np, xn, noalloc=True)
        ref = _run(torch, cfg, idx_np, xn, noalloc=False)
        for g, r in zip(got, ref):
            assert torch.equal(g, r)
        # the oracle's stable counting sort of the same routing
        off, slot_row, row_token = oracle.permute(idx_np, cfg.n_experts, capacity(cfg))
        np.testing.assert_array_equal(got[0].numpy(), off)
        np.testing.assert_array_equal(got[1].numpy(), slot_row)
        np.testing.assert_array_equal(got[2].numpy(), row_token)
        assert torch.equal(got[3], xn.cpu()[torch.from_numpy(row_token)])
        if capacity(cfg) >= 0:
            assert (slot_row < 0).any()


def test_noalloc_permute_rejects_sizes_beyond_its_array():
    # 1024 experts x ceil(65536 * 8 / 256) chunks = 2 Mi entries > MOE_NOALLOC_HIST_INTS
    cfg = moe.Config(n_tokens=65536, d_model=64, n_experts=1024, top_k=8, d_ff=64, dtype="bf16").c()
    st = moe.library().moe_permute_noalloc(ctypes.byref(cfg), 256, 256, 256, 256, 256, 256, None)
    assert st == moe.MOE_ERR_WORKSPACE
    # one chunk past the limit is rejected too: 256 experts x 1025 chunks
    over = moe.Config(n_tokens=32769, d_model=64, n_experts=256, top_k=8, d_ff=64, dtype="bf16").c()
    st = moe.library().moe_permute_noalloc(ctypes.byref(over), 256, 256, 256, 256, 256, 256, None)
    assert st == moe.MOE_ERR_WORKSPACE
