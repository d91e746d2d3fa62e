"""moe_permute_noalloc: the permute for callers that cannot give the library
scratch memory (a plugin or callback that only receives its own buffers, or
a loop that must not allocate while it runs).  Its histograms live in a
fixed device array inside the library instead of a caller workspace.

The GPU test calls it twice in a row through the C ABI, with different
routings, and checks each result against moe_permute with a workspace.
Outputs are integers and copied rows, so they must match bit-exactly.
This file is collected last, so a stop at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest

import sparse_mixture_experts_rmsnorm_b200 as moe


def _routing(rng, n, e, k):
    # k distinct experts per token, skewed so that a capacity cut bites
    p = np.linspace(3.0, 1.0, e)
    p /= p.sum()
    return np.stack([rng.choice(e, size=k, replace=False, p=p) for _ in range(n)]).astype(np.int32)


def _run(torch, cfg, idx_np, xn, noalloc):
    N, E, k, d = cfg.n_tokens, cfg.n_experts, cfg.top_k, cfg.d_model
    kw = dict(dtype=torch.int32, device="cuda")
    idx = torch.tensor(idx_np, **kw)
    offsets = torch.full((E + 1,), -7, **kw)
    slot_row = torch.full((N * k,), -7, **kw)
    row_token = torch.full((N * k,), -7, **kw)
    x_perm = torch.zeros(cfg.rows, d, dtype=xn.dtype, device="cuda")
    if noalloc:
        moe.moe_permute_noalloc(cfg, idx, xn, offsets, slot_row, row_token, x_perm)
    else:
        ws = moe.workspace(cfg)
        moe.moe_permute(cfg, idx, xn, offsets, slot_row, row_token, x_perm, ws)
    torch.cuda.synchronize()
    R = int(offsets[-1])
    return offsets.cpu(), slot_row.cpu(), row_token[:R].cpu(), x_perm[:R].cpu()


@pytest.mark.gpu
def test_noalloc_permute_matches_workspace_permute_twice():
    import torch
    rng = np.random.default_rng(11)
    cases = [
        moe.Config(n_tokens=8192, d_model=7168, n_experts=256, top_k=8, d_ff=2048, dtype="bf16"),
        moe.Config(n_tokens=3000, d_model=512, n_experts=8, top_k=2, d_ff=64, dtype="bf16", capacity_factor=1.1),
    ]
    for cfg in cases:  # two calls in a row, the second after the first filled the shared array
        idx_np = _routing(rng, cfg.n_tokens, cfg.n_experts, cfg.top_k)
        xn = torch.randn(cfg.n_tokens, cfg.d_model, device="cuda").to(torch.bfloat16)
        got = _run(torch, cfg, idx_np, xn, noalloc=True)
        ref = _run(torch, cfg, idx_np, xn, noalloc=False)
        for g, r in zip(got, ref):
            assert torch.equal(g, r)
        counts = np.bincount(idx_np.ravel(), minlength=cfg.n_experts)
        kept = counts if cfg.capacity < 0 else np.minimum(counts, cfg.capacity)
        assert int(got[0][-1]) == int(kept.sum())


def test_noalloc_permute_rejects_sizes_beyond_its_array():
    # 1024 experts x ceil(65536 * 8 / 256) chunks = 2 Mi entries > MOE_NOALLOC_HIST_INTS
    cfg = moe.Config(n_tokens=65536, d_model=64, n_experts=1024, top_k=8, d_ff=64, dtype="bf16").c()
    st = moe.library().moe_permute_noalloc(ctypes.byref(cfg), 256, 256, 256, 256, 256, 256, None)
    assert st == moe.MOE_ERR_WORKSPACE
