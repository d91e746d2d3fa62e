"""Shared pieces of the GPU parity tests: running the CUDA path through the C
ABI on seeded inputs, and the oracle's expected values for the same inputs.

The oracle side regenerates every input on the host from the counter-based
generator, so no expected value is derived from a device tensor.
"""
from __future__ import annotations

import numpy as np

import moe_inputs as mi
import oracle

# Routing comparisons skip tokens whose oracle keys are this close: the
# tolerance stated for this layer.  test_gpu_configs also checks that every
# fp32 key lies within KEY_TIE of the oracle's on each workload (largest errors
# measured on B200: 6.6e-7 for the tensor-core router, 8.9e-7 on the CUDA cores).
KEY_TIE = 1e-6
BF16_REL_RMS = 2e-2     # bf16 layers: max |gpu - oracle| / rms(oracle)
F32_MAX_ABS = 1e-4      # fp32 layer: max |gpu - oracle|


def capacity(cfg) -> int:
    """The oracle's per-expert capacity of a workload or library config (-1: none)."""
    return oracle.capacity_limit(cfg.capacity_factor, cfg.n_tokens, cfg.top_k, cfg.n_experts)


def expert_rows(cfg) -> int:
    """Rows of the expert-sorted buffers: N*k, or at most E*capacity with a capacity."""
    r, cap = cfg.n_tokens * cfg.top_k, capacity(cfg)
    return r if cap < 0 else min(r, cfg.n_experts * cap)


def lib_config(cfg: mi.LayerConfig):
    import sparse_mixture_experts_rmsnorm_b200 as moe
    return moe.Config(cfg.n_tokens, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.d_ff_shared,
                      cfg.dtype, cfg.rms_eps, cfg.capacity_factor)


def to_np(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def run_gpu_layer(cfg: mi.LayerConfig, dev=None, with_route: bool = True) -> dict:
    """Run moe_route (for xn and scores) and moe_layer_forward on the GPU.

    Returns numpy copies of the routing outputs, xn, the layer output and
    the input h, plus the device tensors under "dev".
    """
    import torch
    import sparse_mixture_experts_rmsnorm_b200 as moe

    lc = lib_config(cfg)
    if dev is None:
        dev = mi.device_tensors(cfg)
    N, d, E, k = cfg.n_tokens, cfg.d_model, cfg.n_experts, cfg.top_k
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    ws = moe.workspace(lc)
    r = {"scores": torch.empty(N, E, **f32), "topk_idx": torch.empty(N, k, **i32),
         "topk_gate": torch.empty(N, k, **f32), "counts": torch.empty(E, **i32),
         "offsets": torch.empty(E + 1, **i32), "slot_row": torch.empty(N * k, **i32),
         "row_token": torch.empty(max(N * k, 1), **i32)}
    out = torch.empty_like(dev["h"])
    res = {}
    if with_route:
        xn = torch.empty_like(dev["h"])
        idx2 = torch.empty(N, k, **i32)
        g2 = torch.empty(N, k, **f32)
        c2 = torch.empty(E, **i32)
        moe.moe_route(lc, dev["h"], dev["norm_w"], dev["w_router"], dev["bias"], xn, r["scores"], idx2, g2, c2, ws)
        res.update(xn=to_np(xn), route_idx=to_np(idx2), route_gate=to_np(g2), route_counts=to_np(c2))
    weights = {n: dev[n] for n in ("norm_w", "w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")
               if n in dev}
    moe.moe_layer_forward(lc, weights, dev["h"], dev["bias"], out, ws, routing=r)
    torch.cuda.synchronize()
    st, info = moe.moe_check_device_error(ws)
    assert st == 0, (st, info)
    for n, t in r.items():
        res[n] = to_np(t)
    res["row_token"] = res["row_token"][: int(res["offsets"][-1])]
    res["out"] = to_np(out)
    res["dev"] = dev
    res["ws"] = ws
    return res


def oracle_routing(cfg: mi.LayerConfig) -> dict:
    """xn, scores, keys, chosen experts and gates for every token (host)."""
    h = mi.host_tensor(cfg, "h")
    xn = oracle.rmsnorm(h, mi.host_tensor(cfg, "norm_w"), cfg.rms_eps, cfg.dtype)
    _, scores = oracle.router_scores(xn, mi.host_tensor(cfg, "w_router"))
    idx, key = oracle.select_topk(scores, mi.host_tensor(cfg, "bias"), cfg.top_k)
    gates = oracle.gates_from_scores(scores, idx)
    return {"h": h, "xn": xn, "scores": scores, "key": key, "idx": idx, "gates": gates}


def tie_masks(key: np.ndarray, k: int):
    """(set_ambiguous, order_ambiguous) per token.

    set_ambiguous: the k-th and (k+1)-th largest keys are within KEY_TIE, so
    the chosen set may legitimately differ.  order_ambiguous: any two
    consecutive keys among the top k (+1) are within KEY_TIE, so the order of
    the chosen experts may differ too.
    """
    srt = -np.sort(-key.astype(np.float64), axis=1)
    E = key.shape[1]
    set_amb = np.zeros(key.shape[0], dtype=bool)
    if k < E:
        set_amb = (srt[:, k - 1] - srt[:, k]) < KEY_TIE
    top = srt[:, : min(k + 1, E)]
    order_amb = np.any(np.diff(-top, axis=1) < KEY_TIE, axis=1) if top.shape[1] > 1 else set_amb
    return set_amb, order_amb | set_amb


def check_routing(gpu: dict, ref: dict, k: int, gate_tol: float = 1e-5):
    """Chosen experts bit-exact (set and order) outside the near-tie tokens;
    gates close; counts consistent.  Returns the number of skipped tokens."""
    set_amb, order_amb = tie_masks(ref["key"], k)
    ok = ~order_amb
    gi, ri = gpu["topk_idx"].astype(np.int64), ref["idx"].astype(np.int64)
    bad = np.nonzero(ok & np.any(gi != ri, axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens route differently, e.g. token {bad[:5]}: gpu {gi[bad[:3]]} ref {ri[bad[:3]]}"
    same_set = ~set_amb
    gs, rs = np.sort(gi, axis=1), np.sort(ri, axis=1)
    assert np.array_equal(gs[same_set], rs[same_set])
    np.testing.assert_allclose(gpu["topk_gate"][ok], ref["gates"][ok], rtol=0, atol=gate_tol)
    assert np.all(gpu["topk_gate"] >= 0)
    np.testing.assert_allclose(gpu["topk_gate"].astype(np.float64).sum(1), 1.0, atol=2e-6)
    E = ref["scores"].shape[1]
    counts = np.bincount(gi.ravel(), minlength=E)
    assert np.array_equal(gpu["counts"].astype(np.int64), counts)
    assert counts.sum() == gi.size
    return int(order_amb.sum())


def check_permutation(gpu: dict, E: int, capacity: int):
    """offsets / slot_row / row_token bit-exact against the oracle's counting
    sort of the GPU's own chosen experts (the permutation is a function of
    them alone)."""
    off, slot_row, row_token = oracle.permute(gpu["topk_idx"], E, capacity)
    assert np.array_equal(gpu["offsets"].astype(np.int64), off)
    assert np.array_equal(gpu["slot_row"].astype(np.int64), slot_row)
    assert np.array_equal(gpu["row_token"].astype(np.int64), row_token)
    return off, slot_row


def expert_weights(cfg: mi.LayerConfig, e: int):
    sl = slice(e, e + 1)
    return (mi.host_tensor(cfg, "w_gate", rows=sl)[0], mi.host_tensor(cfg, "w_up", rows=sl)[0],
            mi.host_tensor(cfg, "w_down", rows=sl)[0])


def oracle_outputs(cfg: mi.LayerConfig, ref: dict, tokens, idx, gates, keep) -> np.ndarray:
    """out64 of the given tokens (rows of the result follow `tokens`).

    idx, gates, keep: [N, k] routing, gates and kept-slot mask to use.
    """
    tokens = np.asarray(tokens)
    xn = ref["xn"][tokens]
    y = np.zeros((tokens.size, cfg.top_k, cfg.d_model))
    experts = np.unique(idx[tokens])
    for e in experts.tolist():
        sel_t, sel_j = np.nonzero((idx[tokens] == e) & keep[tokens])
        if sel_t.size == 0:
            continue
        wg, wu, wd = expert_weights(cfg, e)
        y[sel_t, sel_j] = oracle.swiglu_expert(xn[sel_t], wg, wu, wd, cfg.dtype)
    y_shared = None
    if cfg.d_ff_shared > 0:
        y_shared = oracle.swiglu_expert(xn, mi.host_tensor(cfg, "ws_gate"), mi.host_tensor(cfg, "ws_up"),
                                        mi.host_tensor(cfg, "ws_down"), cfg.dtype)
    slot_row = np.where(keep[tokens], 0, -1).ravel()
    return oracle.combine(ref["h"][tokens], y, gates[tokens], slot_row, y_shared)


def rel_rms_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / rms(ref)."""
    return float(np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref ** 2)))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x|: the largest error of rounding an exact
    value to bf16 storage (8 significant bits: x in [2^e, 2^(e+1)) has
    spacing 2^(e-7))."""
    _, e = np.frexp(np.abs(np.asarray(x, dtype=np.float64)))  # |x| = m 2^e, 0.5 <= m < 1
    return np.ldexp(1.0, e - 9)


def bf16_rel_rms_err(got: np.ndarray, ref64: np.ndarray) -> float:
    """Error of a bf16-stored result against the unrounded float64 oracle,
    beyond the half-ulp that storing even the exact value in bf16 costs:
    max(0, |got - ref| - half_ulp(ref)) / rms(ref)."""
    excess = np.maximum(np.abs(got - ref64) - bf16_half_ulp(ref64), 0.0)
    return float(np.max(excess) / np.sqrt(np.mean(ref64 ** 2)))
