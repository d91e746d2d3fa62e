"""The hash router on the GPU ("Mixture of Experts (MoE)" lesson, exercise:
a router that routes by a hash instead of a learned linear layer).

Routing must equal the oracle's SplitMix64 routing bit for bit; the layer
built from moe_route_hash, moe_permute, moe_expert_ffn and moe_combine must
match the oracle's layer with the same routing within the bf16 tolerance.
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from parity_helpers import BF16_REL_RMS, bf16_rel_rms_err, lib_config, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("with_ids", [False, True])
def test_hash_routing_bit_exact(with_ids):
    import torch
    import sparse_mixture_experts_rmsnorm_b200 as moe
    cfg = mi.LayerConfig(name="hash", n_tokens=3000, d_model=256, n_experts=24, top_k=3, d_ff=64, seed=2)
    lc = lib_config(cfg)
    dev = mi.device_tensors(cfg, names=["h", "norm_w"])
    rng = np.random.default_rng(1)
    ids = rng.integers(-(1 << 62), 1 << 62, size=cfg.n_tokens, dtype=np.int64) if with_ids else None
    ws = moe.workspace(lc)
    N, k, E = cfg.n_tokens, cfg.top_k, cfg.n_experts
    xn = torch.empty_like(dev["h"])
    idx = torch.empty(N, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(N, k, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    moe.moe_route_hash(lc, dev["h"], dev["norm_w"], torch.tensor(ids, device="cuda") if with_ids else None,
                       xn, idx, gate, counts, ws)
    torch.cuda.synchronize()
    ref_idx, ref_gate = oracle.hash_route(ids if with_ids else np.arange(N), E, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    assert np.array_equal(gate.cpu().numpy().view(np.uint32), ref_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), np.bincount(ref_idx.ravel(), minlength=E))
    ref_xn = oracle.rmsnorm(mi.host_tensor(cfg, "h"), mi.host_tensor(cfg, "norm_w"), cfg.rms_eps, cfg.dtype)
    np.testing.assert_array_equal(to_np(xn), ref_xn)


def test_hash_routed_layer_through_the_staged_calls():
    import torch
    import sparse_mixture_experts_rmsnorm_b200 as moe
    cfg = mi.LayerConfig(name="hash", n_tokens=700, d_model=512, n_experts=16, top_k=2, d_ff=384, seed=6)
    lc = lib_config(cfg)
    dev = mi.device_tensors(cfg)
    N, k, E, d, H = cfg.n_tokens, cfg.top_k, cfg.n_experts, cfg.d_model, cfg.d_ff
    ws = moe.workspace(lc)
    kw = dict(device="cuda")
    xn = torch.empty_like(dev["h"])
    idx = torch.empty(N, k, dtype=torch.int32, **kw)
    gate = torch.empty(N, k, **kw)
    counts = torch.empty(E, dtype=torch.int32, **kw)
    moe.moe_route_hash(lc, dev["h"], dev["norm_w"], None, xn, idx, gate, counts, ws)
    offsets = torch.empty(E + 1, dtype=torch.int32, **kw)
    slot_row = torch.empty(N * k, dtype=torch.int32, **kw)
    row_token = torch.empty(N * k, dtype=torch.int32, **kw)
    x_perm = torch.empty(N * k, d, dtype=torch.bfloat16, **kw)
    moe.moe_permute(lc, idx, xn, offsets, slot_row, row_token, x_perm, ws)
    y = torch.empty(N * k, d, dtype=torch.bfloat16, **kw)
    moe.moe_expert_ffn(lc, E, offsets, N * k, x_perm, dev["w_gate"], dev["w_up"], dev["w_down"], H, y, ws)
    out = torch.empty_like(dev["h"])
    moe.moe_combine(lc, dev["h"], y, slot_row, gate, None, out)
    torch.cuda.synchronize()

    a = {n: mi.host_tensor(cfg, n) for n in mi.layer_tensor_specs(cfg)}
    ref_xn = oracle.rmsnorm(a["h"], a["norm_w"], cfg.rms_eps, cfg.dtype)
    ref_idx, ref_gate = oracle.hash_route(np.arange(N), E, k)
    _, ref_slot, _ = oracle.permute(ref_idx, E)
    np.testing.assert_array_equal(slot_row.cpu().numpy(), ref_slot)
    ys = np.zeros((N, k, d))
    for e in range(E):
        t_idx, j_idx = np.nonzero(ref_idx == e)
        if t_idx.size:
            ys[t_idx, j_idx] = oracle.swiglu_expert(ref_xn[t_idx], a["w_gate"][e], a["w_up"][e], a["w_down"][e],
                                                    cfg.dtype)
    ref_out = oracle.combine(a["h"], ys, ref_gate.astype(np.float64), ref_slot)
    err = bf16_rel_rms_err(to_np(out), ref_out)
    print(f"hash-routed layer: beyond-storage max err/rms {err:.3e}")
    assert err <= BF16_REL_RMS, err
