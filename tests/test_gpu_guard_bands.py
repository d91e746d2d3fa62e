"""Out-of-bounds write checks without a sanitizer: guard bands.

Every buffer the library writes (the layer output, each routing output, the
staged calls' outputs and the workspace) is placed between two 4 KiB bands of
a known byte inside one larger allocation.  After the layer forward and the
staged calls, every band byte must be unchanged.  The workloads reach each
kernel path: the CUDA-core fp32 GEMMs, the swapped-operand and single-SM
tcgen05 GEMMs, the folded and the separate shared expert, the tensor-core
router (128- and 256-column tiles), capacity drops, the bulk-copy and the
column-split row scatter, and d_model and d_ff that are not multiples of 64.  Parity of the values is
checked by the other GPU tests.
"""
import numpy as np
import pytest

import moe_inputs as mi
from parity_helpers import expert_rows, lib_config

pytestmark = pytest.mark.gpu

BAND = 4096   # bytes on each side; keeps every buffer 256-byte aligned
FILL = 0xA5

CASES = {
    "fp32 CUDA-core GEMMs, shared expert, capacity":
        mi.CONFIGS["tiny_fp32"].with_(d_ff_shared=96, capacity_factor=0.75, skew=(4, 8.0, 3.0), seed=3),
    "bf16 swapped GEMMs, separate shared expert, capacity":
        mi.LayerConfig(name="g1", n_tokens=700, d_model=256, n_experts=16, top_k=4, d_ff=192, d_ff_shared=128,
                       capacity_factor=1.0, router_sigma=0.1, seed=4),
    "bf16 folded shared expert, bulk-copy scatter":
        mi.LayerConfig(name="g2", n_tokens=300, d_model=512, n_experts=32, top_k=4, d_ff=128, d_ff_shared=128,
                       seed=5),
    "bf16 decode-sized, M = 64 tiles, column-split rows":
        mi.LayerConfig(name="g3", n_tokens=64, d_model=512, n_experts=64, top_k=8, d_ff=128, d_ff_shared=128,
                       bias=("uniform", -0.01, 0.01), seed=6),
    "bf16 tensor-core router":
        mi.LayerConfig(name="g4", n_tokens=600, d_model=256, n_experts=128, top_k=4, d_ff=64, seed=7),
    "bf16 tensor-core router, 256-column tiles":
        mi.LayerConfig(name="g6", n_tokens=16384, d_model=256, n_experts=256, top_k=8, d_ff=64, seed=9),
    "bf16 d_model and d_ff not multiples of 64":
        mi.LayerConfig(name="g5", n_tokens=400, d_model=200, n_experts=8, top_k=2, d_ff=136, d_ff_shared=72,
                       capacity_factor=1.1, seed=8),
}


class Guarded:
    """Tensors carved out of band-wrapped allocations."""

    def __init__(self, torch):
        self.torch = torch
        self.bufs = []

    def tensor(self, shape, dtype):
        torch = self.torch
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        buf = torch.full((n + 2 * BAND,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, n))
        return buf[BAND:BAND + n].view(dtype).view(*shape)

    def workspace(self, nbytes):
        torch = self.torch
        buf = torch.full((nbytes + 2 * BAND,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, nbytes))
        return buf[BAND:BAND + nbytes]

    def check(self, what):
        self.torch.cuda.synchronize()
        for i, (buf, n) in enumerate(self.bufs):
            bands = self.torch.cat([buf[:BAND], buf[BAND + n:]]).cpu().numpy()
            bad = np.nonzero(bands != FILL)[0]
            assert bad.size == 0, f"{what}: buffer {i} written outside its bounds at band bytes {bad[:8]}"


@pytest.mark.parametrize("name", list(CASES))
def test_no_write_outside_any_buffer(torch_cuda, name):
    torch = torch_cuda
    import sparse_mixture_experts_rmsnorm_b200 as moe
    cfg = CASES[name]
    lc = lib_config(cfg)
    dev = mi.device_tensors(cfg)
    N, d, E, k, H, Hs = cfg.n_tokens, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff, cfg.d_ff_shared
    R = expert_rows(cfg)
    act = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    i32, f32 = torch.int32, torch.float32
    weights = {n: dev[n] for n in ("norm_w", "w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")
               if n in dev}

    # the whole layer, every routing output returned
    g = Guarded(torch)
    ws = g.workspace(moe.workspace_size(lc))
    assert moe.library().moe_workspace_init(ws.data_ptr(), ws.numel(), None) == moe.MOE_OK
    routing = {"scores": g.tensor((N, E), f32), "topk_idx": g.tensor((N, k), i32),
               "topk_gate": g.tensor((N, k), f32), "counts": g.tensor((E,), i32),
               "offsets": g.tensor((E + 1,), i32), "slot_row": g.tensor((N * k,), i32),
               "row_token": g.tensor((N * k,), i32)}
    out = g.tensor((N, d), act)
    moe.moe_layer_forward(lc, weights, dev["h"], dev["bias"], out, ws, routing=routing)
    g.check("moe_layer_forward")
    st, info = moe.moe_check_device_error(ws)
    assert st == 0, info

    # the staged calls, each output guarded
    s = Guarded(torch)
    ws2 = s.workspace(moe.workspace_size(lc))
    assert moe.library().moe_workspace_init(ws2.data_ptr(), ws2.numel(), None) == moe.MOE_OK
    xn = s.tensor((N, d), act)
    idx, gate, counts = s.tensor((N, k), i32), s.tensor((N, k), f32), s.tensor((E,), i32)
    moe.moe_route(lc, dev["h"], dev["norm_w"], dev["w_router"], dev["bias"], xn, s.tensor((N, E), f32), idx, gate,
                  counts, ws2)
    offsets, slot_row, row_token = s.tensor((E + 1,), i32), s.tensor((N * k,), i32), s.tensor((N * k,), i32)
    x_perm = s.tensor((R, d), act)
    moe.moe_permute(lc, idx, xn, offsets, slot_row, row_token, x_perm, ws2)
    y = s.tensor((R, d), act)
    moe.moe_expert_ffn(lc, E, offsets, R, x_perm, dev["w_gate"], dev["w_up"], dev["w_down"], H, y, ws2)
    y_shared = None
    if Hs:
        y_shared = s.tensor((N, d), act)
        moe.moe_expert_ffn(lc, 1, None, N, xn, dev["ws_gate"], dev["ws_up"], dev["ws_down"], Hs, y_shared, ws2)
    out2 = s.tensor((N, d), act)
    moe.moe_combine(lc, dev["h"], y, slot_row, gate, y_shared, out2)
    s.check("staged calls")
    st, info = moe.moe_check_device_error(ws2)
    assert st == 0, info
    # the two paths agree on the routing (their values are compared to the oracle elsewhere)
    assert torch.equal(idx, routing["topk_idx"]) and torch.equal(slot_row, routing["slot_row"])
