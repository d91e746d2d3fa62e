"""GPU parity of the MoE-layer forward against the CPU oracle, through the C ABI.

Every test here needs a B200 (sm_100a).  Routing, counts, permutation and
drop masks are compared bit-exactly (tokens whose oracle selection keys are
within KEY_TIE = 1e-6 of each other are skipped); outputs within max-abs 1e-4 (fp32
layer) or 2e-2 of the output RMS (bf16 layers, fp32 accumulation); bias
updates bit-exactly.
"""
import json
import os

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from parity_helpers import (BF16_REL_RMS, F32_MAX_ABS, bf16_rel_rms_err, capacity, check_permutation,
                            check_routing, lib_config, oracle_routing, rel_rms_err, run_gpu_layer, tie_masks, to_np)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _full_oracle(cfg):
    a = {n: mi.host_tensor(cfg, n) for n in mi.layer_tensor_specs(cfg)}
    return oracle.layer_forward(a["h"], a["norm_w"], a["w_router"], a["bias"], a["w_gate"], a["w_up"],
                                a["w_down"], top_k=cfg.top_k, eps=cfg.rms_eps, dtype=cfg.dtype,
                                capacity_factor=cfg.capacity_factor, ws_gate=a.get("ws_gate"),
                                ws_up=a.get("ws_up"), ws_down=a.get("ws_down"))


# ----------------------------------------------------------------- generator

def test_device_generator_matches_host(torch_cuda):
    cfg = mi.CONFIGS["dsv3_decode_bf16"]
    dev = mi.device_tensors(cfg, names=["h", "bias", "w_router"])
    for n in ("h", "bias", "w_router"):
        np.testing.assert_array_equal(to_np(dev[n]).astype(np.float32), mi.host_tensor(cfg, n))


# ----------------------------------------------------------------- tiny fp32, whole layer

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_fp32_layer_matches_oracle(torch_cuda, seed):
    cfg = mi.CONFIGS["tiny_fp32"].with_(seed=seed)
    g = run_gpu_layer(cfg)
    ref = _full_oracle(cfg)
    np.testing.assert_array_equal(g["xn"], ref["xn"])
    skipped = check_routing(g, {"key": ref["key"], "idx": ref["idx"], "gates": ref["gates"],
                                "scores": ref["scores"]}, cfg.top_k)
    assert skipped == 0
    check_permutation(g, cfg.n_experts, -1)
    err = np.max(np.abs(g["out"] - ref["out64"]))
    assert err <= F32_MAX_ABS, err


def test_tiny_fp32_staged_calls_equal_layer_forward(torch_cuda):
    torch = torch_cuda
    import sparse_mixture_experts_rmsnorm_b200 as moe
    cfg = mi.CONFIGS["tiny_fp32"]
    lc = lib_config(cfg)
    dev = mi.device_tensors(cfg)
    g = run_gpu_layer(cfg, dev=dev)
    N, d, E, k, H = cfg.n_tokens, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff
    ws = moe.workspace(lc)
    kw = dict(device="cuda")
    xn = torch.empty(N, d, **kw)
    idx = torch.empty(N, k, dtype=torch.int32, **kw)
    gate = torch.empty(N, k, **kw)
    counts = torch.empty(E, dtype=torch.int32, **kw)
    moe.moe_route(lc, dev["h"], dev["norm_w"], dev["w_router"], None, xn, None, idx, gate, counts, ws)
    offsets = torch.empty(E + 1, dtype=torch.int32, **kw)
    slot_row = torch.empty(N * k, dtype=torch.int32, **kw)
    row_token = torch.empty(N * k, dtype=torch.int32, **kw)
    x_perm = torch.empty(N * k, d, **kw)
    moe.moe_permute(lc, idx, xn, offsets, slot_row, row_token, x_perm, ws)
    y = torch.full((N * k, d), float("nan"), **kw)
    moe.moe_expert_ffn(lc, E, offsets, N * k, x_perm, dev["w_gate"], dev["w_up"], dev["w_down"], H, y, ws)
    out = torch.empty(N, d, **kw)
    moe.moe_combine(lc, dev["h"], y, slot_row, gate, None, out, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(idx), g["topk_idx"])
    np.testing.assert_array_equal(to_np(slot_row), g["slot_row"])
    np.testing.assert_array_equal(to_np(out), g["out"])
    # x_perm rows are the tokens' xn rows
    np.testing.assert_array_equal(to_np(x_perm), to_np(xn)[g["row_token"]])


def test_tiny_fp32_layer_with_shared_expert_and_capacity(torch_cuda):
    # the CUDA-core path with an always-on shared expert and dropped slots
    cfg = mi.CONFIGS["tiny_fp32"].with_(d_ff_shared=96, capacity_factor=0.75, skew=(4, 8.0, 3.0), seed=3)
    g = run_gpu_layer(cfg)
    ref = _full_oracle(cfg)
    check_routing(g, {"key": ref["key"], "idx": ref["idx"], "gates": ref["gates"], "scores": ref["scores"]},
                  cfg.top_k)
    check_permutation(g, cfg.n_experts, capacity(cfg))
    assert (g["slot_row"] < 0).any()
    err = np.max(np.abs(g["out"] - ref["out64"]))
    assert err <= F32_MAX_ABS, err


def test_single_expert_and_dense_identities(torch_cuda):
    # E = 1, k = 1: the textbook SwiGLU FFN; k = E (zero bias): dense softmax-weighted sum.
    for over in (dict(n_experts=1, top_k=1), dict(n_experts=4, top_k=4), dict(n_experts=8, top_k=8)):
        cfg = mi.CONFIGS["tiny_fp32"].with_(**over)
        g = run_gpu_layer(cfg)
        ref = _full_oracle(cfg)
        assert np.all(g["counts"] == cfg.n_tokens)
        err = np.max(np.abs(g["out"] - ref["out64"]))
        assert err <= F32_MAX_ABS, (over, err)


def test_exact_ties_choose_lower_expert_index(torch_cuda):
    torch = torch_cuda
    cfg = mi.CONFIGS["tiny_fp32"].with_(n_tokens=64)
    dev = mi.device_tensors(cfg)
    dev["w_router"].zero_()  # every logit 0: all scores equal
    g = run_gpu_layer(cfg, dev=dev)
    assert np.all(g["topk_idx"] == np.array([[0, 1]]))
    np.testing.assert_array_equal(g["topk_gate"], 0.5)
    # a bias breaks the tie in favour of experts 5 and 2
    dev["bias"].copy_(torch.tensor([0, 0, 1e-3, 0, 0, 2e-3, 0, 0], dtype=torch.float32))
    g = run_gpu_layer(cfg, dev=dev)
    assert np.all(g["topk_idx"] == np.array([[5, 2]]))
    np.testing.assert_array_equal(g["topk_gate"], 0.5)


def test_empty_input_is_a_no_op(torch_cuda):
    cfg = mi.CONFIGS["tiny_fp32"].with_(n_tokens=0)
    g = run_gpu_layer(cfg)
    assert g["out"].shape == (0, cfg.d_model)
    assert np.all(g["counts"] == 0) and np.all(g["offsets"] == 0)


# ----------------------------------------------------------------- permutation on the printed example

@pytest.mark.parametrize("capacity_factor,expect_offsets", [
    (0.0, [0, 1, 3, 4, 7, 7, 7, 10, 12]),
    (1.4, [0, 1, 3, 4, 6, 6, 6, 8, 10]),   # cap = floor(1.4 * 6 * 2 / 8) = 2
])
def test_glossary_example_permutation(torch_cuda, capacity_factor, expect_offsets):
    torch = torch_cuda
    import sparse_mixture_experts_rmsnorm_b200 as moe
    fx = json.load(open(os.path.join(GOLDEN, "glossary_top2_example.json")))
    N, E, k, d = fx["n_tokens"], fx["n_experts"], fx["top_k"], 16
    lc = moe.Config(N, d, E, k, 16, dtype="bf16", capacity_factor=capacity_factor)
    ws = moe.workspace(lc)
    idx = torch.tensor(fx["experts_per_token"], dtype=torch.int32, device="cuda")
    xn = torch.arange(N * d, dtype=torch.float32, device="cuda").reshape(N, d).to(torch.bfloat16)
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    slot_row = torch.empty(N * k, dtype=torch.int32, device="cuda")
    row_token = torch.empty(N * k, dtype=torch.int32, device="cuda")
    x_perm = torch.zeros(N * k, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(lc, idx, xn, offsets, slot_row, row_token, x_perm, ws)
    torch.cuda.synchronize()
    off = offsets.cpu().tolist()
    assert off == expect_offsets
    cap = capacity(lc)
    ref_off, ref_slot, ref_rt = oracle.permute(np.array(fx["experts_per_token"]), E, cap)
    assert off == ref_off.tolist()
    assert slot_row.cpu().tolist() == ref_slot.tolist()
    assert row_token.cpu().tolist()[: off[-1]] == ref_rt.tolist()
    rows = x_perm[: off[-1]].float().cpu().numpy()
    np.testing.assert_array_equal(rows, xn.float().cpu().numpy()[ref_rt])


# ----------------------------------------------------------------- tcgen05 grouped GEMM, ragged shapes

def _ffn_case(torch, groups_rows, d, H, seed, with_offsets=True):
    import sparse_mixture_experts_rmsnorm_b200 as moe
    G = len(groups_rows)
    R = int(sum(groups_rows))
    r = np.random.default_rng(seed)
    bf = lambda a: oracle.round_to(a, "bf16")
    x = bf(r.standard_normal((R + 7, d)))
    wg = bf(r.standard_normal((G, H, d)) * 0.05)
    wu = bf(r.standard_normal((G, H, d)) * 0.05)
    wd = bf(r.standard_normal((G, d, H)) * 0.05)
    dev = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda").to(torch.bfloat16).contiguous()
    lc = moe.Config(n_tokens=max(R, 1), d_model=d, n_experts=G, top_k=1, d_ff=H, dtype="bf16")
    ws = moe.workspace(lc)
    offs = np.concatenate([[0], np.cumsum(groups_rows)]).astype(np.int32)
    y = torch.full((R + 7, d), 77.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(lc, G, torch.tensor(offs, device="cuda") if with_offsets else None, R, dev(x), dev(wg),
                       dev(wu), dev(wd), H, y, ws)
    torch.cuda.synchronize()
    st, info = moe.moe_check_device_error(ws)
    assert st == 0, info
    got = to_np(y)
    ref = np.zeros((R, d))
    for g in range(G):
        a, b = offs[g], offs[g + 1]
        if b > a:
            ref[a:b] = oracle.swiglu_expert(x[a:b], wg[g], wu[g], wd[g], "bf16")
    assert np.all(got[R:] == 77.0), "rows past the last group were written"
    return got[:R], ref


@pytest.fixture
def gemm_tiling():
    import sparse_mixture_experts_rmsnorm_b200 as moe

    def set_mode(mode):
        moe.moe_set_gemm_tiling(mode)
    yield set_mode
    moe.moe_set_gemm_tiling(0)


# 1: single-SM 128-row tiles, 2: SM-pair 256-row tiles, 3: operands swapped on SM pairs
# (weight rows on M, each group's rows on N in chunks of at most 256 rounded to 16)
@pytest.mark.parametrize("mode", [1, 2, 3])
@pytest.mark.parametrize("rows,d,H", [
    ([0, 130, 77, 1, 256], 192, 200),      # ragged groups, empty group, partial tiles, 3 k-blocks
    ([300], 4096, 512),                    # one group, many k-blocks
    ([5, 0, 0, 129, 64], 520, 1032),       # K and N not multiples of the tile
    ([700, 1300, 0, 513, 256], 256, 384),  # groups spanning several SM-pair tiles (and 2-6 chunks)
    ([17, 255, 257, 2049, 8], 136, 72),    # chunk edges: 255/257 rows, 9 chunks, one row box of 8
])
def test_expert_ffn_tc_matches_oracle(torch_cuda, gemm_tiling, rows, d, H, mode):
    gemm_tiling(mode)
    got, ref = _ffn_case(torch_cuda, rows, d, H, seed=len(rows) + d)
    err = bf16_rel_rms_err(got, ref)
    print(f"expert FFN tiling {mode} {rows} d={d} H={H}: beyond-storage max err/rms {err:.3e}, "
          f"raw {rel_rms_err(got, ref):.3e}")
    assert err <= BF16_REL_RMS, err


@pytest.mark.parametrize("mode", [1, 2, 3])
def test_expert_ffn_tc_single_group_smaller_than_a_tile(torch_cuda, gemm_tiling, mode):
    gemm_tiling(mode)
    got, ref = _ffn_case(torch_cuda, [64], 256, 256, seed=5, with_offsets=False)
    assert bf16_rel_rms_err(got, ref) <= BF16_REL_RMS


@pytest.mark.parametrize("rows,d,H", [
    # the load-imbalance workload's kept rows per expert: single-SM tiles take
    # fewer waves at d = 4096 (16 column tiles), so the device picks them
    ([629, 726, 586, 1280, 565, 766, 343, 615], 4096, 136),
    # the same groups at d = 256 fit one wave either way: SM pairs are picked
    ([629, 726, 586, 1280, 565, 766, 343, 615], 256, 136),
])
def test_down_projection_tiling_picked_on_the_device(torch_cuda, gemm_tiling, rows, d, H):
    # groups averaging >= 512 rows with H % 64 != 0 (the swapped-operand kernel
    # declines): the down projection launches both other tilings and the
    # device keeps one from the offsets; the output is the oracle's
    gemm_tiling(0)
    got, ref = _ffn_case(torch_cuda, rows, d, H, seed=13)
    assert bf16_rel_rms_err(got, ref) <= BF16_REL_RMS


def test_both_tilings_agree_closely(torch_cuda, gemm_tiling):
    # same products, summation order aside
    gemm_tiling(1)
    a, ref = _ffn_case(torch_cuda, [600, 900], 512, 640, seed=9)
    for mode in (2, 3):
        gemm_tiling(mode)
        b, _ = _ffn_case(torch_cuda, [600, 900], 512, 640, seed=9)
        assert rel_rms_err(a, b) <= 2e-2
        assert bf16_rel_rms_err(b, ref) <= BF16_REL_RMS


@pytest.mark.parametrize("mode", [1, 3])
def test_folded_shared_expert_many_groups(torch_cuda, gemm_tiling, mode):
    # 32 experts of about 200 rows plus a folded shared expert of N rows, the
    # DeepSeek-V3 prefill's per-expert shape in small: modes 1 and 3 force the
    # single-SM and the swapped-operand kernel on the same layer
    gemm_tiling(mode)
    cfg = mi.LayerConfig(name="fold32", n_tokens=800, d_model=256, n_experts=32, top_k=8, d_ff=128,
                         d_ff_shared=128, bias=("uniform", -0.01, 0.01), seed=6)
    g = run_gpu_layer(cfg)
    ref = _full_oracle(cfg)
    check_routing(g, {"key": ref["key"], "idx": ref["idx"], "gates": ref["gates"], "scores": ref["scores"]},
                  cfg.top_k)
    err = bf16_rel_rms_err(g["out"], ref["out64"])
    print(f"folded shared expert, 32 groups, tiling {mode}: beyond-storage max err/rms {err:.3e}")
    assert err <= BF16_REL_RMS, err


# ----------------------------------------------------------------- router on the tensor cores

# 777 tokens run 128-column router tiles; 16424 tokens with 256 experts run
# 256-column ones (fewer waves), the last of 129 row tiles 40 rows (M = 64)
@pytest.mark.parametrize("E,k,N", [(64, 6, 777), (256, 8, 777), (256, 8, 16424)])
def test_router_tc_routing_bit_exact(torch_cuda, E, k, N):
    cfg = mi.LayerConfig(name="router", n_tokens=N, d_model=1024, n_experts=E, top_k=k, d_ff=64,
                         bias=("uniform", -0.01, 0.01), seed=3)
    g = run_gpu_layer(cfg)
    ref = oracle_routing(cfg)
    np.testing.assert_array_equal(g["xn"], ref["xn"])
    np.testing.assert_allclose(g["scores"], ref["scores"], rtol=2e-5, atol=1e-9)
    skipped = check_routing(g, ref, k)
    assert skipped < 0.02 * cfg.n_tokens
    check_permutation(g, E, -1)


# ----------------------------------------------------------------- bias update

def test_bias_update_bit_exact(torch_cuda):
    torch = torch_cuda
    import sparse_mixture_experts_rmsnorm_b200 as moe
    r = np.random.default_rng(7)
    E = 300
    counts = r.integers(0, 2048, size=E).astype(np.int32)
    counts[:5] = 1024
    bias = (r.standard_normal(E) * 1e-2).astype(np.float32)
    b = torch.tensor(bias, device="cuda")
    moe.moe_bias_update(E, torch.tensor(counts, device="cuda"), 1024.0, 1e-3, b)
    got = b.cpu().numpy()
    ref = oracle.bias_update(bias, counts, 1024.0, 1e-3)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------------- load statistics

@pytest.mark.parametrize("capacity_factor", [0.0, 1.0])
def test_load_stats_match_oracle(torch_cuda, capacity_factor):
    torch = torch_cuda
    import ctypes
    import sparse_mixture_experts_rmsnorm_b200 as moe
    cfg = mi.LayerConfig(name="stats", n_tokens=1000, d_model=256, n_experts=16, top_k=4, d_ff=64,
                         capacity_factor=capacity_factor, router_sigma=0.1, seed=5)
    E = cfg.n_experts
    g = run_gpu_layer(cfg, with_route=False)
    # the expected statistics come from the oracle's counts and permutation of
    # the GPU's chosen experts (the routing itself is compared elsewhere)
    idx = g["topk_idx"]
    offsets, _, _ = oracle.permute(idx, E, capacity(cfg))
    ref = oracle.load_stats(oracle.expert_counts(idx, E), offsets, cfg.n_tokens, cfg.top_k, E)
    stats = torch.zeros(ctypes.sizeof(moe.MoeLoadStats), dtype=torch.uint8, device="cuda")
    moe.moe_compute_load_stats(lib_config(cfg), torch.tensor(g["counts"], device="cuda"),
                               torch.tensor(g["offsets"], device="cuda"), stats)
    got = moe.MoeLoadStats.from_buffer_copy(bytes(stats.cpu().numpy()))
    assert (got.routed, got.kept, got.dropped, got.max_count) == (ref["routed"], ref["kept"], ref["dropped"],
                                                                  ref["max_count"])
    assert np.float32(got.max_over_mean).view(np.uint32) == ref["max_over_mean"].view(np.uint32)
    assert (got.dropped > 0) == (capacity_factor > 0)

    # no tokens: every field zero
    empty = cfg.with_(n_tokens=0)
    z = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    stats.fill_(0xFF)
    moe.moe_compute_load_stats(lib_config(empty), z, z, stats)
    got = moe.MoeLoadStats.from_buffer_copy(bytes(stats.cpu().numpy()))
    assert (got.routed, got.kept, got.dropped, got.max_count, got.max_over_mean) == (0, 0, 0, 0, 0.0)


# ----------------------------------------------------------------- bounded device wait

def test_device_wait_times_out_and_reports(torch_cuda):
    torch = torch_cuda
    import sparse_mixture_experts_rmsnorm_b200 as moe
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_set_wait_timeout_ns(2_000_000)  # 2 ms
    try:
        moe.moe_selftest_wait_timeout(ws)
        st, info = moe.moe_check_device_error(ws)
    finally:
        moe.moe_set_wait_timeout_ns(2_000_000_000)
    assert st == moe.MOE_ERR_DEVICE_TIMEOUT
    assert info[0] == moe.MOE_ERR_DEVICE_TIMEOUT and info[1] == 2
    st, info = moe.moe_check_device_error(ws)
    assert st == 0 and info[0] == 0
    # the context is still usable
    x = torch.ones(16, device="cuda")
    assert float(x.sum()) == 16.0


# ----------------------------------------------------------------- small bf16 layers, every output

@pytest.mark.parametrize("over", [
    dict(n_tokens=300, d_model=256, n_experts=16, top_k=4, d_ff=192, d_ff_shared=128),
    dict(n_tokens=515, d_model=512, n_experts=8, top_k=2, d_ff=264, capacity_factor=0.9,
         skew=(5, 8.0, 2.0)),
    dict(n_tokens=97, d_model=128, n_experts=64, top_k=6, d_ff=64, d_ff_shared=64,
         bias=("uniform", -0.01, 0.01)),
    # shared expert as wide as the routed ones (it runs inside the routed GEMMs) plus drops
    dict(n_tokens=400, d_model=256, n_experts=8, top_k=2, d_ff=128, d_ff_shared=128, capacity_factor=0.8,
         skew=(2, 8.0, 2.5)),
    # capacity 0: every routed slot dropped, the folded shared expert alone adds to h
    dict(n_tokens=64, d_model=128, n_experts=16, top_k=2, d_ff=64, d_ff_shared=64, capacity_factor=0.05),
    # few tokens, wide rows: the row scatter and the combine split each row over
    # 3 (top-2, two column blocks per pass) and 2 (top-6) column ranges
    dict(n_tokens=40, d_model=2560, n_experts=8, top_k=2, d_ff=64),
    dict(n_tokens=33, d_model=1544, n_experts=16, top_k=6, d_ff=64, d_ff_shared=64, capacity_factor=0.9),
])
def test_small_bf16_layer_every_output(torch_cuda, over):
    cfg = mi.LayerConfig(name="small", dtype="bf16", seed=4, **over)
    g = run_gpu_layer(cfg)
    ref = _full_oracle(cfg)
    np.testing.assert_array_equal(g["xn"], ref["xn"])
    check_routing(g, {"key": ref["key"], "idx": ref["idx"], "gates": ref["gates"], "scores": ref["scores"]},
                  cfg.top_k)
    check_permutation(g, cfg.n_experts, capacity(cfg))
    err = bf16_rel_rms_err(g["out"], ref["out64"])
    print(f"small bf16 layer {over}: beyond-storage max err/rms {err:.3e}")
    assert err <= BF16_REL_RMS, err
    dropped_all = np.nonzero((g["slot_row"].reshape(cfg.n_tokens, cfg.top_k) < 0).all(axis=1))[0]
    if cfg.d_ff_shared == 0 and dropped_all.size:
        np.testing.assert_array_equal(g["out"][dropped_all], ref["h"][dropped_all] if "h" in ref else
                                      mi.host_tensor(cfg, "h")[dropped_all])


@pytest.mark.parametrize("mode", [1, 2])  # single-SM tiles, SM-pair tiles
def test_folded_shared_expert_in_both_tilings(torch_cuda, gemm_tiling, mode):
    # the shared expert runs as the last group of the routed GEMMs and reads
    # its input rows from xn through its own tensor map, in either kernel
    gemm_tiling(mode)
    cfg = mi.LayerConfig(name="fold", dtype="bf16", seed=7, n_tokens=700, d_model=256, n_experts=8, top_k=2,
                         d_ff=192, d_ff_shared=192)
    g = run_gpu_layer(cfg)
    ref = _full_oracle(cfg)
    err = bf16_rel_rms_err(g["out"], ref["out64"])
    print(f"folded shared expert, tiling {mode}: beyond-storage max err/rms {err:.3e}")
    assert err <= BF16_REL_RMS, err


# ----------------------------------------------------------------- the forward pass as a CUDA graph

# the last case is the DeepSeek-V3 prefill's per-expert shape on 32 experts: the
# swapped-operand GEMMs, the router on the tensor cores and the multi-kernel permute
@pytest.mark.parametrize("name", ["tiny_fp32", "dsv3_decode_bf16", "dsv3_prefill_bf16:32x1024"])
def test_layer_forward_replays_from_a_cuda_graph(torch_cuda, name):
    # moe_layer_forward enqueues work on one stream with no host synchronisation,
    # so a captured graph replays the identical computation
    torch = torch_cuda
    import sparse_mixture_experts_rmsnorm_b200 as moe
    base, _, size = name.partition(":")
    cfg = mi.CONFIGS[base]
    if size:
        e, n = (int(v) for v in size.split("x"))
        cfg = cfg.with_(n_experts=e, n_tokens=n)
    lc = lib_config(cfg)
    dev = mi.device_tensors(cfg)
    w = {n: dev[n] for n in ("norm_w", "w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")
         if n in dev}
    ws = moe.workspace(lc)
    eager = torch.empty_like(dev["h"])
    moe.moe_layer_forward(lc, w, dev["h"], dev["bias"], eager, ws)  # also warms every kernel up
    torch.cuda.synchronize()
    out = torch.zeros_like(dev["h"])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_forward(lc, w, dev["h"], dev["bias"], out, ws)
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    st, info = moe.moe_check_device_error(ws)
    assert st == 0, info


# ----------------------------------------------------------------- the largest routing the ABI allows

@pytest.mark.parametrize("n_tokens", [300, 700])  # router on the CUDA cores, then on the tensor cores
def test_route_with_1024_experts_and_top_32(torch_cuda, n_tokens):
    # with 1024 experts neighbouring keys often fall within KEY_TIE of each other:
    # those tokens are compared as sets only (check_routing), and such ties are
    # counted here
    cfg = mi.LayerConfig(name="wide", n_tokens=n_tokens, d_model=256, n_experts=1024, top_k=32, d_ff=64,
                         bias=("uniform", -1e-4, 1e-4), router_sigma=0.1, seed=8)
    g = run_gpu_layer(cfg)
    ref = oracle_routing(cfg)
    np.testing.assert_array_equal(g["xn"], ref["xn"])
    np.testing.assert_allclose(g["scores"], ref["scores"], rtol=2e-5, atol=1e-10)
    set_amb, _ = tie_masks(ref["key"], cfg.top_k)
    skipped = check_routing(g, ref, cfg.top_k)
    assert set_amb.mean() < 0.05 and skipped < 0.25 * n_tokens, (set_amb.mean(), skipped)
    check_permutation(g, cfg.n_experts, -1)


# ----------------------------------------------------------------- wide rows: the router's shared-memory limit grows

def test_route_rows_wider_than_48k_of_shared_memory_in_growing_order(torch_cuda):
    # the fused RMSNorm + router kernel keeps a row in shared memory; a later
    # call with a wider row must raise the kernel's limit again
    for d in (12800, 16384):  # 51,200 then 65,536 bytes of fp32 row
        cfg = mi.LayerConfig(name="wide_rows", dtype="f32", n_tokens=8, d_model=d, n_experts=8, top_k=2, d_ff=64,
                             seed=11)
        g = run_gpu_layer(cfg)
        ref = _full_oracle(cfg)
        np.testing.assert_allclose(g["xn"], ref["xn"], rtol=2e-6, atol=1e-7)
        check_routing(g, {"key": ref["key"], "idx": ref["idx"], "gates": ref["gates"], "scores": ref["scores"]},
                      cfg.top_k)
        check_permutation(g, cfg.n_experts, -1)
        err = np.max(np.abs(g["out"] - ref["out64"]))
        assert err <= F32_MAX_ABS, (d, err)


def test_fp32_layer_with_rows_split_over_blocks(torch_cuda):
    # 20 tokens of 1028 fp32 columns: the combine splits each row into 3 column
    # ranges (344, 344 and 340 wide); the output must not depend on the split
    cfg = mi.LayerConfig(name="split_rows", dtype="f32", n_tokens=20, d_model=1028, n_experts=8, top_k=2, d_ff=64,
                         seed=12)
    g = run_gpu_layer(cfg)
    ref = _full_oracle(cfg)
    check_permutation(g, cfg.n_experts, -1)
    err = np.max(np.abs(g["out"] - ref["out64"]))
    assert err <= F32_MAX_ABS, err
