"""The iterated auxiliary-loss-free balancing loop on the GPU.

"Mixture of Experts (MoE)" lesson, "Step 2: run 100 tokens through the
router": route, count each expert's load, move every bias by -gamma (over
target) or +gamma (under target), repeat; usage converges towards uniform.
Here one iteration is moe_route followed by moe_bias_update on the same
stream; fifty iterations are captured in one CUDA graph and replayed, and
the bias after every iteration must equal the oracle's bit for bit.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def _skewed_router(seed=5, n=1024, d=32, e=8, a=3.0, skew=0.6):
    # a constant input feature and a ramp on its router weights give the
    # experts increasing logits, so usage starts about 2x over the mean
    r = np.random.default_rng(seed)
    h = r.standard_normal((n, d)).astype(np.float32)
    h[:, 0] = a
    wr = (r.standard_normal((e, d)) / np.sqrt(d)).astype(np.float32)
    wr[:, 0] += skew * np.arange(e, dtype=np.float32) / e
    return h, wr


def test_balancing_loop_in_a_cuda_graph_matches_oracle():
    import torch
    import sparse_mixture_experts_rmsnorm_b200 as moe

    N, d, E, k, iters, gamma = 1024, 32, 8, 2, 50, 5e-3
    target = N * k / E
    h_np, wr_np = _skewed_router(n=N, d=d, e=E)
    cfg = moe.Config(N, d, E, k, 32, dtype="f32")
    dev = lambda a: torch.tensor(a, device="cuda")
    h, wr, norm_w = dev(h_np), dev(wr_np), torch.ones(d, device="cuda")
    ws = moe.workspace(cfg)
    xn = torch.empty(N, d, device="cuda")
    idx = torch.empty(N, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(N, k, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    bias = torch.zeros(E, device="cuda")
    bias_hist = torch.empty(iters, E, device="cuda")
    count_hist = torch.empty(iters, E, dtype=torch.int32, device="cuda")

    def iteration(i):
        moe.moe_route(cfg, h, norm_w, wr, bias, xn, None, idx, gate, counts, ws)
        moe.moe_bias_update(E, counts, target, gamma, bias)
        count_hist[i].copy_(counts)
        bias_hist[i].copy_(bias)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture
        iteration(0)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            iteration(i)
    bias.zero_()
    g.replay()
    torch.cuda.synchronize()

    xn_ref = oracle.rmsnorm(h_np, np.ones(d, np.float32), cfg.rms_eps, "f32")
    _, scores = oracle.router_scores(xn_ref, wr_np)
    ref_counts, ref_bias = oracle.balancing_loop(scores, np.zeros(E, np.float32), k, target, gamma, iters)
    got_counts = count_hist.cpu().numpy()
    got_bias = bias_hist.cpu().numpy()
    for i in range(iters):
        assert np.array_equal(got_counts[i], ref_counts[i]), (i, got_counts[i], ref_counts[i])
        assert np.array_equal(got_bias[i].view(np.uint32), ref_bias[i + 1].view(np.uint32)), i
    ratio = got_counts.max(axis=1) / got_counts.mean(axis=1)
    print(f"max/mean load: iteration 0 {ratio[0]:.3f}, iteration {iters - 1} {ratio[-1]:.3f}")
    assert ratio[0] > 1.8 and ratio[-10:].max() < 1.15


def test_balancing_loop_on_the_stress_skew():
    # The load-imbalance workload (Mixtral shapes, bf16, about 90 % of top-1
    # choices on expert 3), fifty route + bias-update iterations with
    # gamma = 1e-3 in one CUDA graph.  Biases must equal the oracle's bit for
    # bit after every iteration; counts too, except for tokens whose oracle
    # keys at that iteration's bias are within KEY_TIE (the router's fp32 sums
    # may order those either way, and a count only moves the bias when it
    # crosses the target).
    import torch
    import moe_inputs as mi
    import sparse_mixture_experts_rmsnorm_b200 as moe
    from parity_helpers import lib_config, oracle_routing, tie_masks

    cfg = mi.CONFIGS["stress_bf16"]
    N, d, E, k, iters, gamma = cfg.n_tokens, cfg.d_model, cfg.n_experts, cfg.top_k, 50, cfg.gamma
    target = float(np.float32(N * k / E))
    lc = lib_config(cfg)
    dev = mi.device_tensors(cfg, names=["h", "norm_w", "w_router"])
    ws = moe.workspace(lc)
    xn = torch.empty_like(dev["h"])
    idx = torch.empty(N, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(N, k, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    bias = torch.zeros(E, device="cuda")
    bias_hist = torch.empty(iters, E, device="cuda")
    count_hist = torch.empty(iters, E, dtype=torch.int32, device="cuda")

    def iteration(i):
        moe.moe_route(lc, dev["h"], dev["norm_w"], dev["w_router"], bias, xn, None, idx, gate, counts, ws)
        moe.moe_bias_update(E, counts, target, gamma, bias)
        count_hist[i].copy_(counts)
        bias_hist[i].copy_(bias)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture
        iteration(0)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            iteration(i)
    bias.zero_()
    g.replay()
    torch.cuda.synchronize()
    st, info = moe.moe_check_device_error(ws)
    assert st == 0, info

    ref = oracle_routing(cfg)
    ref_counts, ref_bias = oracle.balancing_loop(ref["scores"], np.zeros(E, np.float32), k, target, gamma, iters)
    got_counts = count_hist.cpu().numpy().astype(np.int64)
    got_bias = bias_hist.cpu().numpy()
    for i in range(iters):
        key = ref["scores"].astype(np.float32) + ref_bias[i][None, :]
        near = int(tie_masks(key, k)[0].sum())
        diff = int(np.abs(got_counts[i] - ref_counts[i]).sum())
        assert diff <= 2 * near, (i, got_counts[i], ref_counts[i], near)
        assert np.array_equal(got_bias[i].view(np.uint32), ref_bias[i + 1].view(np.uint32)), i
    ratio = got_counts.max(axis=1) / got_counts.mean(axis=1)
    traj = ", ".join(f"{i}: {ratio[i]:.3f}" for i in (0, 10, 20, 30, 40, iters - 1))
    print(f"BALANCE stress skew, gamma {gamma}: max/mean load by iteration {traj}; "
          f"expert-3 count {got_counts[0][3]} -> {got_counts[-1][3]}; bias[3] {got_bias[-1][3]:.4f}")
    assert np.all(got_counts.sum(axis=1) == N * k)
    # the over-used expert's load falls and its bias only ever moves down
    assert got_counts[-1][3] < got_counts[0][3] and ratio[-1] < ratio[0]
    assert np.all(np.diff(got_bias[:, 3]) <= 0)
