"""Pins of the CPU oracle to what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a value
the pages print, a closed form, an invariant, a textbook or library routine,
or brute force on tiny inputs.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _bf16_torch(x64):
    return torch.tensor(x64, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------- rounding

def test_round_to_bf16_matches_torch_from_fp32():
    # from fp32 values torch rounds once, as the oracle does
    x = (rng.standard_normal(100000) * 5).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_to(x, "bf16"), _bf16_torch(x))


def test_round_to_bf16_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even 1.0;
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: goes to 1+2^-6.
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -30])
    np.testing.assert_array_equal(oracle.round_to(x, "bf16"),
                                  [1.0, 1 + 2.0 ** -6, -1.0, 1 + 2.0 ** -7])


# ---------------------------------------------------------------- a1 RMSNorm

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rmsnorm_matches_torch_rms_norm(dtype):
    h = rng.standard_normal((64, 96)) * 3
    h = oracle.round_to(h, dtype)
    w = oracle.round_to(1 + 0.1 * rng.standard_normal(96), dtype)
    xn = oracle.rmsnorm(h, w, 1e-6, dtype)
    ref = torch.nn.functional.rms_norm(torch.tensor(h), (96,), torch.tensor(w), eps=float(np.float32(1e-6))).numpy()
    # one storage rounding plus three fp32 roundings
    ulp = 2.0 ** -7 if dtype == "bf16" else 2.0 ** -23  # spacing at the bottom of a binade
    assert np.all(np.abs(xn - ref) <= (0.5 * ulp + 4 * 2.0 ** -24) * np.abs(ref) + 1e-30)


def test_rmsnorm_unit_mean_square():
    h = oracle.round_to(rng.standard_normal((32, 4096)) * 7, "bf16")
    xn = oracle.rmsnorm(h, np.ones(4096), 1e-6, "bf16")
    ms = np.mean(xn ** 2, axis=1)
    assert np.all(np.abs(ms - 1) < 3e-3)


def test_rmsnorm_scale_invariance():
    h = oracle.round_to(rng.standard_normal((8, 128)), "f32")
    a = oracle.rmsnorm(h, np.ones(128), 0.0, "f32")
    b = oracle.rmsnorm(h * 4.0, np.ones(128), 0.0, "f32")  # power of two: exact
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- a2 router

def test_router_scores_softmax_properties():
    xn = rng.standard_normal((16, 32))
    wr = rng.standard_normal((8, 32)) * 0.3
    logits, scores = oracle.router_scores(xn, wr)
    np.testing.assert_allclose(logits, np.einsum("td,ed->te", xn, wr), rtol=1e-12)
    np.testing.assert_allclose(scores.sum(1), 1, atol=1e-14)
    ref = torch.softmax(torch.tensor(logits), dim=1).numpy()
    np.testing.assert_allclose(scores, ref, rtol=1e-13)


# ---------------------------------------------------------------- a3 top-k

def _brute_topk(key_row, k):
    """Subset with the largest sum of keys; among equal sums the
    lexicographically smallest index tuple (lower index wins ties)."""
    best, best_sum = None, None
    for sub in itertools.combinations(range(len(key_row)), k):
        s = float(np.sum(key_row[list(sub)], dtype=np.float64))
        if best is None or s > best_sum:
            best, best_sum = sub, s
    return set(best)


@pytest.mark.parametrize("E,k", [(4, 1), (5, 2), (8, 2), (8, 3), (6, 6)])
def test_topk_matches_brute_force(E, k):
    for _ in range(50):
        scores = rng.random((1, E))
        scores /= scores.sum()
        bias = (rng.random(E) - 0.5) * 0.2
        idx, key = oracle.select_topk(scores, bias, k)
        assert set(idx[0].tolist()) == _brute_topk(key[0].astype(np.float64), k)
        # ordered by descending key
        assert np.all(np.diff(key[0][idx[0]]) <= 0)


def test_topk_ties_lower_index_wins():
    scores = np.array([[0.1, 0.3, 0.3, 0.3]])
    idx, _ = oracle.select_topk(scores, np.zeros(4), 2)
    assert idx.tolist() == [[1, 2]]
    idx, _ = oracle.select_topk(np.full((1, 8), 0.125), np.zeros(8), 3)
    assert idx.tolist() == [[0, 1, 2]]
    for _ in range(20):
        vals = rng.integers(0, 3, size=6).astype(np.float64) / 8
        idx, key = oracle.select_topk(vals[None, :], np.zeros(6), 3)
        assert set(idx[0].tolist()) == _brute_topk(key[0].astype(np.float64), 3)


def test_selection_uses_bias_but_gates_do_not():
    # [LESSON] "The load-balancing problem": selection on scores + bias,
    # gating probabilities from the unmodified scores.
    scores = np.array([[0.40, 0.30, 0.20, 0.10]])
    idx0, _ = oracle.select_topk(scores, np.zeros(4), 2)
    idx1, _ = oracle.select_topk(scores, np.array([0.0, -0.5, 0.0, 0.0]), 2)
    assert sorted(idx0[0]) == [0, 1] and sorted(idx1[0]) == [0, 2]
    g1 = oracle.gates_from_scores(scores, idx1)
    assert np.allclose(g1[0], [0.4 / 0.6, 0.2 / 0.6], rtol=1e-15)
    # a bias that keeps the same chosen set leaves the gates bit-identical
    idx2, _ = oracle.select_topk(scores, np.array([0.05, 0.01, -0.02, 0.0]), 2)
    assert idx2[0].tolist() == idx0[0].tolist()
    np.testing.assert_array_equal(oracle.gates_from_scores(scores, idx2),
                                  oracle.gates_from_scores(scores, idx0))


def test_large_bias_forces_expert_into_every_topk():
    xn = rng.standard_normal((200, 16))
    _, scores = oracle.router_scores(xn, rng.standard_normal((8, 16)))
    bias = np.zeros(8)
    bias[5] = 2.0
    idx, _ = oracle.select_topk(scores, bias, 2)
    assert np.all(idx[:, 0] == 5)


def test_gates_equal_lesson_softmax_over_chosen_logits():
    # [LESSON] "Step 1: the router" forms gates as a max-shifted softmax over
    # the chosen raw scores; renormalised softmax probabilities are the same.
    xn = rng.standard_normal((50, 24))
    logits, scores = oracle.router_scores(xn, rng.standard_normal((8, 24)) * 0.5)
    idx, _ = oracle.select_topk(scores, np.zeros(8), 3)
    g = oracle.gates_from_scores(scores, idx)
    for t in range(50):
        chosen = logits[t, idx[t]]
        ex = [np.exp(c - max(chosen)) for c in chosen]
        np.testing.assert_allclose(g[t], np.array(ex) / sum(ex), rtol=1e-13)
    assert np.all(g >= 0)
    np.testing.assert_allclose(g.sum(1), 1, atol=1e-15)


# ---------------------------------------------------------------- a4 counts/permute

def test_glossary_printed_routing_example():
    fx = json.load(open(os.path.join(GOLDEN, "glossary_top2_example.json")))
    idx = np.array(fx["experts_per_token"])
    counts = oracle.expert_counts(idx, fx["n_experts"])
    assert counts.tolist() == fx["tokens_per_expert"]
    assert counts.sum() == fx["n_tokens"] * fx["top_k"]
    offsets, slot_row, row_token = oracle.permute(idx, 8)
    assert offsets.tolist() == [0, 1, 3, 4, 7, 7, 7, 10, 12]
    # per-expert token lists in token order
    lists = {e: row_token[offsets[e]:offsets[e + 1]].tolist() for e in range(8)}
    assert lists == {0: [2], 1: [3, 4], 2: [5], 3: [0, 3, 5], 4: [], 5: [], 6: [0, 1, 4], 7: [1, 2]}
    assert sorted(slot_row.tolist()) == list(range(12))


def test_glossary_example_with_capacity_two():
    fx = json.load(open(os.path.join(GOLDEN, "glossary_top2_example.json")))
    idx = np.array(fx["experts_per_token"])
    offsets, slot_row, row_token = oracle.permute(idx, 8, capacity=2)
    # experts 3 and 6 keep their first two tokens (0, 3) and (0, 1)
    assert offsets.tolist() == [0, 1, 3, 4, 6, 6, 6, 8, 10]
    lists = {e: row_token[offsets[e]:offsets[e + 1]].tolist() for e in range(8)}
    assert lists[3] == [0, 3] and lists[6] == [0, 1]
    dropped = [s for s in range(12) if slot_row[s] < 0]
    assert dropped == [4 * 2 + 0, 5 * 2 + 1]  # token 4 -> expert 6, token 5 -> expert 3


def test_load_stats_of_the_glossary_example():
    # The printed example: 12 slots over 8 experts (mean load 1.5), the
    # busiest experts (3 and 6) take three tokens each, so max/mean = 2; a
    # capacity of 2 drops one slot at each of them and at no other expert.
    fx = json.load(open(os.path.join(GOLDEN, "glossary_top2_example.json")))
    idx = np.array(fx["experts_per_token"])
    n, E, k = fx["n_tokens"], fx["n_experts"], fx["top_k"]
    counts = np.array(fx["tokens_per_expert"])
    free, _, _ = oracle.permute(idx, E)
    st = oracle.load_stats(counts, free, n, k, E)
    assert (st["routed"], st["kept"], st["dropped"], st["max_count"]) == (12, 12, 0, 3)
    assert st["max_over_mean"] == np.float32(2.0)
    capped, _, _ = oracle.permute(idx, E, capacity=2)
    st = oracle.load_stats(counts, capped, n, k, E)
    # the maximum is taken before the cut, as the bias update's usage is
    assert (st["routed"], st["kept"], st["dropped"], st["max_count"]) == (12, 10, 2, 3)
    assert st["max_over_mean"] == np.float32(2.0)


def test_load_stats_closed_forms():
    # perfect balance gives max/mean = 1 exactly; every slot on one expert gives E
    E, k, n = 16, 4, 64
    even = np.full(E, n * k // E)
    st = oracle.load_stats(even, np.concatenate([[0], np.cumsum(even)]), n, k, E)
    assert st["max_over_mean"] == np.float32(1.0) and st["dropped"] == 0
    one = np.zeros(E, dtype=np.int64)
    one[7] = n * k
    st = oracle.load_stats(one, np.concatenate([[0], np.cumsum(one)]), n, k, E)
    assert st["max_over_mean"] == np.float32(E) and st["max_count"] == n * k
    st = oracle.load_stats(np.zeros(E), np.zeros(E + 1), 0, k, E)
    assert (st["routed"], st["kept"], st["dropped"], st["max_count"], st["max_over_mean"]) == (0, 0, 0, 0, 0.0)


def test_permute_brute_force_small():
    for _ in range(30):
        n, E, k = 13, 5, 2
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(n)])
        cap = int(rng.integers(1, 6))
        offsets, slot_row, row_token = oracle.permute(idx, E, cap)
        for e in range(E):
            toks = [t for t in range(n) for j in range(k) if idx[t, j] == e][:cap]
            assert row_token[offsets[e]:offsets[e + 1]].tolist() == toks
        for t in range(n):
            for j in range(k):
                r = slot_row[t * k + j]
                if r >= 0:
                    assert row_token[r] == t and offsets[idx[t, j]] <= r < offsets[idx[t, j] + 1]


def test_capacity_formula():
    assert oracle.capacity_limit(1.25, 4096, 2, 8) == 1280
    assert oracle.capacity_limit(0.0, 4096, 2, 8) == -1
    assert oracle.capacity_limit(1.0, 10, 1, 3) == 3


# ---------------------------------------------------------------- experts and layer

def _tiny_layer(E=4, k=2, d=16, H=24, n=40, dtype="f32", cf=0.0, shared=False, seed=0):
    r = np.random.default_rng(seed)
    rd = lambda *s, sc=1.0: oracle.round_to(r.standard_normal(s) * sc, dtype)
    args = dict(h=rd(n, d), norm_w=oracle.round_to(1 + 0.1 * r.standard_normal(d), dtype),
                w_router=rd(E, d, sc=0.3), bias=np.zeros(E),
                w_gate=rd(E, H, d, sc=0.25), w_up=rd(E, H, d, sc=0.25), w_down=rd(E, d, H, sc=0.2))
    if shared:
        args.update(ws_gate=rd(H, d, sc=0.25), ws_up=rd(H, d, sc=0.25), ws_down=rd(d, H, sc=0.2))
    return args


def _torch_swiglu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.tensor(a, dtype=torch.float64) for a in (x, wg, wu, wd))
    return (torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def test_single_expert_top1_is_textbook_swiglu_ffn():
    a = _tiny_layer(E=1, k=1, dtype="f32")
    res = oracle.layer_forward(**a, top_k=1, eps=1e-6, dtype="f32")
    xn = torch.nn.functional.rms_norm(torch.tensor(a["h"]), (16,), torch.tensor(a["norm_w"]),
                                      eps=float(np.float32(1e-6)))
    ref = torch.tensor(a["h"]) + _torch_swiglu(xn.numpy(), a["w_gate"][0], a["w_up"][0], a["w_down"][0])
    np.testing.assert_allclose(res["out64"], ref.numpy(), rtol=1e-5, atol=1e-5)
    np.testing.assert_array_equal(res["gates"], 1.0)


def test_k_equals_E_is_dense_softmax_weighted_sum():
    # spec identity: with k = E and zero bias the layer is the dense,
    # softmax-weighted sum of every expert (computed here as a plain loop).
    E = 5
    a = _tiny_layer(E=E, k=E, dtype="f32", shared=True)
    res = oracle.layer_forward(**a, top_k=E, eps=1e-6, dtype="f32")
    xn = torch.nn.functional.rms_norm(torch.tensor(a["h"]), (16,), torch.tensor(a["norm_w"]),
                                      eps=float(np.float32(1e-6))).numpy()
    p = torch.softmax(torch.tensor(xn) @ torch.tensor(a["w_router"]).T, dim=1).numpy()
    ref = a["h"].copy()
    for e in range(E):
        ref = ref + p[:, e:e + 1] * _torch_swiglu(xn, a["w_gate"][e], a["w_up"][e], a["w_down"][e]).numpy()
    ref = ref + _torch_swiglu(xn, a["ws_gate"], a["ws_up"], a["ws_down"]).numpy()
    np.testing.assert_allclose(res["out64"], ref, rtol=1e-5, atol=1e-5)
    assert np.all(res["counts"] == 40)


def test_layer_invariants_and_shared_expert_additivity():
    a = _tiny_layer(E=6, k=2, dtype="bf16", shared=True)
    res = oracle.layer_forward(**a, top_k=2, eps=1e-6, dtype="bf16")
    assert res["counts"].sum() == 40 * 2
    np.testing.assert_allclose(res["gates"].sum(1), 1, atol=1e-15)
    b = {k: v for k, v in a.items() if not k.startswith("ws_")}
    res2 = oracle.layer_forward(**b, top_k=2, eps=1e-6, dtype="bf16")
    np.testing.assert_allclose(res["out64"] - res2["out64"], res["y_shared"], atol=1e-12)
    # routed part as an explicit per-token sum, slot by slot
    for t in range(0, 40, 7):
        acc = a["h"][t].astype(np.float64).copy()
        for j in range(2):
            e = res["idx"][t, j]
            acc += res["gates"][t, j] * _torch_swiglu(res["xn"][t:t + 1], a["w_gate"][e], a["w_up"][e],
                                                       a["w_down"][e]).numpy()[0]
        np.testing.assert_allclose(res2["out64"][t], acc, rtol=2e-2, atol=2e-2)


def test_dropped_tokens_pass_through_on_residual():
    # [GLOSSARY] "Load balancing and expert capacity": tokens over the limit
    # skip the layer's experts and continue on the residual.
    a = _tiny_layer(E=4, k=1, n=64, dtype="bf16")
    a["w_router"][1] += 3.0  # skew routing towards expert 1
    res = oracle.layer_forward(**a, top_k=1, eps=1e-6, dtype="bf16", capacity_factor=0.5)
    cap = res["capacity"]
    assert cap == 8
    kept = np.diff(res["offsets"])
    assert np.all(kept <= cap) and np.all(kept == np.minimum(res["counts"], cap))
    dropped = res["slot_row"] < 0
    assert dropped.sum() == res["counts"].sum() - kept.sum() > 0
    np.testing.assert_array_equal(res["out"][dropped], a["h"][dropped])
    np.testing.assert_array_equal(res["out64"][dropped], a["h"][dropped])


def test_partially_dropped_token_keeps_its_unrenormalised_gate():
    # [GLOSSARY] "Load balancing and expert capacity": a slot over the limit
    # skips its expert and the token continues on the residual for that slot.
    # Reading: the kept slot adds gate_kept * y_kept with the gate computed
    # over all k chosen experts (no renormalisation over the kept ones).
    # Hand-built case, E = 3, k = 2, N = 2, C = 0.75: cap = floor(0.75*2*2/3) = 1.
    # Token 0 chooses experts {0, 1}, token 1 chooses {0, 2}; expert 0's one
    # place goes to token 0, so token 1 keeps only its slot on expert 2.
    d, H = 8, 12
    r = np.random.default_rng(5)
    h = 0.01 * r.standard_normal((2, d))
    h[0, 0] += 1.0
    h[1, 1] += 1.0
    w_router = np.zeros((3, d))
    w_router[0, :2] = [2.0, 2.0]
    w_router[1, :2] = [1.0, -1.0]
    w_router[2, :2] = [-1.0, 1.0]
    wg, wu, wd = r.standard_normal((3, H, d)) * 0.4, r.standard_normal((3, H, d)) * 0.4, r.standard_normal((3, d, H))
    res = oracle.layer_forward(h, np.ones(d), w_router, np.zeros(3), wg, wu, wd, top_k=2, eps=1e-6, dtype="f32",
                               capacity_factor=0.75)
    assert res["capacity"] == 1
    assert res["idx"].tolist() == [[0, 1], [0, 2]]
    assert res["slot_row"].tolist() == [0, 1, -1, 2]  # token 1's slot on expert 0 is dropped
    # the expected token-1 output, written out with torch from the definitions
    xn = torch.nn.functional.rms_norm(torch.tensor(h), (d,), eps=float(np.float32(1e-6)))
    p = torch.softmax(xn @ torch.tensor(w_router).T, dim=1)
    g_kept = float(p[1, 2] / (p[1, 0] + p[1, 2]))  # gate of expert 2 over the two chosen experts
    y2 = _torch_swiglu(xn[1:2].numpy(), wg[2], wu[2], wd[2]).numpy()[0]
    expect = h[1] + g_kept * y2
    np.testing.assert_allclose(res["out64"][1], expect, rtol=1e-5, atol=1e-6)
    # the plausible wrong readings are far from it: renormalised over the kept
    # slot (gate 1), or the kept gate scaled by 1/k
    assert 0.01 < g_kept < 0.4 and np.linalg.norm(y2) > 0.5
    for wrong in (h[1] + y2, h[1] + 0.5 * y2):
        assert np.max(np.abs(res["out64"][1] - wrong)) > 0.05
    # token 0 keeps both slots: the plain gated sum
    g0 = (p[0, [0, 1]] / p[0, [0, 1]].sum()).numpy()
    y0 = [_torch_swiglu(xn[0:1].numpy(), wg[e], wu[e], wd[e]).numpy()[0] for e in (0, 1)]
    np.testing.assert_allclose(res["out64"][0], h[0] + g0[0] * y0[0] + g0[1] * y0[1], rtol=1e-5, atol=1e-6)


# ---------------------------------------------------------------- a10 bias update

def test_bias_update_exact_fp32_sign_rule():
    bias = np.array([0.0, 1e-3, -2e-3, 0.5, 3.0e-8, -0.0], dtype=np.float32)
    counts = np.array([10, 30, 20, 20, 19, 21])
    out = oracle.bias_update(bias, counts, 20.0, 1e-3)
    g = np.float32(1e-3)
    exp = np.array([bias[0] + g, bias[1] - g, bias[2], bias[3], bias[4] + g, bias[5] - g], dtype=np.float32)
    np.testing.assert_array_equal(out, exp)
    assert out.dtype == np.float32


def test_stress_recipe_skews_top1_to_expert3_and_bias_signs():
    cfg = mi.CONFIGS["stress_bf16"]
    h = mi.host_tensor(cfg, "h")
    xn = oracle.rmsnorm(h, mi.host_tensor(cfg, "norm_w"), cfg.rms_eps, cfg.dtype)
    _, scores = oracle.router_scores(xn, mi.host_tensor(cfg, "w_router"))
    idx, _ = oracle.select_topk(scores, mi.host_tensor(cfg, "bias"), cfg.top_k)
    share = np.mean(idx[:, 0] == 3)
    assert abs(share - 0.90) <= 0.01, share
    counts = oracle.expert_counts(idx, cfg.n_experts)
    target = np.float32(cfg.n_tokens * cfg.top_k / cfg.n_experts)
    nb = oracle.bias_update(np.zeros(8, np.float32), counts, target, cfg.gamma)
    g = np.float32(cfg.gamma)
    assert nb[3] == -g and all(nb[e] == g for e in range(8) if e != 3)
    assert oracle.capacity_limit(cfg.capacity_factor, cfg.n_tokens, cfg.top_k, cfg.n_experts) == 1280


# ---------------------------------------------------------------- iterated balancing (lesson, Step 2)

def test_balancing_loop_two_experts_hand_derived_trajectory():
    # Every token scores (0.625, 0.375); gamma = 2^-7, so all sums are exact.
    # Expert 0 takes all tokens while 0.625 - n*g > 0.375 + n*g, i.e. for
    # n = 0..15; at n = 16 the keys tie (0.5, 0.5) and the lower index keeps
    # them, so the bias moves once more; at n = 17 expert 1 wins, the biases
    # step back to n = 16 and the pair oscillates: counts alternate from then on.
    n_tok, g = 10, 2.0 ** -7
    scores = np.tile([0.625, 0.375], (n_tok, 1))
    counts, biases = oracle.balancing_loop(scores, [0.0, 0.0], 1, n_tok / 2, g, 22)
    assert counts[:17, 0].tolist() == [n_tok] * 17
    assert counts[17:, 0].tolist() == [0, n_tok, 0, n_tok, 0]
    assert biases[17].tolist() == [-17 * g, 17 * g]
    assert biases[18].tolist() == [-16 * g, 16 * g]
    assert biases[22].tolist() == [-16 * g, 16 * g]
    assert counts.sum(axis=1).tolist() == [n_tok] * 22


def test_balancing_loop_reduces_imbalance():
    # [LESSON] "Step 2": with the bias loop, skewed usage moves to a near
    # uniform one within some tens of iterations.  Router logits with
    # per-expert offsets 0 .. 2 start about 2.3x over the mean load.
    r = np.random.default_rng(3)
    xn = r.standard_normal((1024, 32))
    logits = xn @ (r.standard_normal((8, 32)) / np.sqrt(32)).T + np.linspace(0, 2, 8)
    ex = np.exp(logits - logits.max(1, keepdims=True))
    scores = ex / ex.sum(1, keepdims=True)
    counts, biases = oracle.balancing_loop(scores, np.zeros(8), 2, 1024 * 2 / 8, 5e-3, 50)
    ratio = counts.max(axis=1) / counts.mean(axis=1)
    assert ratio[0] > 2.0 and ratio[-10:].max() < 1.2 and ratio[-1] < 1.1
    assert np.all(counts.sum(axis=1) == 2048)
    # the most loaded expert at the start ends with the lowest bias
    assert np.argmin(biases[-1]) == np.argmax(counts[0])


# ---------------------------------------------------------------- hash router (lesson exercise)

def test_splitmix64_published_first_output():
    # the first SplitMix64 output from state 0 (Vigna's splitmix64.c)
    assert oracle.splitmix64(0) == 0xE220A8397B1DCDAF


def test_hash_route_properties():
    E, k = 16, 3
    ids = np.arange(20000)
    idx, gates = oracle.hash_route(ids, E, k)
    assert idx[0, 0] == 0xE220A8397B1DCDAF % E
    # k distinct, consecutive (mod E) experts; gates 1/k in fp32
    assert np.all((idx[:, 1] - idx[:, 0]) % E == 1) and np.all((idx[:, 2] - idx[:, 0]) % E == 2)
    np.testing.assert_array_equal(gates, np.float32(1 / 3))
    # the first choice is close to uniform over the experts (chi-square, 15 dof, p ~ 1e-4 bound)
    c = np.bincount(idx[:, 0], minlength=E)
    chi2 = ((c - len(ids) / E) ** 2 / (len(ids) / E)).sum()
    assert chi2 < 45
    # the same id always routes the same way
    again, _ = oracle.hash_route(ids[::-1], E, k)
    np.testing.assert_array_equal(again[::-1], idx)
