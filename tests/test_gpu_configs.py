"""GPU parity of the four bf16 layer workloads at their full sizes, and of
the DeepSeek-V3-shaped prefill at four and eight times its tokens (N = 32768:
full 256-row chunks, 1024 permutation chunks; N = 65536: the expert-sorted
rows hold 3.76e9 elements, past 32-bit element offsets, the largest layer the
tests run, about 45 GB on the device).

Routing, counts, permutation and drop masks are checked on every token;
outputs on a stratified sample the oracle computes token by token (each
expert's weights regenerated on the host once): the first and last kept row
of every expert, so every expert's GEMM tiles and ragged tails are reached,
the ends of the shared expert's group, the last rows in tile order, and some
random tokens; bias updates bit-exactly.
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from parity_helpers import (BF16_REL_RMS, KEY_TIE, bf16_half_ulp, bf16_rel_rms_err, capacity, check_permutation,
                            check_routing, oracle_outputs, oracle_routing, rel_rms_err, run_gpu_layer, tie_masks,
                            to_np)

pytestmark = pytest.mark.gpu

# random tokens sampled on top of the stratified ones
SAMPLES = {"mixtral_bf16": 24, "dsv3_prefill_bf16": 32, "dsv3_decode_bf16": 64, "stress_bf16": 16,
           "dsv3_prefill_bf16@32768": 16, "dsv3_prefill_bf16@65536": 16}


def stratified_tokens(offsets, row_token, eligible, n_tokens, rng, n_random, late=8):
    """Tokens whose outputs are compared: for every expert the tokens of its
    first and last kept rows (its ragged last tile included), the first and
    last token (the ends of the shared expert's group, which runs last), the
    tokens of the last `late` routed rows (late in the GEMM tile order), and
    `n_random` more.  Only tokens marked eligible are taken; an expert whose
    rows are all ineligible is skipped.  Returns the sorted tokens."""
    picks = []
    for e in range(len(offsets) - 1):
        rows = row_token[offsets[e]:offsets[e + 1]]
        rows = rows[eligible[rows]]
        if rows.size:
            picks += [rows[0], rows[-1]]
    ends = [t for t in (0, n_tokens - 1) if n_tokens and eligible[t]]
    tail = row_token[max(0, int(offsets[-1]) - late):int(offsets[-1])]
    pool = np.nonzero(eligible)[0]
    rand = rng.choice(pool, size=min(n_random, pool.size), replace=False) if pool.size else []
    return np.unique(np.concatenate([np.asarray(picks, dtype=np.int64), np.asarray(ends, dtype=np.int64),
                                     tail[eligible[tail]].astype(np.int64), np.asarray(rand, dtype=np.int64)]))


@pytest.mark.parametrize("name", list(SAMPLES))
def test_config_parity(name):
    import torch
    import sparse_mixture_experts_rmsnorm_b200 as moe

    base, _, n_tokens = name.partition("@")
    cfg = mi.CONFIGS[base]
    if n_tokens:
        cfg = cfg.with_(n_tokens=int(n_tokens))
    N, E, k = cfg.n_tokens, cfg.n_experts, cfg.top_k
    g = run_gpu_layer(cfg)
    ref = oracle_routing(cfg)
    np.testing.assert_array_equal(g["xn"], ref["xn"])
    # every fp32 selection key within the tie window of the oracle's
    bias32 = mi.host_tensor(cfg, "bias").astype(np.float32)
    key_err = float(np.max(np.abs((g["scores"].astype(np.float32) + bias32[None, :]).astype(np.float64)
                                  - ref["key"])))
    assert key_err <= KEY_TIE, key_err
    skipped = check_routing(g, ref, k)
    assert skipped <= max(2, 0.01 * N), skipped
    cap = capacity(cfg)
    check_permutation(g, E, cap)

    # drop decisions against the oracle's own routing: equal up to the first
    # token whose routing was ambiguous (a near tie) when a capacity applies
    ref_off, ref_slot, ref_rt = oracle.permute(ref["idx"], E, cap)
    ref_keep = (ref_slot >= 0).reshape(N, k)
    gpu_keep = (g["slot_row"] >= 0).reshape(N, k)
    _, order_amb = tie_masks(ref["key"], k)
    upto = N if cap < 0 or not order_amb.any() else int(np.argmax(order_amb))
    assert np.array_equal(gpu_keep[:upto], ref_keep[:upto])

    # sampled outputs: a row of every expert, chosen from the oracle's own
    # permutation among the tokens whose routing is unambiguous
    rng = np.random.default_rng(0)
    eligible = ~order_amb
    eligible[upto:] = False
    tokens = stratified_tokens(ref_off, ref_rt, eligible, N, rng, SAMPLES[name])
    dropped_any = np.nonzero(~ref_keep[:upto].all(axis=1) & eligible[:upto])[0]
    if dropped_any.size:
        tokens = np.unique(np.concatenate([tokens, rng.choice(dropped_any, size=min(8, dropped_any.size),
                                                              replace=False)]))
    covered = np.unique(ref["idx"][tokens][ref_keep[tokens]])
    reachable = np.unique(ref["idx"][eligible][ref_keep[eligible]])
    assert np.array_equal(covered, reachable), (covered.size, reachable.size)
    ref_out = oracle_outputs(cfg, ref, tokens, ref["idx"], ref["gates"], ref_keep)
    got = g["out"][tokens]
    # the tolerance bounds the arithmetic; storing out in bf16 adds up to half
    # a bf16 spacing on top of it even for an exact result
    err = bf16_rel_rms_err(got, ref_out)
    raw = rel_rms_err(got, ref_out)
    raw_delta = rel_rms_err(got - ref["h"][tokens], ref_out - ref["h"][tokens])
    # the same beyond-storage error, relative to the layer's contribution out - h
    delta_rms = float(np.sqrt(np.mean((ref_out - ref["h"][tokens]) ** 2)))
    bs_delta = float(np.max(np.maximum(np.abs(got - ref_out) - bf16_half_ulp(ref_out), 0.0)) / delta_rms)
    print(f"PARITY {name}: beyond-storage max err/rms(out) = {err:.3e}; raw max|err|/rms(out) = {raw:.3e}; "
          f"raw max|err| on out-h / rms(out-h) = {raw_delta:.3e}; beyond-storage max err / rms(out-h) = "
          f"{bs_delta:.3e}; rms(out) = {np.sqrt(np.mean(ref_out ** 2)):.3f}, rms(out-h) = {delta_rms:.4f}; "
          f"tokens {tokens.size}, experts covered "
          f"{covered.size} of {E}{' + shared' if cfg.d_ff_shared else ''}, skipped ties {skipped}, "
          f"dropped slots {int((~gpu_keep).sum())}, max key err {key_err:.2e}")
    assert err <= BF16_REL_RMS, err

    if cap >= 0:
        # a token whose every slot was dropped passes through unchanged (no shared expert here)
        all_dropped = np.nonzero(~gpu_keep.any(axis=1))[0]
        if cfg.d_ff_shared == 0 and all_dropped.size:
            np.testing.assert_array_equal(g["out"][all_dropped], ref["h"][all_dropped])
        kept = np.diff(g["offsets"])
        assert np.all(kept <= cap)

    if base == "stress_bf16":
        top1_share = float(np.mean(g["topk_idx"][:, 0] == 3))
        assert abs(top1_share - 0.90) <= 0.011, top1_share
        target = np.float32(N * k / E)
        bias = g["dev"]["bias"].clone()
        moe.moe_bias_update(E, torch.tensor(g["counts"], dtype=torch.int32, device="cuda"), float(target),
                            cfg.gamma, bias)
        ref_counts = oracle.expert_counts(ref["idx"], E)
        assert np.array_equal(g["counts"].astype(np.int64), ref_counts)
        exp = oracle.bias_update(mi.host_tensor(cfg, "bias"), ref_counts, target, cfg.gamma)
        assert np.array_equal(to_np(bias).astype(np.float32).view(np.uint32), exp.view(np.uint32))
