"""Host-side arithmetic of bench.py that the JSON line reports, on CPU.

The algorithmic FLOPs and bytes are counted here a second way, expert by
expert from the routing's group sizes, and checked against the closed forms
bench.py uses; the figures quoted for the DeepSeek-V3-shaped prefill (its
kept-row count is fixed by the top-8 routing without a capacity) are checked
as numbers.  The DRAM traffic figure is only reported on the gate/up kernel
sources it was captured on.
"""
import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import moe_inputs as mi  # noqa: E402


def _per_expert(cfg, offsets):
    """FLOPs and gate/up bytes summed group by group (shapes written out)."""
    d, H, Hs, N = cfg.d_model, cfg.d_ff, cfg.d_ff_shared, cfg.n_tokens
    gate_up = down = 0.0
    gu_bytes = 0.0
    for g in range(cfg.n_experts):
        m = int(offsets[g + 1] - offsets[g])
        gate_up += 2 * m * d * H * 2       # [m x d] times [d x H], twice (gate, up)
        down += 2 * m * H * d              # [m x H] times [H x d]
        if m:
            gu_bytes += 2 * (H * d * 2)    # the expert's gate and up weights, bf16, once
        gu_bytes += m * d * 2 + m * H * 2  # its rows in, its activations out
    # the shared expert as one more group of all N tokens
    gate_up += 2 * N * d * Hs * 2
    down += 2 * N * Hs * d
    gu_bytes += 2 * (Hs * d * 2) + N * d * 2 + N * Hs * 2
    return gate_up, down, gu_bytes


def test_flops_and_bytes_match_a_per_expert_count():
    cfg = mi.CONFIGS["dsv3_prefill_bf16"].with_(n_tokens=512, n_experts=16)
    rng = np.random.default_rng(3)
    counts = rng.multinomial(cfg.n_tokens * cfg.top_k, np.ones(cfg.n_experts) / cfg.n_experts)
    counts[5] = 0  # an untouched expert moves no weights
    counts[6] += cfg.n_tokens * cfg.top_k - counts.sum()
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    fb = bench.workload_flops_bytes(cfg, offsets)
    gate_up, down, gu_bytes = _per_expert(cfg, offsets)
    assert fb["shared_folded"]
    assert fb["touched_experts"] == int((counts > 0).sum())
    assert fb["gate_up_flops"] == gate_up
    assert fb["down_flops"] == down
    assert fb["gate_up_bytes"] == gu_bytes
    assert fb["expert_flops"] == gate_up + down


def test_dsv3_prefill_figures_quoted_in_the_bench_line():
    cfg = mi.CONFIGS["dsv3_prefill_bf16"]
    fb = bench.workload_flops_bytes(cfg)  # no capacity: R = N * k kept rows
    assert fb["rows"] == 65536
    assert fb["gate_up_flops"] == 4329327034368.0  # 2 * (65536 + 8192) * 7168 * 4096
    assert fb["expert_flops"] == 6493990551552.0


def test_whole_job_throughput_counts_every_rank():
    assert bench.whole_job_tokens_per_s(8192, 1, 8.0) == 1024000.0
    assert bench.whole_job_tokens_per_s(8192, 4, 8.0) == 4096000.0


def test_set_overrides_keep_field_types():
    args = argparse.Namespace(workload="dsv3_prefill_bf16", set=["n_experts=32", "n_tokens=1024"])
    cfg = bench.workload(args)
    assert cfg.n_experts == 32 and isinstance(cfg.n_experts, int)
    assert cfg.n_tokens == 1024
    assert cfg.d_model == mi.CONFIGS["dsv3_prefill_bf16"].d_model


def test_traffic_figure_belongs_to_the_current_gemm_sources():
    # the ratio is reported only while the gate/up kernel's sources hash to the captured one
    assert bench.TRAFFIC["kernel_sha"] == bench._kernel_sha(), (
        "the gate/up kernel's sources changed since the DRAM traffic capture: take it again on the "
        "32-expert DeepSeek-V3-shaped case and update bench.TRAFFIC")
    assert 0.9 < bench.TRAFFIC["per_algorithmic_byte"] < 1.2
