"""Derive the constant c of the load-imbalance stress recipe.

The recipe adds a = 8 to feature 0 of every token and c / a to router weight
[3, 0], which raises expert 3's router logit by about c for every token.
Bisection on c, with the oracle router at seed 0, finds the c that sends
90% of top-1 choices to expert 3.  Uses only the input generator and the
oracle.  Run:  python tests/golden/derive_stress_c.py
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402


def top1_share(c: float) -> float:
    cfg = mi.CONFIGS["stress_bf16"].with_(skew=(3, 8.0, c))
    xn = oracle.rmsnorm(mi.host_tensor(cfg, "h"), mi.host_tensor(cfg, "norm_w"), cfg.rms_eps, cfg.dtype)
    _, scores = oracle.router_scores(xn, mi.host_tensor(cfg, "w_router"))
    idx, _ = oracle.select_topk(scores, mi.host_tensor(cfg, "bias"), cfg.top_k)
    return float(np.mean(idx[:, 0] == 3))


def main():
    lo, hi = 0.0, 8.0
    for _ in range(14):
        mid = 0.5 * (lo + hi)
        if top1_share(mid) < 0.90:
            lo = mid
        else:
            hi = mid
    c = round(hi, 2)
    print(f"c = {c}  top-1 share on expert 3 = {top1_share(c):.4f}")


if __name__ == "__main__":
    main()
