"""The five synthetic layer workloads and the tensor recipe for each.

Shapes follow the MoE models the pages describe: a tiny fp32 layer, a
Mixtral-8x7B-shaped layer (8 experts, top-2, d_model 4096, SwiGLU hidden
14336), a DeepSeek-V3-shaped layer (256 routed experts, top-8, d_model 7168,
hidden 2048, one always-on shared expert) at prefill (8192 tokens) and
decode (64 tokens) sizes, and a load-imbalance stress case on Mixtral shapes
with an expert capacity and one bias update.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

# Tensor ids of the counter hash (one id per layer input).
TID_H, TID_W_ROUTER, TID_BIAS = 1, 2, 3
TID_W_GATE, TID_W_UP, TID_W_DOWN = 4, 5, 6
TID_WS_GATE, TID_WS_UP, TID_WS_DOWN = 7, 8, 9
TID_NORM_W = 10


@dataclass(frozen=True)
class LayerConfig:
    name: str
    n_tokens: int
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    d_ff_shared: int = 0
    dtype: str = "bf16"            # storage/act dtype: "f32" or "bf16"; accumulation is fp32 or wider
    x_sigma: float = 1.0
    router_sigma: float = 0.02
    w_sigma: float = 0.02          # gate/up/down of routed and shared experts
    fan_in_init: bool = False      # if True: every weight ~N(0, 1/fan_in) instead of w_sigma
    bias: tuple = ("const", 0.0)   # selection bias recipe
    capacity_factor: float = 0.0   # <= 0: no capacity limit
    rms_eps: float = 1e-6
    gamma: float = 1e-3            # bias update step
    # (expert, a, c): add a to h[:, 0] and c/a to w_router[expert, 0]
    skew: tuple | None = None
    seed: int = 0
    description: str = ""

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)


@dataclass(frozen=True)
class TensorSpec:
    shape: tuple
    tensor_id: int
    dist: tuple
    fp32: bool = False             # always fp32, whatever the layer dtype


def _sigma(cfg: LayerConfig, fan_in: int, default: float) -> float:
    return 1.0 / math.sqrt(fan_in) if cfg.fan_in_init else default


def layer_tensor_specs(cfg: LayerConfig) -> dict:
    N, d, E, H, Hs = cfg.n_tokens, cfg.d_model, cfg.n_experts, cfg.d_ff, cfg.d_ff_shared
    s = {
        "h": TensorSpec((N, d), TID_H, ("normal", cfg.x_sigma)),
        "norm_w": TensorSpec((d,), TID_NORM_W, ("const", 1.0)),
        "w_router": TensorSpec((E, d), TID_W_ROUTER, ("normal", _sigma(cfg, d, cfg.router_sigma))),
        "bias": TensorSpec((E,), TID_BIAS, cfg.bias, fp32=True),
        "w_gate": TensorSpec((E, H, d), TID_W_GATE, ("normal", _sigma(cfg, d, cfg.w_sigma))),
        "w_up": TensorSpec((E, H, d), TID_W_UP, ("normal", _sigma(cfg, d, cfg.w_sigma))),
        "w_down": TensorSpec((E, d, H), TID_W_DOWN, ("normal", _sigma(cfg, H, cfg.w_sigma))),
    }
    if Hs > 0:
        s["ws_gate"] = TensorSpec((Hs, d), TID_WS_GATE, ("normal", _sigma(cfg, d, cfg.w_sigma)))
        s["ws_up"] = TensorSpec((Hs, d), TID_WS_UP, ("normal", _sigma(cfg, d, cfg.w_sigma)))
        s["ws_down"] = TensorSpec((d, Hs), TID_WS_DOWN, ("normal", _sigma(cfg, Hs, cfg.w_sigma)))
    return s


# Constant c of the stress recipe: chosen by bisection with the oracle router
# at seed 0 so that 90% (+-1%) of top-1 choices land on expert 3; the not-gpu
# test suite re-derives the share from the oracle.
STRESS_C = 3.83

CONFIGS = {
    "tiny_fp32": LayerConfig(
        name="tiny_fp32", n_tokens=256, d_model=64, n_experts=8, top_k=2, d_ff=128,
        dtype="f32", fan_in_init=True,
        description="Tiny fp32 MoE layer: N=256, d=64, E=8, k=2, H=128, zero bias, no capacity"),
    "mixtral_bf16": LayerConfig(
        name="mixtral_bf16", n_tokens=4096, d_model=4096, n_experts=8, top_k=2, d_ff=14336,
        description="Mixtral-8x7B-shaped layer, bf16: N=4096, d=4096, E=8, k=2, H=14336"),
    "dsv3_prefill_bf16": LayerConfig(
        name="dsv3_prefill_bf16", n_tokens=8192, d_model=7168, n_experts=256, top_k=8,
        d_ff=2048, d_ff_shared=2048, bias=("uniform", -0.01, 0.01),
        description="DeepSeek-V3-shaped prefill, bf16: N=8192, d=7168, E=256, k=8, H=2048, 1 shared"),
    "dsv3_decode_bf16": LayerConfig(
        name="dsv3_decode_bf16", n_tokens=64, d_model=7168, n_experts=256, top_k=8,
        d_ff=2048, d_ff_shared=2048, bias=("uniform", -0.01, 0.01),
        description="DeepSeek-V3-shaped decode step, bf16: N=64, same shapes as prefill"),
    "stress_bf16": LayerConfig(
        name="stress_bf16", n_tokens=4096, d_model=4096, n_experts=8, top_k=2, d_ff=14336,
        capacity_factor=1.25, skew=(3, 8.0, STRESS_C),
        description="Load-imbalance stress, Mixtral shapes, ~90% top-1 on expert 3, C=1.25, "
                    "then one bias update with gamma=1e-3"),
}
