"""CPU oracle of the top-k routed MoE FFN layer forward -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm may import this module.  The CUDA library never
calls it, and it shares no code with the CUDA library.

Plain, slow and readable on purpose: numpy in float64 with library matmuls,
no blocking or fusion, one function per step of the method.  Sources (by
page title and section):

* [LESSON]   "Mixture of Experts (MoE)" lesson, AI Engineering from Scratch,
             Phase 07 Transformers Deep Dive (and its re-translation on
             nextadmin.net, "MoE architecture: load balancing and gating").
* [GLOSSARY] Ultralytics glossary, "Mixture of Experts (MoE)".
* [EP]       aiunderstanding.org, "Expert parallelism for MoE serving".

The layer, from [LESSON] "The concept / Swapping the FFN" (MoE block):
    scores = router(norm(h)); top_k = argmax_k(scores);
    h = h + sum_{e in top_k} gate(scores[e]) * Expert_e(norm(h))
with SwiGLU experts ("each expert is an independent FFN, usually SwiGLU"),
a linear router without bias, selection on scores + bias with gates from the
raw scores ([LESSON] "The load-balancing problem", DeepSeek-V3 approach, and
"Step 1: the router"), an optional always-on shared expert ([LESSON]
"Shared experts"), optional expert capacity with overflow slots skipping the
experts ([LESSON] "The load-balancing problem"; [GLOSSARY] "Load balancing
and expert capacity"), and the +-gamma bias update ([LESSON] "Step 2").

Readings taken where the pages are silent (each one is listed with its
reason in the design notes):
* norm = RMSNorm, x / sqrt(mean(x^2) + eps) * w, one normalised xn feeding
  the router, the routed experts and the shared expert.
* scores = softmax over the E router logits; the selection key is
  score + bias in fp32; ties go to the lower expert index (the lesson's
  route() sorts stably); gates = chosen scores renormalised over the k
  chosen, which equals the lesson's softmax over the chosen raw logits.
* capacity = floor(C * N * k / E); slots are taken in (token, rank) order
  and the first `capacity` slots of an expert are kept; a dropped slot adds
  nothing and the remaining gates are not renormalised.
* bias_e += gamma * sign(target - count_e), sign(0) = 0, counts taken
  before the capacity cut, in fp32.
* Quantisation points (storage dtype "bf16" or "f32"): xn, the SwiGLU
  activation and the layer output are rounded to the storage dtype; the
  rounding of xn is decided in fp32 (the kernel's precision), as
  bf16(fl32(fl32(h * r) * w)) with r = fl32(1 / sqrt(mean(h^2) + eps))
  and mean(h^2) summed in float64.  Everything else is float64.

Parity of the expert GEMM values is pinned only through the E=1 / k=1
textbook-SwiGLU identity and the k=E dense identity of the test suite.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_to", "rmsnorm", "router_scores", "select_topk", "gates_from_scores",
    "expert_counts", "capacity_limit", "permute", "silu", "swiglu_expert",
    "combine", "layer_forward", "bias_update", "balancing_loop", "load_stats", "splitmix64", "hash_route",
]


# ----------------------------------------------------------------------------
# Storage rounding
# ----------------------------------------------------------------------------

def round_to(x, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype, returned as float64.

    "f32": IEEE round to nearest even.  "bf16": nearest value with an 8-bit
    significand, ties to even (frexp gives x = m * 2**e with 0.5 <= |m| < 1,
    so m * 256 holds the 8 kept bits; np.rint rounds half to even).  Valid for
    the normal range of bf16, which every value here lies in.
    """
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        m, e = np.frexp(x)
        return np.ldexp(np.rint(m * 256.0), e - 8)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# a1. RMSNorm  ([LESSON] MoE block: norm(h) feeds both router and experts)
# ----------------------------------------------------------------------------

def rmsnorm(h, norm_w, eps: float, dtype: str) -> np.ndarray:
    """xn = h / sqrt(mean(h^2) + eps) * w, rounded to the storage dtype.

    The mean of squares is summed in float64; the scale r and the two
    products are fp32 so that the storage rounding is decided in fp32.
    """
    h = np.asarray(h)
    h64 = h.astype(np.float64)
    ms = np.mean(h64 * h64, axis=1)
    r32 = (1.0 / np.sqrt(ms + float(np.float32(eps)))).astype(np.float32)
    t = h.astype(np.float32) * r32[:, None]
    t = t * np.asarray(norm_w, dtype=np.float32)[None, :]
    return round_to(t.astype(np.float64), dtype)


# ----------------------------------------------------------------------------
# a2. Router: linear layer without bias, then softmax over the E experts
#     ([LESSON] "Step 1: the router": scores[e] = sum_i h_i * W_router[e, i];
#      [GLOSSARY] "How an MoE layer works": one linear layer scores every
#      expert, outputs are weighted by the normalised router scores)
# ----------------------------------------------------------------------------

def router_scores(xn, w_router):
    """Return (logits, scores): logits = xn @ W_router^T, scores = softmax(logits)."""
    logits = np.asarray(xn, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T
    shifted = logits - logits.max(axis=1, keepdims=True)
    ex = np.exp(shifted)
    return logits, ex / ex.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# a3. Top-k on scores + bias; gates from the raw scores
#     ([LESSON] "The load-balancing problem", DeepSeek-V3: selection uses
#      scores + bias, gating uses the unmodified scores; "Step 1: the router":
#      stable sort by -biased, softmax over the chosen ORIGINAL scores)
# ----------------------------------------------------------------------------

def select_topk(scores, bias, k: int):
    """Choose k experts per token by descending key = fl32(score) + fl32(bias).

    Returns (idx [N, k] int32 ordered by descending key, key [N, E] fp32).
    Equal keys keep ascending expert order (a stable sort), so the lower
    expert index wins a tie.
    """
    key = np.asarray(scores).astype(np.float32) + np.asarray(bias, dtype=np.float32)[None, :]
    order = np.argsort(-key, axis=1, kind="stable")
    return order[:, :k].astype(np.int32), key


def gates_from_scores(scores, idx) -> np.ndarray:
    """gate_j = score[idx_j] / sum over the chosen k of score."""
    chosen = np.take_along_axis(np.asarray(scores, dtype=np.float64), idx.astype(np.int64), axis=1)
    return chosen / chosen.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# a4. Per-expert counts, capacity and the stable permutation
#     ([LESSON] "The load-balancing problem": capacity C x N / E, overflow
#      tokens pass the layer; [GLOSSARY] "Load balancing and expert
#      capacity": tokens per expert by bincount, overflow continues on the
#      residual; [EP] "Technical insight": dispatch groups each expert's
#      tokens, capacity keeps each expert's GEMM shape predictable)
# ----------------------------------------------------------------------------

def expert_counts(idx, n_experts: int) -> np.ndarray:
    """Tokens routed to each expert before any capacity cut (sum = N * k)."""
    return np.bincount(np.asarray(idx).ravel(), minlength=n_experts).astype(np.int64)


def capacity_limit(capacity_factor: float, n_tokens: int, top_k: int, n_experts: int) -> int:
    """floor(C * N * k / E) with C taken as fp32; -1 (no limit) when C <= 0."""
    c = float(np.float32(capacity_factor))
    if c <= 0:
        return -1
    return int(np.floor(c * n_tokens * top_k / n_experts))


def permute(idx, n_experts: int, capacity: int = -1):
    """Stable counting sort of the N*k routing slots by expert.

    Slot s = t * k + j is visited in increasing s (token, then rank).  Its
    rank within expert e is the number of earlier slots routed to e; with a
    capacity, slots of rank >= capacity are dropped.  Kept slots of expert e
    take rows offsets[e] + rank of the expert-contiguous buffer.

    Returns (offsets [E+1], slot_row [N*k] (-1 = dropped), row_token [R]).
    """
    flat = np.asarray(idx).ravel().astype(np.int64)
    k = np.asarray(idx).shape[1]
    rank = np.empty(flat.size, dtype=np.int64)
    seen = np.zeros(n_experts, dtype=np.int64)
    for s, e in enumerate(flat.tolist()):
        rank[s] = seen[e]
        seen[e] += 1
    kept_per_expert = seen if capacity < 0 else np.minimum(seen, capacity)
    offsets = np.concatenate([[0], np.cumsum(kept_per_expert)]).astype(np.int64)
    keep = np.ones(flat.size, dtype=bool) if capacity < 0 else rank < capacity
    slot_row = np.where(keep, offsets[flat] + rank, -1).astype(np.int64)
    row_token = np.empty(int(offsets[-1]), dtype=np.int64)
    row_token[slot_row[keep]] = (np.arange(flat.size) // k)[keep]
    return offsets, slot_row, row_token


# ----------------------------------------------------------------------------
# a6-a8. SwiGLU expert FFN ([LESSON] "each expert is an independent FFN,
#        usually SwiGLU"); the shared expert is the same FFN applied to every
#        token ([LESSON] "Shared experts")
# ----------------------------------------------------------------------------

def silu(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_expert(x, w_gate, w_up, w_down, dtype: str) -> np.ndarray:
    """y = W_down (silu(W_gate x) * (W_up x)), activation rounded to dtype.

    x: [rows, d]; w_gate, w_up: [H, d]; w_down: [d, H].  Returns [rows, d].
    """
    x = np.asarray(x, dtype=np.float64)
    u = x @ np.asarray(w_gate, dtype=np.float64).T
    v = x @ np.asarray(w_up, dtype=np.float64).T
    a = round_to(silu(u) * v, dtype)
    return a @ np.asarray(w_down, dtype=np.float64).T


# ----------------------------------------------------------------------------
# a9. Gated combine plus residual ([LESSON] MoE block: h + sum gate * Expert;
#     [GLOSSARY] example: out[token] += weight * expert(token))
# ----------------------------------------------------------------------------

def combine(h, y_slots, gates, slot_row, y_shared=None):
    """out = h + sum over kept slots j of gate_j * y_j (+ y_shared), float64.

    y_slots: [N, k, d] expert outputs per slot (ignored where dropped);
    slot_row: [N*k] with -1 for a dropped slot.  The caller rounds the
    result to the storage dtype with ``round_to``.
    """
    h64 = np.asarray(h, dtype=np.float64)
    n, k = gates.shape
    kept = (np.asarray(slot_row).reshape(n, k) >= 0).astype(np.float64)
    out = h64 + np.einsum("tj,tjd->td", gates * kept, np.asarray(y_slots, dtype=np.float64))
    if y_shared is not None:
        out = out + y_shared
    return out


# ----------------------------------------------------------------------------
# a10. Aux-loss-free bias update ([LESSON] "The load-balancing problem":
#      after each step, +-gamma per expert by over- or under-use against the
#      target; "Step 2": -gamma for over-used, +gamma for under-used)
# ----------------------------------------------------------------------------

def bias_update(bias, counts, target: float, gamma: float) -> np.ndarray:
    """bias_e <- fl32(bias_e + gamma * sign(target - count_e)), sign(0) = 0."""
    b = np.asarray(bias, dtype=np.float32)
    c = np.asarray(counts).astype(np.float32)
    s = np.sign(np.float32(target) - c).astype(np.float32)
    return (b + s * np.float32(gamma)).astype(np.float32)


def balancing_loop(scores, bias0, k: int, target: float, gamma: float, iterations: int):
    """Repeated aux-loss-free balancing on fixed router scores.

    [LESSON] "Step 2: run 100 tokens through the router": route every token,
    count each expert's load, move every bias by -gamma (over target) or
    +gamma (under target), repeat.  Each iteration selects on the current
    bias (select_topk), counts before any capacity cut (expert_counts) and
    applies bias_update.  Returns (counts [iterations, E], biases
    [iterations + 1, E] fp32), biases[0] = bias0.
    """
    bias = np.asarray(bias0, dtype=np.float32).copy()
    n_experts = np.asarray(scores).shape[1]
    counts, biases = [], [bias.copy()]
    for _ in range(iterations):
        idx, _ = select_topk(scores, bias, k)
        c = expert_counts(idx, n_experts)
        bias = bias_update(bias, c, target, gamma)
        counts.append(c)
        biases.append(bias.copy())
    return np.array(counts), np.array(biases)


def load_stats(counts, offsets, n_tokens: int, top_k: int, n_experts: int) -> dict:
    """Load statistics of one routing.

    [LESSON] "The load-balancing problem" (each expert's usage against the
    target N*k/E; with a capacity, overflow slots are dropped and pass the
    layer) and [GLOSSARY] "Load balancing and expert capacity" (tokens per
    expert counted; overflow continues on the residual).  routed = N*k
    slots; kept = the slots the capacity let through (offsets[E]); dropped =
    routed - kept; max_count = the largest count before the cut; and
    max_over_mean = max_count over the mean load N*k/E, both divisions in
    fp32 rounded to nearest, as the library defines it.  All zero for N = 0.
    """
    routed = int(n_tokens) * int(top_k)
    if routed == 0:
        return {"routed": 0, "kept": 0, "dropped": 0, "max_count": 0, "max_over_mean": np.float32(0.0)}
    kept = int(np.asarray(offsets)[n_experts])
    max_count = int(np.max(np.asarray(counts)))
    mean = np.float32(np.float32(routed) / np.float32(n_experts))
    return {"routed": routed, "kept": kept, "dropped": routed - kept, "max_count": max_count,
            "max_over_mean": np.float32(np.float32(max_count) / mean)}


# ----------------------------------------------------------------------------
# Hash router ([LESSON] "Exercises": a hash router that routes tokens without
# learning).  Reading taken: the expert of choice j is (h(id) + j) mod E, with
# h the SplitMix64 output function (Steele, Lea, Flood 2014) applied to the
# token id, and every chosen expert gets gate 1/k.
# ----------------------------------------------------------------------------

_M64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One SplitMix64 output for state x: mix(x + golden gamma), 64-bit wrap."""
    z = (x + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def hash_route(token_ids, n_experts: int, k: int):
    """Returns (idx [N, k] int64, gates [N, k] float32)."""
    ids = [int(t) & _M64 for t in np.asarray(token_ids).ravel().tolist()]
    idx = np.empty((len(ids), k), dtype=np.int64)
    for t, tid in enumerate(ids):
        e0 = splitmix64(tid) % n_experts
        for j in range(k):
            idx[t, j] = (e0 + j) % n_experts
    gates = np.full((len(ids), k), np.float32(1.0) / np.float32(k), dtype=np.float32)
    return idx, gates


# ----------------------------------------------------------------------------
# The whole layer (small problems; large ones use the steps above on samples)
# ----------------------------------------------------------------------------

def layer_forward(h, norm_w, w_router, bias, w_gate, w_up, w_down, *, top_k: int,
                  eps: float, dtype: str, capacity_factor: float = 0.0,
                  ws_gate=None, ws_up=None, ws_down=None) -> dict:
    """Forward pass of the MoE layer, following the MoE block of [LESSON].

    The routed experts run as in the [GLOSSARY] example: for each expert,
    gather the kept slots that chose it, run its FFN on their tokens, and
    scatter the results back to the slots.
    """
    h = np.asarray(h)
    n, d = h.shape
    n_experts = np.asarray(w_router).shape[0]
    xn = rmsnorm(h, norm_w, eps, dtype)
    logits, scores = router_scores(xn, w_router)
    idx, key = select_topk(scores, bias, top_k)
    gates = gates_from_scores(scores, idx)
    counts = expert_counts(idx, n_experts)
    cap = capacity_limit(capacity_factor, n, top_k, n_experts)
    offsets, slot_row, row_token = permute(idx, n_experts, cap)
    kept = (slot_row >= 0).reshape(n, top_k)
    y = np.zeros((n, top_k, d), dtype=np.float64)
    for e in range(n_experts):
        t_idx, j_idx = np.nonzero((idx == e) & kept)
        if t_idx.size:
            y[t_idx, j_idx] = swiglu_expert(xn[t_idx], w_gate[e], w_up[e], w_down[e], dtype)
    y_shared = None
    if ws_gate is not None:
        y_shared = swiglu_expert(xn, ws_gate, ws_up, ws_down, dtype)
    out64 = combine(h, y, gates, slot_row, y_shared)
    return {
        "xn": xn, "logits": logits, "scores": scores, "key": key, "idx": idx,
        "gates": gates, "counts": counts, "capacity": cap, "offsets": offsets,
        "slot_row": slot_row, "row_token": row_token, "y": y, "y_shared": y_shared,
        "out64": out64, "out": round_to(out64, dtype),
    }
