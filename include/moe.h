/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE-layer forward library, libmoe_b200.so.
 *
 * The library computes the forward pass of a top-k routed Mixture-of-Experts
 * FFN layer with an optional always-on shared expert:
 *
 *     xn  = RMSNorm(h)
 *     out = h + sum_{e in topk(score + bias)} gate_e * SwiGLU_e(xn) [+ SwiGLU_shared(xn)]
 *
 * as stated by the "Mixture of Experts (MoE)" lesson of AI Engineering from
 * Scratch (Phase 07), section "The concept / Swapping the FFN" (the MoE
 * block: scores = router(norm(h)), top_k = argmax_k(scores),
 * h = h + sum gate(scores[e]) * Expert_e(norm(h))), with its load-balancing
 * sections (capacity, auxiliary-loss-free bias) and "Shared experts".
 *
 * Conventions (every entry point):
 *  - Every pointer argument is DEVICE memory owned by the caller, except
 *    where a comment says "host".  The library never allocates or frees
 *    memory and never synchronises the stream (moe_check_device_error is the
 *    one exception, and says so).  All work is enqueued on `stream`, a
 *    cudaStream_t passed as void* (NULL = the legacy default stream), on the
 *    calling thread's current device.
 *  - Tensors are dense and row-major (last index fastest), with the
 *    element type given by moe_config.dtype ("act dtype") unless stated.
 *    Accumulation is always fp32 or wider.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns an error status and enqueues nothing.  Launch
 *    failures map to MOE_ERR_CUDA.  A device-side wait that exceeds its limit
 *    records MOE_ERR_DEVICE_TIMEOUT in the workspace header; it is reported by
 *    moe_check_device_error.
 *  - Calls are asynchronous: outputs are valid once the stream reaches them.
 *    Calls that share a workspace must not overlap on the GPU.
 *  - Entry points may be called from several host threads at once.  The
 *    library's host state is per-device caches (SM count, kernel shared-memory
 *    limits, the tensor-map encoder) guarded by atomics and a mutex, and the
 *    two process-wide settings (moe_set_wait_timeout_ns, moe_set_gemm_tiling),
 *    which apply to calls that start after them.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,     /* a NULL required pointer, a bad size or a bad dtype */
  MOE_ERR_UNSUPPORTED = 2,     /* valid, but outside what the kernels handle (e.g. bf16 d % 8 != 0) */
  MOE_ERR_WORKSPACE = 3,       /* ws_bytes smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,            /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 5   /* a bounded device-side wait gave up (see moe_check_device_error) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Layer shape and options. */
typedef struct {
  int32_t n_tokens;        /* N >= 0 (N = 0 is a no-op) */
  int32_t d_model;         /* d >= 1 */
  int32_t n_experts;       /* E in [1, 1024] routed experts */
  int32_t top_k;           /* k in [1, min(E, 32)] */
  int32_t d_ff;            /* H >= 1, hidden width of each routed SwiGLU expert */
  int32_t d_ff_shared;     /* Hs >= 0, hidden width of the shared expert; 0 = none */
  int32_t dtype;           /* moe_dtype of activations and weights */
  float rms_eps;           /* RMSNorm epsilon, >= 0 (1e-6 in every workload here) */
  float capacity_factor;   /* <= 0: no capacity; else cap = floor(C * N * k / E) slots per expert */
} moe_config;

/* Device pointers to the layer weights (act dtype unless stated). */
typedef struct {
  const void* norm_w;      /* [d]          RMSNorm scale */
  const void* w_router;    /* [E][d]       router, no bias (nn.Linear out x in) */
  const void* w_gate;      /* [E][H][d]    routed experts, gate projection */
  const void* w_up;        /* [E][H][d]    routed experts, up projection */
  const void* w_down;      /* [E][d][H]    routed experts, down projection */
  const void* ws_gate;     /* [Hs][d]      shared expert (NULL when Hs = 0) */
  const void* ws_up;       /* [Hs][d] */
  const void* ws_down;     /* [d][Hs] */
} moe_weights;

/* Optional device outputs of the routing steps.  Any member may be NULL; a
 * NULL member is kept in the workspace instead (scores: not produced). */
typedef struct {
  float* scores;           /* [N][E]   fp32 softmax router scores */
  int32_t* topk_idx;       /* [N][k]   chosen experts, descending score + bias, lower index first on ties */
  float* topk_gate;        /* [N][k]   fp32 gates: chosen scores renormalised over the k */
  int32_t* counts;         /* [E]      tokens routed to each expert before the capacity cut (sum = N*k) */
  int32_t* offsets;        /* [E+1]    exclusive scan of the kept counts */
  int32_t* slot_row;       /* [N*k]    row of slot t*k+j in the expert-sorted buffers, -1 = dropped */
  int32_t* row_token;      /* [N*k]    token of each expert-sorted row (first offsets[E] valid) */
} moe_routing;

/* Optional stage timing: each non-NULL member is a cudaEvent_t recorded on
 * the stream when moe_layer_forward reaches that point. */
typedef struct {
  void* start;             /* before the first kernel */
  void* routed;            /* after RMSNorm, router, top-k (moe_route) */
  void* permuted;          /* after counting sort and gather (moe_permute) */
  void* gate_up;           /* after the routed gate/up + SwiGLU grouped GEMM */
  void* down;              /* after the routed down grouped GEMM */
  void* shared;            /* after the shared expert (== down when Hs = 0) */
  void* combined;          /* after the combine + residual */
} moe_trace;

/* Human-readable name of a status code (static storage). */
const char* moe_status_string(int32_t status);

/* Library build string (static storage). */
const char* moe_version(void);

/* Bytes of device workspace that moe_layer_forward needs for this config,
 * and that is also enough for every staged call below with the same config;
 * 0 if the config is invalid.  The workspace holds a 256-byte header (the
 * device error word, and the tile counter of the swapped-operand expert GEMMs,
 * which each of their launches zeroes first), xn, the routing buffers that
 * moe_routing leaves NULL, router
 * logits, permutation histograms, the expert-sorted rows x_perm [R][d],
 * activations [max(R*H, N*Hs)] and expert outputs y_perm [R][d], y_shared
 * [N][d], where R = N*k, or min(N*k, E*cap) with a capacity.  When the
 * shared expert is as wide as the routed ones (bf16, Hs == H) it runs as one
 * more group of the routed expert GEMMs, reading its input rows from xn:
 * act and y_perm then hold R + N rows and there is no separate y_shared. */
size_t moe_workspace_size(const moe_config* cfg);

/* Zero the workspace header (the device error word).  Call once after
 * allocating a workspace, before its first use. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Steps a1-a3: RMSNorm, router and top-k selection.
 * Lesson "Step 1: the router" (scores of every expert, selection on
 * scores + bias, gates from the chosen raw scores) and "The load-balancing
 * problem" (DeepSeek-V3 bias on selection only).
 *   h        [N][d]  input hidden states
 *   norm_w   [d]     RMSNorm scale
 *   w_router [E][d]
 *   bias     [E]     fp32 selection bias, NULL = zeros
 *   xn       [N][d]  out: RMSNorm(h), act dtype
 *   scores   [N][E]  out (NULL = not written): fp32 softmax of the router logits
 *   topk_idx [N][k], topk_gate [N][k] (fp32), counts [E]: out, as in moe_routing;
 *                    counts is overwritten (not accumulated).
 * xn = bf16/fp32(fl32(fl32(h * r) * w)), r = fl32(1/sqrt(mean(h^2) + eps)), mean in fp64. */
moe_status moe_route(const moe_config* cfg, const void* h, const void* norm_w, const void* w_router,
                     const float* bias, void* xn, float* scores, int32_t* topk_idx, float* topk_gate,
                     int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/* Hash routing in place of steps a2-a3 (the lesson's exercise of a hash
 * router that routes without learning: "Mixture of Experts (MoE)" lesson,
 * "Exercises").  Computes xn = RMSNorm(h) as moe_route does, then for token
 * t with id x = token_ids[t] (token_ids NULL: x = t) chooses experts
 *   e_j = (splitmix64(x) + j) mod E,  j = 0 .. k-1,
 * splitmix64 being the SplitMix64 output function (Steele, Lea and Flood,
 * 2014), with every gate 1/k.  The result feeds moe_permute, moe_expert_ffn
 * and moe_combine unchanged.
 *   token_ids [N] int64 device or NULL; xn, topk_idx, topk_gate, counts: out,
 *   as in moe_route.  Errors as moe_route. */
moe_status moe_route_hash(const moe_config* cfg, const void* h, const void* norm_w, const int64_t* token_ids,
                          void* xn, int32_t* topk_idx, float* topk_gate, int32_t* counts, void* ws, size_t ws_bytes,
                          void* stream);

/* Step a4-a5: per-expert counting sort of the N*k routing slots, capacity and
 * gather.  Glossary "Load balancing and expert capacity" (tokens per expert,
 * overflow continues on the residual); lesson "The load-balancing problem"
 * (capacity C x N / E); "Expert parallelism for MoE serving", "Technical
 * insight" (dispatch groups tokens by expert; capacity keeps GEMM shapes
 * predictable).  Slot s = t*k + j is ranked among the slots of its expert
 * in increasing s; ranks >= cap are dropped (slot_row = -1).
 *   topk_idx  [N][k] in
 *   xn        [N][d] in
 *   offsets   [E+1]  out: offsets[e] = sum of kept counts of experts < e
 *   slot_row  [N*k]  out
 *   row_token [N*k]  out (first offsets[E] entries valid)
 *   x_perm    [R][d] out: x_perm[slot_row[s]] = xn[s / k] for kept slots
 * The gather's device-side waits (on its bulk row copies) are bounded by
 * moe_set_wait_timeout_ns; a time-out is recorded in the workspace error
 * word (moe_check_device_error). */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* xn, int32_t* offsets,
                       int32_t* slot_row, int32_t* row_token, void* x_perm, void* ws, size_t ws_bytes,
                       void* stream);

/* Maximum histogram entries, E * ceil(N*k / 256), that moe_permute_noalloc
 * can handle: 262144 int32 (1 MiB). */
#define MOE_NOALLOC_HIST_INTS 262144

/* moe_permute without a workspace, for callers that cannot hand the library
 * device memory for scratch: a plugin or callback that only receives its
 * own input and output buffers, or a loop that must not allocate once it is
 * running (cudaMalloc can synchronise the device and take unbounded time).
 * The pages have no counterpart to this call; it is a deployment variant of
 * moe_permute.
 *
 * Arguments, results and errors are those of moe_permute, minus ws/ws_bytes.
 * The chunk histograms live in a fixed 1 MiB device array inside the
 * library instead; every GPU that loads the library holds it until the
 * process exits.  Rules:
 *  - E * ceil(N*k / 256) must not exceed MOE_NOALLOC_HIST_INTS, else the
 *    call returns MOE_ERR_WORKSPACE and enqueues nothing;
 *  - the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it for the process; make that first
 *    call before any stream capture.  The cached address belongs to the
 *    device's primary context: after cudaDeviceReset, or with another
 *    driver-API context current, the call is not supported;
 *  - every call on a device shares the one array: calls that overlap on the
 *    GPU (other streams, other threads) race and give wrong results;
 *  - with no workspace there is no error word: a device-side wait of the
 *    gather that runs out (see moe_permute) ends its block without a record.
 * The call allocates nothing and frees nothing. */
moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx, const void* xn, int32_t* offsets,
                               int32_t* slot_row, int32_t* row_token, void* x_perm, void* stream);

/* Steps a6-a8: grouped SwiGLU expert FFN, y = W_down(silu(W_gate x) * (W_up x)).
 * Lesson "The concept" (each expert an independent FFN, usually SwiGLU);
 * "Expert parallelism for MoE serving", "Future" (GEMM units that batch many
 * experts).  Rows [offsets[g], offsets[g+1]) of x use expert g's weights.
 *   n_groups  G >= 1 experts stacked in w_gate/w_up [G][d_ff][d], w_down [G][d][d_ff]
 *   offsets   [G+1] device, nondecreasing, offsets[G] <= max_rows; NULL = one
 *             group of max_rows rows (the shared expert: x = xn, max_rows = N)
 *   max_rows  rows that x and y hold (a host-side bound on offsets[G])
 *   x         [max_rows][d] in;  y [max_rows][d] out, act dtype; rows at or
 *             past offsets[G] are not written.
 * The SwiGLU activation (act dtype) is kept in the workspace. */
moe_status moe_expert_ffn(const moe_config* cfg, int32_t n_groups, const int32_t* offsets, int32_t max_rows,
                          const void* x, const void* w_gate, const void* w_up, const void* w_down,
                          int32_t d_ff, void* y, void* ws, size_t ws_bytes, void* stream);

/* Step a9: gated combine plus residual, in gather form (deterministic):
 * out[t] = h[t] + sum_{j, slot kept} gate[t][j] * y_perm[slot_row[t*k+j]] (+ y_shared[t]),
 * summed in fp32 and rounded once.  Lesson MoE block (h + sum gate * Expert);
 * glossary example (out[token] += weight * expert(token)).
 *   h [N][d], y_perm [R][d], slot_row [N*k], topk_gate [N][k] fp32,
 *   y_shared [N][d] or NULL, out [N][d] (may equal h).
 * y_perm may be NULL only when the capacity is 0 (every slot dropped). */
moe_status moe_combine(const moe_config* cfg, const void* h, const void* y_perm, const int32_t* slot_row,
                       const float* topk_gate, const void* y_shared, void* out, void* stream);

/* The whole forward pass: moe_route, moe_permute, moe_expert_ffn (routed
 * experts, then the shared expert when Hs > 0) and moe_combine, on one
 * stream with no host synchronisation.
 *   weights   device pointers (struct itself on the host)
 *   h [N][d] in, bias [E] fp32 or NULL, out [N][d] (may equal h)
 *   routing   host struct of optional device outputs, or NULL
 *   trace     host struct of optional cudaEvent_t, or NULL */
moe_status moe_layer_forward(const moe_config* cfg, const moe_weights* weights, const void* h,
                             const float* bias, void* out, const moe_routing* routing,
                             const moe_trace* trace, void* ws, size_t ws_bytes, void* stream);

/* Step a10: auxiliary-loss-free bias update.  Lesson "The load-balancing
 * problem" (after each step, +-gamma per expert by usage above or below
 * target) and "Step 2" (-gamma for over-used, +gamma for under-used experts):
 *   bias[e] = fl32(bias[e] + gamma * sign(target - counts[e])), sign(0) = 0.
 *   counts [E] int32 in, bias [E] fp32 in/out. */
moe_status moe_bias_update(int32_t n_experts, const int32_t* counts, float target, float gamma, float* bias,
                           void* stream);

/* Load statistics of one routing (steps a4 and a10).  Lesson "The
 * load-balancing problem" (usage per expert against the target; with a
 * capacity of C x N / E, overflow tokens pass the layer unprocessed) and
 * "Step 2" (the usage that moves each bias); Ultralytics glossary "Load
 * balancing and expert capacity" (tokens per expert counted; overflow
 * continues on the residual).
 *   routed        = N*k, the slots the top-k chose;
 *   kept          = offsets[E], the slots that reached an expert;
 *   dropped       = routed - kept (0 without a capacity);
 *   max_count     = max over e of counts[e], taken before the capacity cut;
 *   max_over_mean = fl32(max_count) / fl32(fl32(N*k) / fl32(E)), fp32
 *                   divisions rounded to nearest (the mean load is the
 *                   target usage N*k/E; 1 is perfect balance).
 * counts [E] and offsets [E+1] are device int32 from moe_route / moe_permute
 * or the moe_routing outputs of moe_layer_forward, for the same config;
 * stats is one device moe_load_stats, written by one small kernel on
 * `stream`.  MOE_ERR_INVALID_ARG for an invalid config or a NULL pointer
 * (N = 0 writes routed = kept = dropped = max_count = 0, max_over_mean = 0). */
typedef struct {
  int32_t routed;
  int32_t kept;
  int32_t dropped;
  int32_t max_count;
  float max_over_mean;
} moe_load_stats;

moe_status moe_compute_load_stats(const moe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                  moe_load_stats* stats, void* stream);

/* Synchronise `stream`, read and clear the workspace's device error word.
 * Returns MOE_OK, the recorded status (e.g. MOE_ERR_DEVICE_TIMEOUT) or
 * MOE_ERR_CUDA.  info (host, may be NULL) receives 4 int32 of detail
 * (status, kernel id, block, wait site).  This call blocks the host. */
moe_status moe_check_device_error(void* ws, size_t ws_bytes, void* stream, int32_t* info);

/* Limit, in nanoseconds, of every bounded device-side wait in kernels
 * launched after this call (process-wide; default 2e9 = 2 s; 0 = give up at
 * the first unsuccessful poll). */
moe_status moe_set_wait_timeout_ns(int64_t ns);

/* Tile shape of the bf16 grouped expert GEMMs for launches after this call
 * (process-wide): 0 = choose per launch (the default: SM-pair tiles with the
 * operands swapped -- 256 weight rows on M, up to 256 of a group's rows on
 * N, padded to 16 -- for every gate/up projection with d % 64 == 0, and for
 * the down projection when the groups average at least 64 rows and
 * H % 64 == 0; single-SM 128-row tiles (64-row for small groups) for the
 * other gate/up launches and the other down projections of smaller groups;
 * for the other down projections of groups averaging at least 512 rows,
 * single-SM or SM-pair 256-row tiles picked on the device from the group
 * sizes), 1 = single-SM tiles, 2 = SM-pair tiles, 3 = swapped-operand SM-pair
 * tiles for both expert GEMMs where the shape allows (K % 64 == 0).  The
 * tensor-core router (bf16, E >= 64, N >= 512) always runs single-SM
 * tiles of 128 rows and 128 columns (256 when that takes fewer waves) whose
 * fp32 accumulation restarts every 256 along d, the partial sums added in
 * fp32 registers, whatever the mode.  Results are the
 * same up to floating-point summation order; this is a performance control.
 * MOE_ERR_INVALID_ARG for any other mode. */
moe_status moe_set_gemm_tiling(int32_t mode);

/* Launch one block that waits on a workspace flag that nothing sets, with
 * the current wait limit: it must give up and record MOE_ERR_DEVICE_TIMEOUT.
 * Exercises the timeout path without faulting or hanging the GPU. */
moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
