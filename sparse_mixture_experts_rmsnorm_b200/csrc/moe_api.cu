// C-ABI entry points of libmoe_b200.so: argument checks, the workspace
// layout and the order of the kernels on the caller's stream.  No entry
// point allocates device memory, and only moe_check_device_error
// synchronises.

#include "moe_common.cuh"
#include "moe_kernels.h"
#include "tcgen05.cuh"

namespace moe_host {

static std::atomic<uint64_t> g_wait_ns{2000000000ull};
uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int sm_count() {
  static std::atomic<int> cache[64] = {};
  int d = current_device();
  if (d >= 0 && d < 64) {
    const int c = cache[d].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
  if (d >= 0 && d < 64) cache[d].store(n, std::memory_order_relaxed);
  return n;
}

// ---------------------------------------------------------------------------
// Workspace layout (every region 256-byte aligned)
// ---------------------------------------------------------------------------
struct Layout {
  size_t hdr, xn, logits, idx, gate, counts, offsets, offsets_ext, slot_row, row_token, hist, x_perm, act, y_perm,
      y_shared, total;
  bool fold;         // the shared expert runs as one more group of the routed GEMMs
  int64_t rows;      // R: rows of the expert-sorted buffers
  int64_t act_elems; // max(R * H, N * Hs)
};

// floor(C*N*k/E), clamped to N*k: an expert never receives more than N*k
// slots, so any larger cap keeps every slot, and the clamped value always fits
// an int (config_ok bounds N*k).
int64_t capacity_of(const moe_config* c) {
  if (!(c->capacity_factor > 0.f)) return -1;
  const int64_t slots = (int64_t)c->n_tokens * c->top_k;
  const double cap = floor((double)c->capacity_factor * (double)c->n_tokens * (double)c->top_k / (double)c->n_experts);
  return cap >= (double)slots ? slots : (int64_t)cap;
}

static Layout layout_of(const moe_config* c) {
  Layout L;
  const size_t es = c->dtype == MOE_BF16 ? 2 : 4;
  const int64_t N = c->n_tokens, d = c->d_model, E = c->n_experts, k = c->top_k;
  const int64_t cap = capacity_of(c);
  int64_t R = N * k;
  if (cap >= 0 && E * cap < R) R = E * cap;
  L.rows = R;
  // bf16 layers with a shared expert as wide as the routed ones fold it into
  // the routed GEMMs: its N rows follow the R routed rows in act and y_perm,
  // and the gate/up GEMM reads its input rows straight from xn
  L.fold = c->dtype == MOE_BF16 && c->d_ff_shared > 0 && c->d_ff_shared == c->d_ff &&
           c->n_experts < moe::TC_MAX_GROUPS;
  const int64_t Rx = R + (L.fold ? N : 0);
  L.act_elems = Rx * c->d_ff;
  if (N * (int64_t)c->d_ff_shared > L.act_elems) L.act_elems = N * c->d_ff_shared;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.hdr = take(moe::kHeaderBytes);
  L.xn = take(N * d * es);
  L.logits = take(N * E * 4);
  L.idx = take(N * k * 4);
  L.gate = take(N * k * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.offsets_ext = take((E + 2) * 4);
  L.slot_row = take(N * k * 4);
  L.row_token = take(N * k * 4);
  L.hist = take(permute_hist_ints(N * k, (int)E) * 4);
  L.x_perm = take(R * d * es);
  L.act = take(L.act_elems * es);
  L.y_perm = take(Rx * d * es);
  L.y_shared = take(c->d_ff_shared > 0 && !L.fold ? N * d * es : 0);
  L.total = o;
  return L;
}

bool config_ok(const moe_config* c) {
  if (c == nullptr) return false;
  if (c->n_tokens < 0 || c->d_model < 1 || c->n_experts < 1 || c->n_experts > 1024) return false;
  if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > 32) return false;
  if (c->d_ff < 1 || c->d_ff_shared < 0) return false;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return false;
  if (!(c->rms_eps >= 0.f)) return false;
  if ((int64_t)c->n_tokens * c->top_k > 0x7fffffffLL) return false;
  return true;
}

// Shapes the kernels do not cover: bf16 rows must be whole 16-byte units for
// TMA (d % 8 == 0, H % 8 == 0, Hs % 8 == 0), and d <= 49152.
bool config_supported(const moe_config* c) {
  if (c->dtype == MOE_BF16) {
    if (c->d_model % 8 || c->d_ff % 8 || c->d_ff_shared % 8) return false;
  }
  if (c->d_model > 49152) return false;  // RMSNorm stages one fp32 row in shared memory
  return true;
}

static bool use_tc(const moe_config* c) { return c->dtype == MOE_BF16; }

static moe_status check_common(const moe_config* c, const void* ws, size_t ws_bytes) {
  if (!config_ok(c)) return MOE_ERR_INVALID_ARG;
  if (!config_supported(c)) return MOE_ERR_UNSUPPORTED;
  if (ws == nullptr || ((uintptr_t)ws % 256) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < layout_of(c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

#define MOE_TRY(x)                 \
  do {                             \
    moe_status _st = (x);          \
    if (_st != MOE_OK) return _st; \
  } while (0)

static inline char* wsp(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

// a2 on the tensor cores pays off once there are many tokens and experts;
// below that the router dot products ride along with RMSNorm.
static bool router_on_tc(const moe_config* c) {
  return use_tc(c) && c->n_experts >= 64 && c->n_tokens >= 512;
}

// counts == nullptr: no counts here (the layer forward takes them from the
// permute's scan instead, which needs no atomics).
static moe_status route_impl(const moe_config* c, const void* h, const void* norm_w, const void* w_router,
                             const float* bias, void* xn, float* scores, int32_t* topk_idx, float* topk_gate,
                             int32_t* counts, void* ws, cudaStream_t s) {
  const Layout L = layout_of(c);
  int32_t* hdr = (int32_t*)wsp(ws, L.hdr);
  float* logits = (float*)wsp(ws, L.logits);
  if (c->n_tokens > 0) {
    if (router_on_tc(c)) {
      MOE_TRY(launch_rmsnorm_router(c->dtype, h, norm_w, nullptr, xn, nullptr, c->n_tokens, c->d_model,
                                    c->n_experts, c->rms_eps, s));
      MOE_TRY(launch_gemm_tc(EPI_F32, xn, w_router, nullptr, nullptr, 1, c->n_tokens, c->n_experts, c->d_model,
                             logits, c->n_experts, hdr, s));
    } else {
      MOE_TRY(launch_rmsnorm_router(c->dtype, h, norm_w, w_router, xn, logits, c->n_tokens, c->d_model,
                                    c->n_experts, c->rms_eps, s));
    }
  }
  return launch_topk(logits, bias, scores, topk_idx, topk_gate, counts, c->n_tokens, c->n_experts, c->top_k, s);
}

static moe_status permute_impl(const moe_config* c, const int32_t* topk_idx, const void* xn, int32_t* offsets,
                               int32_t* slot_row, int32_t* row_token, void* x_perm, void* ws, cudaStream_t s,
                               int32_t* counts = nullptr) {
  const Layout L = layout_of(c);
  const int cap = (int)capacity_of(c);
  MOE_TRY(launch_permute(topk_idx, c->n_tokens, c->top_k, c->n_experts, cap, (int32_t*)wsp(ws, L.hist), offsets,
                         slot_row, row_token, s, nullptr, 0, counts));
  return launch_gather(c->dtype, xn, slot_row, c->n_tokens, c->top_k, x_perm, c->d_model, s, (int32_t*)wsp(ws, L.hdr));
}

static moe_status ffn_impl(const moe_config* c, int groups, const int32_t* offsets, int max_rows, const void* x,
                           const void* w_gate, const void* w_up, const void* w_down, int d_ff, void* y, void* ws,
                           cudaStream_t s) {
  const Layout L = layout_of(c);
  void* act = wsp(ws, L.act);
  int32_t* hdr = (int32_t*)wsp(ws, L.hdr);
  if (max_rows == 0) return MOE_OK;
  if (use_tc(c)) {
    MOE_TRY(launch_gemm_tc(EPI_SWIGLU, x, w_gate, w_up, offsets, groups, max_rows, d_ff, c->d_model, act, d_ff, hdr,
                           s));
    return launch_gemm_tc(EPI_STORE, act, w_down, nullptr, offsets, groups, max_rows, c->d_model, d_ff, y,
                          c->d_model, hdr, s);
  }
  MOE_TRY(launch_gemm_simt(c->dtype, EPI_SWIGLU, x, w_gate, w_up, offsets, groups, max_rows, d_ff, c->d_model, act,
                           d_ff, s));
  return launch_gemm_simt(c->dtype, EPI_STORE, act, w_down, nullptr, offsets, groups, max_rows, c->d_model, d_ff, y,
                          c->d_model, s);
}

}  // namespace moe_host

using namespace moe_host;

extern "C" {

const char* moe_status_string(int32_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or alignment not covered by the kernels";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace smaller than moe_workspace_size()";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a bounded device-side wait gave up";
    default: return "unknown moe_status";
  }
}

const char* moe_version(void) { return "moe_b200 0.1 (sm_100a; tcgen05 grouped GEMM, TMA, TMEM)"; }

size_t moe_workspace_size(const moe_config* cfg) {
  if (!config_ok(cfg)) return 0;
  return layout_of(cfg).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < moe::kHeaderBytes || ((uintptr_t)ws % 256) != 0) return MOE_ERR_INVALID_ARG;
  if (cudaMemsetAsync(ws, 0, moe::kHeaderBytes, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const void* h, const void* norm_w, const void* w_router,
                     const float* bias, void* xn, float* scores, int32_t* topk_idx, float* topk_gate,
                     int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  NvtxScope range("moe_route");
  MOE_TRY(check_common(cfg, ws, ws_bytes));
  if (cfg->n_tokens > 0 && (!h || !norm_w || !w_router || !xn || !topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if (!counts) return MOE_ERR_INVALID_ARG;
  return route_impl(cfg, h, norm_w, w_router, bias, xn, scores, topk_idx, topk_gate, counts, ws,
                    (cudaStream_t)stream);
}

moe_status moe_route_hash(const moe_config* cfg, const void* h, const void* norm_w, const int64_t* token_ids,
                          void* xn, int32_t* topk_idx, float* topk_gate, int32_t* counts, void* ws, size_t ws_bytes,
                          void* stream) {
  NvtxScope range("moe_route_hash");
  MOE_TRY(check_common(cfg, ws, ws_bytes));
  if (cfg->n_tokens > 0 && (!h || !norm_w || !xn || !topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if (!counts) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cfg->n_tokens > 0)
    MOE_TRY(launch_rmsnorm_router(cfg->dtype, h, norm_w, nullptr, xn, nullptr, cfg->n_tokens, cfg->d_model,
                                  cfg->n_experts, cfg->rms_eps, s));
  return launch_hash_route(token_ids, topk_idx, topk_gate, counts, cfg->n_tokens, cfg->n_experts, cfg->top_k, s);
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* xn, int32_t* offsets,
                       int32_t* slot_row, int32_t* row_token, void* x_perm, void* ws, size_t ws_bytes,
                       void* stream) {
  NvtxScope range("moe_permute");
  MOE_TRY(check_common(cfg, ws, ws_bytes));
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (cfg->n_tokens > 0 && (!topk_idx || !xn || !slot_row || !row_token || !x_perm)) return MOE_ERR_INVALID_ARG;
  return permute_impl(cfg, topk_idx, xn, offsets, slot_row, row_token, x_perm, ws, (cudaStream_t)stream);
}

moe_status moe_expert_ffn(const moe_config* cfg, int32_t n_groups, const int32_t* offsets, int32_t max_rows,
                          const void* x, const void* w_gate, const void* w_up, const void* w_down, int32_t d_ff,
                          void* y, void* ws, size_t ws_bytes, void* stream) {
  NvtxScope range("moe_expert_ffn");
  MOE_TRY(check_common(cfg, ws, ws_bytes));
  if (n_groups < 1 || n_groups > 1024 || max_rows < 0 || d_ff < 1) return MOE_ERR_INVALID_ARG;
  if (offsets == nullptr && n_groups != 1) return MOE_ERR_INVALID_ARG;
  if (cfg->dtype == MOE_BF16 && d_ff % 8) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)max_rows * d_ff > layout_of(cfg).act_elems) return MOE_ERR_WORKSPACE;
  if (max_rows > 0 && (!x || !w_gate || !w_up || !w_down || !y)) return MOE_ERR_INVALID_ARG;
  return ffn_impl(cfg, n_groups, offsets, max_rows, x, w_gate, w_up, w_down, d_ff, y, ws, (cudaStream_t)stream);
}

moe_status moe_combine(const moe_config* cfg, const void* h, const void* y_perm, const int32_t* slot_row,
                       const float* topk_gate, const void* y_shared, void* out, void* stream) {
  NvtxScope range("moe_combine");
  if (!config_ok(cfg)) return MOE_ERR_INVALID_ARG;
  if (!config_supported(cfg)) return MOE_ERR_UNSUPPORTED;
  if (cfg->n_tokens > 0 && (!h || !slot_row || !topk_gate || !out)) return MOE_ERR_INVALID_ARG;
  // y_perm may be NULL only when a capacity of 0 drops every slot
  if (cfg->n_tokens > 0 && capacity_of(cfg) != 0 && !y_perm) return MOE_ERR_INVALID_ARG;
  return launch_combine(cfg->dtype, h, y_perm, slot_row, topk_gate, y_shared, out, cfg->n_tokens, cfg->d_model,
                        cfg->top_k, (cudaStream_t)stream);
}

moe_status moe_layer_forward(const moe_config* cfg, const moe_weights* w, const void* h, const float* bias,
                             void* out, const moe_routing* routing, const moe_trace* trace, void* ws,
                             size_t ws_bytes, void* stream) {
  MOE_TRY(check_common(cfg, ws, ws_bytes));
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  const bool shared = cfg->d_ff_shared > 0;
  if (cfg->n_tokens > 0) {
    if (!h || !out || !w->norm_w || !w->w_router || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
    if (shared && (!w->ws_gate || !w->ws_up || !w->ws_down)) return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  const Layout L = layout_of(cfg);
  auto pick = [&](void* user, size_t off) { return user ? user : (void*)wsp(ws, off); };
  void* xn = wsp(ws, L.xn);
  float* scores = routing ? routing->scores : nullptr;
  int32_t* idx = (int32_t*)pick(routing ? routing->topk_idx : nullptr, L.idx);
  float* gate = (float*)pick(routing ? routing->topk_gate : nullptr, L.gate);
  int32_t* counts = (int32_t*)pick(routing ? routing->counts : nullptr, L.counts);
  int32_t* offsets = (int32_t*)pick(routing ? routing->offsets : nullptr, L.offsets);
  int32_t* slot_row = (int32_t*)pick(routing ? routing->slot_row : nullptr, L.slot_row);
  int32_t* row_token = (int32_t*)pick(routing ? routing->row_token : nullptr, L.row_token);
  void* x_perm = wsp(ws, L.x_perm);
  void* y_perm = wsp(ws, L.y_perm);
  void* y_shared = shared ? wsp(ws, L.y_shared) : nullptr;
  NvtxScope call_range("moe_layer_forward");
  NvtxStages stages;
  // records the trace event of a stage boundary and opens the next stage's range
  auto mark = [&](void* ev, const char* next) -> moe_status {
    stages.next(next);
    if (ev && cudaEventRecord((cudaEvent_t)ev, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  };
  MOE_TRY(mark(trace ? trace->start : nullptr, "route"));
  // the counts come from the permute's scan below
  MOE_TRY(route_impl(cfg, h, w->norm_w, w->w_router, bias, xn, scores, idx, gate, nullptr, ws, s));
  MOE_TRY(mark(trace ? trace->routed : nullptr, "permute"));
  const int R = (int)L.rows;
  const int N = cfg->n_tokens;
  void* act = wsp(ws, L.act);
  int32_t* hdr = (int32_t*)wsp(ws, L.hdr);
  if (L.fold) {
    // routed experts 0..E-1 plus the shared expert as group E over all N tokens
    int32_t* offs_ext = (int32_t*)wsp(ws, L.offsets_ext);
    MOE_TRY(launch_permute(idx, N, cfg->top_k, cfg->n_experts, (int)capacity_of(cfg), (int32_t*)wsp(ws, L.hist),
                           offsets, slot_row, row_token, s, offs_ext, N, counts));
    MOE_TRY(launch_gather(cfg->dtype, xn, slot_row, N, cfg->top_k, x_perm, cfg->d_model, s, hdr));
    MOE_TRY(mark(trace ? trace->permuted : nullptr, "gate_up"));
    if (N > 0) {
      MOE_TRY(launch_gemm_tc(EPI_SWIGLU, x_perm, w->w_gate, w->w_up, offs_ext, cfg->n_experts + 1, R + N, cfg->d_ff,
                             cfg->d_model, act, cfg->d_ff, hdr, s, w->ws_gate, w->ws_up, xn, N));
      MOE_TRY(mark(trace ? trace->gate_up : nullptr, "down"));
      MOE_TRY(launch_gemm_tc(EPI_STORE, act, w->w_down, nullptr, offs_ext, cfg->n_experts + 1, R + N, cfg->d_model,
                             cfg->d_ff, y_perm, cfg->d_model, hdr, s, w->ws_down, nullptr));
    } else {
      MOE_TRY(mark(trace ? trace->gate_up : nullptr, "down"));
    }
    MOE_TRY(mark(trace ? trace->down : nullptr, "shared"));
    MOE_TRY(mark(trace ? trace->shared : nullptr, "combine"));  // included in the two launches above
    MOE_TRY(launch_combine(cfg->dtype, h, y_perm, slot_row, gate, nullptr, out, N, cfg->d_model, cfg->top_k, s,
                           offs_ext, cfg->n_experts));
    MOE_TRY(mark(trace ? trace->combined : nullptr, nullptr));
    return MOE_OK;
  }
  MOE_TRY(permute_impl(cfg, idx, xn, offsets, slot_row, row_token, x_perm, ws, s, counts));
  MOE_TRY(mark(trace ? trace->permuted : nullptr, "gate_up"));
  if (R > 0) {
    if (use_tc(cfg)) {
      MOE_TRY(launch_gemm_tc(EPI_SWIGLU, x_perm, w->w_gate, w->w_up, offsets, cfg->n_experts, R, cfg->d_ff,
                             cfg->d_model, act, cfg->d_ff, hdr, s));
      MOE_TRY(mark(trace ? trace->gate_up : nullptr, "down"));
      MOE_TRY(launch_gemm_tc(EPI_STORE, act, w->w_down, nullptr, offsets, cfg->n_experts, R, cfg->d_model,
                             cfg->d_ff, y_perm, cfg->d_model, hdr, s));
    } else {
      MOE_TRY(launch_gemm_simt(cfg->dtype, EPI_SWIGLU, x_perm, w->w_gate, w->w_up, offsets, cfg->n_experts, R,
                               cfg->d_ff, cfg->d_model, act, cfg->d_ff, s));
      MOE_TRY(mark(trace ? trace->gate_up : nullptr, "down"));
      MOE_TRY(launch_gemm_simt(cfg->dtype, EPI_STORE, act, w->w_down, nullptr, offsets, cfg->n_experts, R,
                               cfg->d_model, cfg->d_ff, y_perm, cfg->d_model, s));
    }
  } else {
    MOE_TRY(mark(trace ? trace->gate_up : nullptr, "down"));
  }
  MOE_TRY(mark(trace ? trace->down : nullptr, "shared"));
  if (shared && N > 0)
    MOE_TRY(ffn_impl(cfg, 1, nullptr, N, xn, w->ws_gate, w->ws_up, w->ws_down, cfg->d_ff_shared, y_shared, ws, s));
  MOE_TRY(mark(trace ? trace->shared : nullptr, "combine"));
  MOE_TRY(launch_combine(cfg->dtype, h, y_perm, slot_row, gate, y_shared, out, N, cfg->d_model, cfg->top_k, s));
  MOE_TRY(mark(trace ? trace->combined : nullptr, nullptr));
  return MOE_OK;
}

moe_status moe_bias_update(int32_t n_experts, const int32_t* counts, float target, float gamma, float* bias,
                           void* stream) {
  NvtxScope range("moe_bias_update");
  if (n_experts < 1 || n_experts > 1024 || !counts || !bias) return MOE_ERR_INVALID_ARG;
  return launch_bias_update(n_experts, counts, target, gamma, bias, (cudaStream_t)stream);
}

moe_status moe_compute_load_stats(const moe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                  moe_load_stats* stats, void* stream) {
  NvtxScope range("moe_compute_load_stats");
  if (!config_ok(cfg) || !counts || !offsets || !stats) return MOE_ERR_INVALID_ARG;
  return launch_load_stats(cfg->n_tokens * cfg->top_k, cfg->n_experts, counts, offsets, stats, (cudaStream_t)stream);
}

moe_status moe_check_device_error(void* ws, size_t ws_bytes, void* stream, int32_t* info) {
  if (ws == nullptr || ws_bytes < moe::kHeaderBytes) return MOE_ERR_INVALID_ARG;
  int32_t h[4] = {0, 0, 0, 0};
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (info) {
    for (int i = 0; i < 4; ++i) info[i] = h[i];
  }
  if (h[0] != 0) {
    if (cudaMemsetAsync(ws, 0, moe::kHeaderBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    return (moe_status)h[0];
  }
  return MOE_OK;
}

moe_status moe_set_wait_timeout_ns(int64_t ns) {
  if (ns < 0) return MOE_ERR_INVALID_ARG;
  g_wait_ns.store((uint64_t)ns, std::memory_order_relaxed);
  return MOE_OK;
}

moe_status moe_set_gemm_tiling(int32_t mode) {
  if (mode < 0 || mode > 3) return MOE_ERR_INVALID_ARG;
  set_tc_pairing(mode);
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < moe::kHeaderBytes || ((uintptr_t)ws % 256) != 0) return MOE_ERR_INVALID_ARG;
  return launch_selftest_wait((int32_t*)ws, (cudaStream_t)stream);
}

}  // extern "C"
