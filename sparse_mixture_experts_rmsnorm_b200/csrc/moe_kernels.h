// Host-side launchers of the library's kernels.  Each enqueues work on
// `stream` and returns cudaGetLastError() mapped to a moe_status; none
// allocates or synchronises.  Argument checking happens in moe_api.cu.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe_host {

// NVTX ranges on the host thread that enqueues the launches: one per entry
// point and, inside moe_layer_forward, one per stage, so that a profiler
// collecting NVTX attributes each kernel launch to its step.  Without such a
// tool attached every NVTX call returns at once.
struct NvtxScope {
  explicit NvtxScope(const char* name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
  NvtxScope(const NvtxScope&) = delete;
  NvtxScope& operator=(const NvtxScope&) = delete;
};

struct NvtxStages {
  bool open = false;
  void next(const char* stage) {
    if (open) nvtxRangePop();
    open = stage != nullptr;
    if (open) nvtxRangePushA(stage);
  }
  ~NvtxStages() { next(nullptr); }
};

// Config checks and the capacity rule shared by the entry points (moe_api.cu).
bool config_ok(const moe_config* c);          // sizes and dtype valid
bool config_supported(const moe_config* c);   // covered by the kernels
int64_t capacity_of(const moe_config* c);     // floor(C*N*k/E), or -1 without a capacity

// a1: xn = RMSNorm(h), and with logits != nullptr also a2 on the CUDA
// cores: logits [N][E] fp32 = xn . W_router^T (one block per token and
// group of up to 32 experts).  One row of shared memory per block.
moe_status launch_rmsnorm_router(int dtype, const void* h, const void* norm_w, const void* w_router, void* xn,
                                 float* logits, int n, int d, int e, float eps, cudaStream_t s);

// a3: softmax over the router logits, top-k on score + bias, renormalised
// gates and the per-expert counts (counts are zeroed here first; with
// counts == nullptr none are taken).
moe_status launch_topk(const float* logits, const float* bias, float* scores, int32_t* topk_idx,
                       float* topk_gate, int32_t* counts, int n, int e, int k, cudaStream_t s);

// Hash router: choice j of token t is (splitmix64(id) + j) mod E, id =
// token_ids[t] (or t when token_ids is null), gates 1/k; counts zeroed first.
moe_status launch_hash_route(const int64_t* token_ids, int32_t* topk_idx, float* topk_gate, int32_t* counts, int n,
                             int e, int k, cudaStream_t s);

// a4: stable counting sort of the N*k slots by expert with optional capacity.
//   hist: workspace of permute_hist_ints(n*k, e) int32.
//   offsets_ext != nullptr: also writes offsets_ext[0..E] = offsets and
//   offsets_ext[E+1] = offsets[E] + extra (a trailing group of `extra` rows).
//   counts != nullptr: also writes the per-expert slot counts (before the
//   capacity cut), the `counts` that launch_topk would give.
size_t permute_hist_ints(int64_t slots, int e);
moe_status launch_permute(const int32_t* topk_idx, int n, int k, int e, int cap, int32_t* hist,
                          int32_t* offsets, int32_t* slot_row, int32_t* row_token, cudaStream_t s,
                          int32_t* offsets_ext = nullptr, int extra = 0, int32_t* counts = nullptr);

// a5: x_perm[slot_row[t * k + j]] = xn[t] for every kept slot (that is,
// x_perm[r] = xn[row_token[r]] for r < R = offsets[e], a device count).
// Token order: each xn row is read once.  k <= 32.  hdr: the workspace's
// error word for the bounded waits of the bulk-copy form (may be null).
moe_status launch_gather(int dtype, const void* xn, const int32_t* slot_row, int n, int k, void* x_perm, int d,
                         cudaStream_t s, int32_t* hdr = nullptr);

// a9: out = h + sum_j gate_j * y_perm[slot_row] (+ y_shared).  With
// shared_offsets != nullptr the shared rows are y_perm rows from
// shared_offsets[e] on (the folded shared expert) and y_shared is ignored.
moe_status launch_combine(int dtype, const void* h, const void* y_perm, const int32_t* slot_row,
                          const float* topk_gate, const void* y_shared, void* out, int n, int d, int k,
                          cudaStream_t s, const int32_t* shared_offsets = nullptr, int e = 0);

// a10: bias[e] += gamma * sign(target - counts[e]).
moe_status launch_bias_update(int e, const int32_t* counts, float target, float gamma, float* bias,
                              cudaStream_t s);

// a4 / a10: load statistics of one routing of `slots` = N*k slots (one block).
moe_status launch_load_stats(int slots, int e, const int32_t* counts, const int32_t* offsets, moe_load_stats* stats,
                             cudaStream_t s);

// Grouped GEMM epilogues.
enum GemmEpilogue { EPI_F32 = 0, EPI_SWIGLU = 1, EPI_STORE = 2 };

// Grouped GEMM on CUDA cores (fp32 or bf16 operands, fp32 accumulation):
//   rows [off[g], off[g+1]) of A [max_rows][k] times B_g^T, B_g = B + g*nout*k ([nout][k]).
//   EPI_SWIGLU: C = silu(A B_g^T) * (A B2_g^T) in the act dtype;
//   EPI_STORE: C = A B_g^T in the act dtype; EPI_F32: C = A B_g^T in fp32.
//   offsets == nullptr: one group of max_rows rows.  ldc = row stride of C.
moe_status launch_gemm_simt(int dtype, int epi, const void* a, const void* b, const void* b2,
                            const int32_t* offsets, int groups, int max_rows, int nout, int k, void* c,
                            int ldc, cudaStream_t s);

// The same grouped GEMM on the tcgen05 tensor cores (bf16 operands only,
// TMA-fed, TMEM accumulators, persistent over the SMs).  k % 8 == 0.
//   hdr: workspace header that receives a device time-out, if any.
//   sb, sb2 != nullptr: the last group is the shared expert, with its own
//   [nout][k] weights sb (gate or down) and sb2 (up).
//   sa != nullptr (with sb): that group's A rows are sa [sa_rows][k] instead
//   of rows offsets[G-1].. of a.
moe_status launch_gemm_tc(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                          int groups, int max_rows, int nout, int k, void* c, int ldc, int32_t* hdr, cudaStream_t s,
                          const void* sb = nullptr, const void* sb2 = nullptr, const void* sa = nullptr,
                          int sa_rows = 0);

// A block that waits, with the bounded wait of the pipelined kernels, on a
// barrier that nothing completes.
moe_status launch_selftest_wait(int32_t* hdr, cudaStream_t s);

}  // namespace moe_host
