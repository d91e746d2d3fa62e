// moe_permute_noalloc: the counting-sort permute (steps a4-a5) without a
// caller-provided workspace.
//
// Some callers cannot give the library device memory for scratch. Two examples:
//  - code that only receives its input and output buffers, such as a plugin
//    or callback inside another framework that owns every device allocation;
//  - code that must not allocate once it is running, such as a latency-bound
//    serving loop, because cudaMalloc can synchronise the device and take an
//    unbounded time.
// This entry point keeps the permute's only scratch, the per-chunk expert
// histograms, in a fixed device array of this library.  The array is sized
// for DeepSeek-V3-scale routing: 262144 int32 = 1 MiB.
//
// The caller still passes every input and output.  The array is a
// file-scope __device__ variable, so every GPU that loads the library holds
// its 1 MiB until the process exits.
//
// In host code the name `g_perm_hist` does not hold a device address; it is
// a host-side stand-in.  A kernel given that name faults, or, where the GPU
// can reach host memory, silently uses the wrong memory.  The device address
// is therefore looked up once per device with cudaGetSymbolAddress, on the
// first call made with that device current, and passed to the kernels.
#include <mutex>

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace {

constexpr size_t kNoAllocHistInts = MOE_NOALLOC_HIST_INTS;

// Shared by every call on a device; the contents of the last call remain.
static __device__ __align__(256) int32_t g_perm_hist[kNoAllocHistInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_hist_ptr[kMaxDevices] = {};

// Device address of g_perm_hist for the current device (set-up on first use).
// The address is cached per device ordinal for the life of the process: it
// belongs to the device's primary context, the one the runtime API uses.  A
// cudaDeviceReset, or a caller that makes another driver-API context
// current, would need the lookup again; neither is supported by this call.
// A failed lookup clears the runtime's error state, so the failure is
// reported once, by this call, and not again by the next launch check.
moe_status hist_address(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_hist_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_perm_hist) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_hist_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_hist_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx, const void* xn,
                                          int32_t* offsets, int32_t* slot_row, int32_t* row_token, void* x_perm,
                                          void* stream) {
  using namespace moe_host;
  NvtxScope range("moe_permute_noalloc");
  if (!config_ok(cfg)) return MOE_ERR_INVALID_ARG;
  if (!config_supported(cfg)) return MOE_ERR_UNSUPPORTED;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (cfg->n_tokens > 0 && (!topk_idx || !xn || !slot_row || !row_token || !x_perm)) return MOE_ERR_INVALID_ARG;
  const int64_t slots = (int64_t)cfg->n_tokens * cfg->top_k;
  // Every histogram entry that the kernels read is written earlier in the
  // same call, so nothing needs clearing between calls.
  if (permute_hist_ints(slots, cfg->n_experts) > kNoAllocHistInts) return MOE_ERR_WORKSPACE;
  int32_t* hist = nullptr;
  moe_status st = hist_address(&hist);
  if (st != MOE_OK) return st;
  const int64_t cap = capacity_of(cfg);
  cudaStream_t s = (cudaStream_t)stream;
  st = launch_permute(topk_idx, cfg->n_tokens, cfg->top_k, cfg->n_experts, (int)cap, hist, offsets, slot_row,
                      row_token, s);
  if (st != MOE_OK) return st;
  return launch_gather(cfg->dtype, xn, slot_row, cfg->n_tokens, cfg->top_k, x_perm, cfg->d_model, s);
}
