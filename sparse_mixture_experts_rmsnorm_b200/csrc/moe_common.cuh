// Shared device helpers of the MoE-layer forward library (sm_100a only).
//
// Holds: the element-type helpers, the workspace header that carries the
// device error word, the bounded mbarrier wait used by every pipelined
// kernel, and the launch plumbing (SM count, error mapping) of the host side.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace moe {

// ---------------------------------------------------------------------------
// Element types
// ---------------------------------------------------------------------------
typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
// Round to nearest even, as the storage rounding of every quantisation point.
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// Workspace header: the first 256 bytes of every workspace.
//   word 0: status (0 = ok, else a moe_status), word 1: kernel id,
//   word 2: block index, word 3: wait site.  The first failure wins.
// ---------------------------------------------------------------------------
constexpr size_t kHeaderBytes = 256;

enum KernelId : int32_t {
  KID_GEMM_TC = 1,
  KID_SELFTEST = 2,
  KID_SCATTER = 3,
};

__device__ __forceinline__ void record_error(int32_t* hdr, int32_t status, int32_t kernel, int32_t block,
                                             int32_t site) {
  if (hdr == nullptr) return;
  if (atomicCAS(hdr, 0, status) == 0) {
    hdr[1] = kernel;
    hdr[2] = block;
    hdr[3] = site;
    __threadfence();
  }
}

// ---------------------------------------------------------------------------
// mbarrier primitives (shared::cta) and the bounded wait
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait until the phase of `bar` with the given parity has completed, for at
// most `limit_ns` nanoseconds (the clock starts at the first failed poll).
// Returns false on time-out after recording MOE_ERR_DEVICE_TIMEOUT, or at
// once when `*abort` is already set by another role of the same block.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                  volatile int* abort, int32_t* hdr, int32_t kernel,
                                                  int32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t polls = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++polls & 63u) == 0u) {
      if (abort != nullptr && *abort) return false;
      if (global_timer_ns() - t0 >= limit_ns) {
        record_error(hdr, MOE_ERR_DEVICE_TIMEOUT, kernel, blockIdx.x, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

}  // namespace moe

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
namespace moe_host {

int sm_count();                       // SMs of the current device (cached per device)
int current_device();
uint64_t wait_limit_ns();             // limit of every bounded device wait

inline moe_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Grid of the row-wise kernels (one 128-thread block per token, grid-stride):
// up to 16 blocks per SM over the tokens and, when there are fewer tokens
// than two blocks per SM, each row split into column ranges (at least one
// 128-thread pass of `vec` elements each) across gridDim.y.
inline dim3 row_split_grid(int n, int d, int vec) {
  const int sms = sm_count();
  const int x = n < sms * 16 ? n : sms * 16;
  const int passes = (d + 128 * vec - 1) / (128 * vec);
  const int want = (2 * sms + x - 1) / x;
  const int y = passes < want ? passes : want;
  return dim3((unsigned)x, (unsigned)(y > 1 ? y : 1));
}

// Dynamic shared-memory limit already granted to one kernel, per device (up to 64 devices; others set it on every
// call). The atomic keeps the common path lock-free; the mutex serialises the attribute calls, so the recorded
// value is always one that was actually set and concurrent first calls from several host threads are safe.
struct SmemLimit {
  std::atomic<int> bytes[64] = {};
  std::mutex mu;
};

// Raises `kernel`'s dynamic shared-memory limit on the current device to at least `need` bytes.
template <typename K>
inline moe_status ensure_smem_limit(K* kernel, int need, SmemLimit& lim) {
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && lim.bytes[dev].load(std::memory_order_acquire) >= need) return MOE_OK;
  std::lock_guard<std::mutex> g(lim.mu);
  if (dev >= 0 && dev < 64 && lim.bytes[dev].load(std::memory_order_relaxed) >= need) return MOE_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, need) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (dev >= 0 && dev < 64) lim.bytes[dev].store(need, std::memory_order_release);
  return MOE_OK;
}

}  // namespace moe_host
