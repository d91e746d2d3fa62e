// Steps a1 and a3 of the MoE layer: RMSNorm, and the router's softmax,
// top-k on score + bias with gates from the raw scores, and expert counts.
//
// Sources: "Mixture of Experts (MoE)" lesson (AI Engineering from Scratch,
// Phase 07), "The concept / Swapping the FFN" (one norm(h) feeds the router
// and the experts), "Step 1: the router" (selection on scores + bias, gates
// as a softmax over the chosen raw scores, stable sort so the lower index
// wins a tie) and "The load-balancing problem" (DeepSeek-V3: bias changes
// selection only); Ultralytics glossary "Mixture of Experts (MoE)", "How an
// MoE layer works" (outputs weighted by the normalised router scores).
// The router logits themselves come from the grouped GEMM kernels.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// a1. RMSNorm: xn = h / sqrt(mean(h^2) + eps) * w.
// mean(h^2) is summed in fp64 (every h^2 is exact there); the scale
// r = fl32(1 / sqrt(ms + eps)) is taken in fp64 and rounded once, then
// xn = round(fl32(fl32(h * r) * w)), so the storage rounding is decided in fp32.
// One block per token, grid-stride over tokens.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T* __restrict__ h, const T* __restrict__ w,
                                                      T* __restrict__ xn, int n, int d, float eps) {
  __shared__ double part[8];
  __shared__ float r_sh;
  for (int t = blockIdx.x; t < n; t += gridDim.x) {
    const T* row = h + (size_t)t * d;
    double acc = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      double v = (double)to_f32(row[i]);
      acc += v * v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane_id() == 0) part[warp_id()] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double s = 0.0;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += part[i];
      double ms = s / (double)d;
      r_sh = (float)(1.0 / sqrt(ms + (double)eps));
    }
    __syncthreads();
    const float r = r_sh;
    T* out = xn + (size_t)t * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      float v = __fmul_rn(__fmul_rn(to_f32(row[i]), r), to_f32(w[i]));
      out[i] = from_f32<T>(v);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// a3. One warp per token.  Lane l holds experts l, l + 32, ... (EPL of them).
//   score = softmax(logits) in fp32; key = fl32(score + bias);
//   k rounds of a warp arg-max on key (equal keys: lower expert wins);
//   gate_j = score_j / sum of the chosen scores.
// counts: per-block shared histogram, added to the global one at the end.
// ---------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, float* __restrict__ scores,
                                                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                                                   int32_t* __restrict__ counts, int n, int E, int k) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int lane = lane_id();
  const int warps = blockDim.x >> 5;
  for (int t = blockIdx.x * warps + warp_id(); t < n; t += gridDim.x * warps) {
    const float* lrow = logits + (size_t)t * E;
    float v[EPL];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      int e = lane + 32 * i;
      v[i] = (e < E) ? lrow[e] : -INFINITY;
      m = fmaxf(m, v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      int e = lane + 32 * i;
      v[i] = (e < E) ? expf(v[i] - m) : 0.f;
      s += v[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    float key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      int e = lane + 32 * i;
      v[i] = __fdiv_rn(v[i], s);  // score
      key[i] = (e < E) ? __fadd_rn(v[i], bias ? bias[e] : 0.f) : -INFINITY;
      if (scores && e < E) scores[(size_t)t * E + e] = v[i];
    }
    uint32_t taken = 0;  // bit i: expert lane + 32 i already chosen
    float chosen_sum = 0.f;
    float my_score = 0.f;  // lane j < k keeps the score of the j-th choice
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
      float bk = -INFINITY;
      int be = 0x7fffffff;
      float bs = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        int e = lane + 32 * i;
        bool free_ = !((taken >> i) & 1u) && e < E;
        if (free_ && (key[i] > bk || (key[i] == bk && e < be))) {
          bk = key[i];
          be = e;
          bs = v[i];
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        float ok = __shfl_xor_sync(0xffffffffu, bk, o);
        int oe = __shfl_xor_sync(0xffffffffu, be, o);
        float os = __shfl_xor_sync(0xffffffffu, bs, o);
        if (ok > bk || (ok == bk && oe < be)) {
          bk = ok;
          be = oe;
          bs = os;
        }
      }
      // every lane now holds the winner (be, bs)
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      chosen_sum = __fadd_rn(chosen_sum, bs);
      if (lane == j) {
        my_score = bs;
        my_idx = be;
      }
    }
    if (lane < k) {
      topk_idx[(size_t)t * k + lane] = my_idx;
      topk_gate[(size_t)t * k + lane] = __fdiv_rn(my_score, chosen_sum);
      atomicAdd(&hist[my_idx], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

}  // namespace moe

namespace moe_host {

moe_status launch_rmsnorm(int dtype, const void* h, const void* norm_w, void* xn, int n, int d, float eps,
                          cudaStream_t s) {
  if (n == 0) return MOE_OK;
  int grid = n < sm_count() * 16 ? n : sm_count() * 16;
  if (dtype == MOE_BF16)
    moe::rmsnorm_kernel<moe::bf16><<<grid, 256, 0, s>>>((const moe::bf16*)h, (const moe::bf16*)norm_w,
                                                        (moe::bf16*)xn, n, d, eps);
  else
    moe::rmsnorm_kernel<float><<<grid, 256, 0, s>>>((const float*)h, (const float*)norm_w, (float*)xn, n, d,
                                                    eps);
  return launch_status();
}

moe_status launch_topk(const float* logits, const float* bias, float* scores, int32_t* topk_idx,
                       float* topk_gate, int32_t* counts, int n, int e, int k, cudaStream_t s) {
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * e, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (n == 0) return MOE_OK;
  const int warps = 8;
  int blocks = (n + warps - 1) / warps;
  if (blocks > sm_count() * 8) blocks = sm_count() * 8;
  size_t smem = sizeof(int32_t) * e;
  int epl = (e + 31) / 32;
#define MOE_TOPK(EPL) \
  moe::topk_kernel<EPL><<<blocks, warps * 32, smem, s>>>(logits, bias, scores, topk_idx, topk_gate, counts, n, e, k)
  if (epl <= 1) MOE_TOPK(1);
  else if (epl <= 2) MOE_TOPK(2);
  else if (epl <= 4) MOE_TOPK(4);
  else if (epl <= 8) MOE_TOPK(8);
  else if (epl <= 16) MOE_TOPK(16);
  else MOE_TOPK(32);
#undef MOE_TOPK
  return launch_status();
}

}  // namespace moe_host
