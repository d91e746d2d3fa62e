// Steps a1-a3 of the MoE layer: RMSNorm (with the router dot products on
// the CUDA cores when that is the faster place for them), and the router's
// softmax, top-k on score + bias with gates from the raw scores, and counts.
//
// Sources: "Mixture of Experts (MoE)" lesson (AI Engineering from Scratch,
// Phase 07), "The concept / Swapping the FFN" (one norm(h) feeds the router
// and the experts), "Step 1: the router" (selection on scores + bias, gates
// as a softmax over the chosen raw scores, stable sort so the lower index
// wins a tie) and "The load-balancing problem" (DeepSeek-V3: bias changes
// selection only); Ultralytics glossary "Mixture of Experts (MoE)", "How an
// MoE layer works" (outputs weighted by the normalised router scores).
// With many experts and many tokens the router logits come from the tcgen05
// grouped GEMM instead.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// a1 (+ a2 on the CUDA cores). RMSNorm: xn = h / sqrt(mean(h^2) + eps) * w.
// mean(h^2) is summed in fp64 (every h^2 is exact there); the scale
// r = fl32(1 / sqrt(ms + eps)) is taken in fp64 and rounded once, then
// xn = round(fl32(fl32(h * r) * w)), so the storage rounding is decided in fp32.
//
// One block per token (grid-stride), V elements per 16-byte access.  The
// row is staged in shared memory in its own dtype; when `logits` is given, the
// block's warps then take the router dot products of the rounded xn row
// with experts [e0, e0 + epb) (e0 = blockIdx.y * epb), one expert per warp
// at a time, fp32 FMA per lane (dot_accum) and a warp tree sum.  Blocks with
// blockIdx.y == 0 write xn.
// ---------------------------------------------------------------------------
template <typename T, int V>
struct Vec {
  static_assert(V * sizeof(T) == 16 || V == 1, "V elements must fill 16 bytes");
  T v[V];
};

template <typename T, int V>
__device__ __forceinline__ void vec_to_f32(const Vec<T, V>& x, float (&f)[V]) {
#pragma unroll
  for (int j = 0; j < V; ++j) f[j] = to_f32(x.v[j]);
}

template <typename T, int V>
__device__ __forceinline__ Vec<T, V> ld_vec(const T* p) {
  Vec<T, V> x;
  if (V * sizeof(T) == 16) *reinterpret_cast<uint4*>(&x) = *reinterpret_cast<const uint4*>(p);
  else x.v[0] = p[0];
  return x;
}

template <typename T, int V>
__device__ __forceinline__ void st_vec(T* p, const Vec<T, V>& x) {
  if (V * sizeof(T) == 16) *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(&x);
  else p[0] = x.v[0];
}

// s += x[j] * w[j] for j = 0 .. V-1 in order, each an fp32 FMA with one
// rounding.  A bf16 value widens to fp32 exactly, so the bf16 form below (the
// sm_100 FMA that takes bf16 sources and an fp32 addend and result) gives the
// same bits as widening both operands first, without the conversions that
// otherwise take most of the router's issue slots.
template <typename T, int V>
__device__ __forceinline__ float dot_accum(const T* x, const T* w, float s) {
  float xf[V], wf[V];
  vec_to_f32(ld_vec<T, V>(x), xf);
  vec_to_f32(ld_vec<T, V>(w), wf);
#pragma unroll
  for (int j = 0; j < V; ++j) s = __fmaf_rn(xf[j], wf[j], s);
  return s;
}

__device__ __forceinline__ float fma_bf16x2(uint32_t a, uint32_t b, float c) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(c)
      : "r"(a), "r"(b));
  return c;
}

template <>
__device__ __forceinline__ float dot_accum<bf16, 8>(const bf16* x, const bf16* w, float s) {
  const uint4 a = *reinterpret_cast<const uint4*>(x);
  const uint4 b = *reinterpret_cast<const uint4*>(w);
  s = fma_bf16x2(a.x, b.x, s);
  s = fma_bf16x2(a.y, b.y, s);
  s = fma_bf16x2(a.z, b.z, s);
  s = fma_bf16x2(a.w, b.w, s);
  return s;
}

template <typename T, int V>
__global__ void __launch_bounds__(256) rmsnorm_router_kernel(const T* __restrict__ h, const T* __restrict__ w,
                                                             const T* __restrict__ w_router, T* __restrict__ xn,
                                                             float* __restrict__ logits, int n, int d, int E,
                                                             int epb, float eps) {
  extern __shared__ __align__(16) uint8_t row_raw[];  // one row of d elements of T
  T* row = reinterpret_cast<T*>(row_raw);
  __shared__ double part[8];
  __shared__ float r_sh;
  const int e0 = blockIdx.y * epb;
  const int e1 = min(E, e0 + epb);
  const int warps = blockDim.x >> 5;
  const int step = blockDim.x * V;  // elements per pass of the block
  for (int t = blockIdx.x; t < n; t += gridDim.x) {
    const T* hr = h + (size_t)t * d;
    double acc = 0.0;
    for (int i = threadIdx.x * V; i < d; i += step) {
      const Vec<T, V> x = ld_vec<T, V>(hr + i);
      float f[V];
      vec_to_f32(x, f);
#pragma unroll
      for (int j = 0; j < V; ++j) acc += (double)f[j] * (double)f[j];
      st_vec<T, V>(row + i, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane_id() == 0) part[warp_id()] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double s = 0.0;
      for (int i = 0; i < warps; ++i) s += part[i];
      r_sh = (float)(1.0 / sqrt(s / (double)d + (double)eps));
    }
    __syncthreads();
    const float r = r_sh;
    const bool store = (blockIdx.y == 0) && xn != nullptr;
    for (int i = threadIdx.x * V; i < d; i += step) {
      float f[V], wf[V];
      vec_to_f32(ld_vec<T, V>(row + i), f);
      vec_to_f32(ld_vec<T, V>(w + i), wf);
      Vec<T, V> q;
#pragma unroll
      for (int j = 0; j < V; ++j) q.v[j] = from_f32<T>(__fmul_rn(__fmul_rn(f[j], r), wf[j]));
      st_vec<T, V>(row + i, q);
      if (store) st_vec<T, V>(xn + (size_t)t * d + i, q);
    }
    __syncthreads();
    if (logits != nullptr) {
      for (int e = e0 + warp_id(); e < e1; e += warps) {
        const T* wr = w_router + (size_t)e * d;
        float s = 0.f;
        for (int i = lane_id() * V; i < d; i += 32 * V) s = dot_accum<T, V>(row + i, wr + i, s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane_id() == 0) logits[(size_t)t * E + e] = s;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// a3. One warp per token.  Lane l holds experts l, l + 32, ... (EPL of them).
//   score = softmax(logits) in fp32; key = fl32(score + bias);
//   k rounds of a warp arg-max on key (equal keys: lower expert wins), each a
//   lane-local scan and two warp reductions (largest key, then lowest expert
//   holding it);
//   gate_j = score_j / sum of the chosen scores.
// counts: per-block shared histogram, added to the global one at the end
// (skipped when counts is null).
// ---------------------------------------------------------------------------
// Unsigned image of a float that orders as the float does (-0 taken as +0,
// so equal keys map to equal images).
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t u = __float_as_uint(__fadd_rn(x, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int EPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, float* __restrict__ scores,
                                                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                                                   int32_t* __restrict__ counts, int n, int E, int k) {
  extern __shared__ int32_t hist[];
  if (counts != nullptr) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
  }
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
      // this lane's best free expert (strict >: the lowest i, i.e. the lowest
      // expert, among equal keys) ...
      float bk = -INFINITY;
      int bi = -1;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const bool free_ = !((taken >> i) & 1u) && lane + 32 * i < E;
        if (free_ && (bi < 0 || key[i] > bk)) {
          bk = key[i];
          bi = i;
        }
      }
      // ... then the warp's largest key, and the lowest expert holding it
      const uint32_t mk = bi >= 0 ? ordered_bits(bk) : 0u;
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, mk);
      const uint32_t be = __reduce_min_sync(0xffffffffu, (bi >= 0 && mk == kmax) ? (uint32_t)(lane + 32 * bi)
                                                                                   : 0xffffffffu);
      const int wi = (int)(be >> 5);
      float mine = v[0];
#pragma unroll
      for (int i = 1; i < EPL; ++i)
        if (wi == i) mine = v[i];
      const float bs = __shfl_sync(0xffffffffu, mine, (int)(be & 31u));  // the winner's score
      if ((int)(be & 31u) == lane) taken |= 1u << wi;
      chosen_sum = __fadd_rn(chosen_sum, bs);
      if (lane == j) {
        my_score = bs;
        my_idx = (int)be;
      }
    }
    if (lane < k) {
      topk_idx[(size_t)t * k + lane] = my_idx;
      topk_gate[(size_t)t * k + lane] = __fdiv_rn(my_score, chosen_sum);
      if (counts != nullptr) atomicAdd(&hist[my_idx], 1);
    }
  }
  if (counts == nullptr) return;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

// ---------------------------------------------------------------------------
// Hash router ("Mixture of Experts (MoE)" lesson, "Exercises": route tokens
// with a hash instead of a learned router).  Choice j of a token with id x is
// (h(x) + j) mod E, h the SplitMix64 output function (Steele, Lea and Flood,
// "Fast splittable pseudorandom number generators", 2014); every gate 1/k.
// One thread per token; counts through a per-block shared histogram.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t splitmix64_mix(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void __launch_bounds__(256) hash_route_kernel(const int64_t* __restrict__ token_ids, int n, int E, int k,
                                                         int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                                                         int32_t* __restrict__ counts) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const float g = __fdiv_rn(1.f, (float)k);
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
    const uint64_t id = token_ids ? (uint64_t)token_ids[t] : (uint64_t)t;
    const int e0 = (int)(splitmix64_mix(id) % (uint64_t)E);
    for (int j = 0; j < k; ++j) {
      int e = e0 + j;
      if (e >= E) e -= E;
      topk_idx[(size_t)t * k + j] = e;
      topk_gate[(size_t)t * k + j] = g;
      atomicAdd(&hist[e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

}  // namespace moe

namespace moe_host {

moe_status launch_hash_route(const int64_t* token_ids, int32_t* topk_idx, float* topk_gate, int32_t* counts, int n,
                             int e, int k, cudaStream_t s) {
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * e, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (n == 0) return MOE_OK;
  int blocks = (n + 255) / 256;
  if (blocks > sm_count() * 4) blocks = sm_count() * 4;
  moe::hash_route_kernel<<<blocks, 256, sizeof(int32_t) * e, s>>>(token_ids, n, e, k, topk_idx, topk_gate, counts);
  return launch_status();
}


template <typename T, int V>
static moe_status launch_rr(const void* h, const void* norm_w, const void* w_router, void* xn, float* logits, int n,
                            int d, int e, float eps, cudaStream_t s) {
  const size_t smem = sizeof(T) * (size_t)d;
  auto kern = moe::rmsnorm_router_kernel<T, V>;
  if (smem > 48 * 1024) {
    static SmemLimit lim;
    const moe_status st = ensure_smem_limit(kern, (int)smem, lim);
    if (st != MOE_OK) return st;
  }
  const int epb = (logits == nullptr) ? 1 : (e <= 32 ? e : 32);
  const int yb = (logits == nullptr) ? 1 : (e + epb - 1) / epb;
  // RMSNorm alone: 128-thread blocks, so twice as many tokens are in flight per SM
  const int threads = logits == nullptr ? 128 : 256;
  int xb = n < sm_count() * 16 ? n : sm_count() * 16;
  kern<<<dim3(xb, yb), threads, smem, s>>>((const T*)h, (const T*)norm_w, (const T*)w_router, (T*)xn, logits, n, d, e,
                                       epb, eps);
  return launch_status();
}

moe_status launch_rmsnorm_router(int dtype, const void* h, const void* norm_w, const void* w_router, void* xn,
                                 float* logits, int n, int d, int e, float eps, cudaStream_t s) {
  if (n == 0) return MOE_OK;
  const uintptr_t addr = (uintptr_t)h | (uintptr_t)norm_w | (uintptr_t)xn | (uintptr_t)(w_router ? w_router : h);
  if (dtype == MOE_BF16) {
    if (d % 8 == 0 && addr % 16 == 0) return launch_rr<moe::bf16, 8>(h, norm_w, w_router, xn, logits, n, d, e, eps, s);
    return launch_rr<moe::bf16, 1>(h, norm_w, w_router, xn, logits, n, d, e, eps, s);
  }
  if (d % 4 == 0 && addr % 16 == 0) return launch_rr<float, 4>(h, norm_w, w_router, xn, logits, n, d, e, eps, s);
  return launch_rr<float, 1>(h, norm_w, w_router, xn, logits, n, d, e, eps, s);
}

moe_status launch_topk(const float* logits, const float* bias, float* scores, int32_t* topk_idx,
                       float* topk_gate, int32_t* counts, int n, int e, int k, cudaStream_t s) {
  if (counts != nullptr && cudaMemsetAsync(counts, 0, sizeof(int32_t) * e, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (n == 0) return MOE_OK;
  const int warps = 8;
  int blocks = (n + warps - 1) / warps;
  if (blocks > sm_count() * 8) blocks = sm_count() * 8;
  size_t smem = counts != nullptr ? sizeof(int32_t) * e : 0;
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
