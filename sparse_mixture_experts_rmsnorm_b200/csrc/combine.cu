// Steps a9 and a10 of the MoE layer: the gated combine fused with the
// residual add, and the auxiliary-loss-free bias update.
//
// Sources: "Mixture of Experts (MoE)" lesson (AI Engineering from Scratch,
// Phase 07), "The concept / Swapping the FFN" (h = h + sum over the chosen
// experts of gate * Expert(norm(h))), "Shared experts" (every token also
// passes the shared expert), "The load-balancing problem" and "Step 2"
// (after each step every expert's bias moves by -gamma when it was used above
// the target and by +gamma when below); Ultralytics glossary "Mixture of
// Experts (MoE)" example (out[token] += weight * expert(token)) and "Load
// balancing and expert capacity" (a dropped token continues on the residual).
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

// Gather form: each output element reads its token's k expert rows, so no
// atomics are needed and the sum order is fixed:
//   acc = h; acc = fma(gate_j, y_j, acc) for kept j in rank order; acc += y_shared;
//   out = round(acc).
// A token whose slots are all dropped (and no shared expert) returns h exactly.
// VEC consecutive elements per thread (VEC * sizeof(T) = 16 bytes when aligned).
// Block (x, y) takes tokens x, x + gridDim.x, ... and the y-th of gridDim.y
// column ranges of each row (a multiple of VEC wide), so that few tokens
// still fill the GPU.
__device__ __forceinline__ void column_range(int d, int vec, int& cb, int& ce) {
  const int parts = (int)gridDim.y;
  int w = (d + parts - 1) / parts;
  w = (w + vec - 1) / vec * vec;
  cb = min(d, (int)blockIdx.y * w);
  ce = min(d, cb + w);
}

template <typename T, int VEC, int KC>
__global__ void __launch_bounds__(128) combine_kernel(const T* __restrict__ h, const T* __restrict__ y_perm,
                                                      const int32_t* __restrict__ slot_row,
                                                      const float* __restrict__ gates,
                                                      const T* __restrict__ y_shared, T* out, int n, int d,
                                                      int k, const int32_t* __restrict__ shared_offsets, int E) {
  __shared__ int32_t rows[32];
  // the folded shared expert: its rows follow the routed rows of y_perm
  if (shared_offsets != nullptr) y_shared = y_perm + (size_t)shared_offsets[E] * d;
  __shared__ float g[32];
  int cb, ce;
  column_range(d, VEC, cb, ce);
  for (int t = blockIdx.x; t < n; t += gridDim.x) {
    if (threadIdx.x < k) {
      rows[threadIdx.x] = slot_row[(size_t)t * k + threadIdx.x];
      g[threadIdx.x] = gates[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    for (int c = cb + threadIdx.x * VEC; c < ce; c += blockDim.x * VEC) {
      float acc[VEC];
      T tmp[VEC];
      const size_t off = (size_t)t * d + c;
      if (VEC > 1) {
        *reinterpret_cast<uint4*>(tmp) = *reinterpret_cast<const uint4*>(h + off);
      } else {
        tmp[0] = h[off];
      }
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = to_f32(tmp[i]);
      // up to KC slot rows in flight per thread, summed in rank order
      for (int j0 = 0; j0 < k; j0 += KC) {
        T yv[KC][VEC];
#pragma unroll
        for (int jj = 0; jj < KC; ++jj) {
          const int j = j0 + jj;
          if (j < k && rows[j] >= 0) {
            const T* yr = y_perm + (size_t)rows[j] * d + c;
            if (VEC > 1) *reinterpret_cast<uint4*>(yv[jj]) = *reinterpret_cast<const uint4*>(yr);
            else yv[jj][0] = yr[0];
          }
        }
#pragma unroll
        for (int jj = 0; jj < KC; ++jj) {
          const int j = j0 + jj;
          if (j < k && rows[j] >= 0) {
            const float gj = g[j];
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc[i] = __fmaf_rn(gj, to_f32(yv[jj][i]), acc[i]);
          }
        }
      }
      if (y_shared != nullptr) {
        if (VEC > 1) {
          *reinterpret_cast<uint4*>(tmp) = *reinterpret_cast<const uint4*>(y_shared + off);
        } else {
          tmp[0] = y_shared[off];
        }
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], to_f32(tmp[i]));
      }
#pragma unroll
      for (int i = 0; i < VEC; ++i) tmp[i] = from_f32<T>(acc[i]);
      if (VEC > 1) {
        *reinterpret_cast<uint4*>(out + off) = *reinterpret_cast<const uint4*>(tmp);
      } else {
        out[off] = tmp[0];
      }
    }
    __syncthreads();
  }
}

// The same combine for small k, CU column blocks per thread per pass: all
// their h and y loads are issued before any block is combined and stored, so
// a thread has CU times the loads in flight (the blocks are disjoint, so this
// holds when out == h too).  Same arithmetic, in the same order, per element.
template <typename T, int VEC, int KC, int CU>
__global__ void __launch_bounds__(128) combine_cols_kernel(const T* __restrict__ h, const T* __restrict__ y_perm,
                                                      const int32_t* __restrict__ slot_row,
                                                      const float* __restrict__ gates,
                                                      const T* __restrict__ y_shared, T* out, int n, int d,
                                                      int k, const int32_t* __restrict__ shared_offsets, int E) {
  __shared__ int32_t rows[32];
  // the folded shared expert: its rows follow the routed rows of y_perm
  if (shared_offsets != nullptr) y_shared = y_perm + (size_t)shared_offsets[E] * d;
  __shared__ float g[32];
  const int cstep = blockDim.x * VEC;
  int cb, ce;
  column_range(d, VEC, cb, ce);
  for (int t = blockIdx.x; t < n; t += gridDim.x) {
    if (threadIdx.x < k) {
      rows[threadIdx.x] = slot_row[(size_t)t * k + threadIdx.x];
      g[threadIdx.x] = gates[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    for (int c0 = cb + threadIdx.x * VEC; c0 < ce; c0 += cstep * CU) {
      float acc[CU][VEC];
      T tmp[CU][VEC];
#pragma unroll
      for (int u = 0; u < CU; ++u) {
        const int c = c0 + u * cstep;
        if (c >= ce) break;
        const size_t off = (size_t)t * d + c;
        if (VEC > 1) {
          *reinterpret_cast<uint4*>(tmp[u]) = *reinterpret_cast<const uint4*>(h + off);
        } else {
          tmp[u][0] = h[off];
        }
      }
#pragma unroll
      for (int u = 0; u < CU; ++u)
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[u][i] = to_f32(tmp[u][i]);
      // up to KC slot rows in flight per column block, summed in rank order
      for (int j0 = 0; j0 < k; j0 += KC) {
        T yv[CU][KC][VEC];
#pragma unroll
        for (int u = 0; u < CU; ++u) {
          const int c = c0 + u * cstep;
#pragma unroll
          for (int jj = 0; jj < KC; ++jj) {
            const int j = j0 + jj;
            if (c < ce && j < k && rows[j] >= 0) {
              const T* yr = y_perm + (size_t)rows[j] * d + c;
              if (VEC > 1) *reinterpret_cast<uint4*>(yv[u][jj]) = *reinterpret_cast<const uint4*>(yr);
              else yv[u][jj][0] = yr[0];
            }
          }
        }
#pragma unroll
        for (int u = 0; u < CU; ++u)
#pragma unroll
          for (int jj = 0; jj < KC; ++jj) {
            const int j = j0 + jj;
            if (j < k && rows[j] >= 0) {
              const float gj = g[j];
#pragma unroll
              for (int i = 0; i < VEC; ++i) acc[u][i] = __fmaf_rn(gj, to_f32(yv[u][jj][i]), acc[u][i]);
            }
          }
      }
#pragma unroll
      for (int u = 0; u < CU; ++u) {
        const int c = c0 + u * cstep;
        if (c >= ce) break;
        const size_t off = (size_t)t * d + c;
        if (y_shared != nullptr) {
          if (VEC > 1) {
            *reinterpret_cast<uint4*>(tmp[u]) = *reinterpret_cast<const uint4*>(y_shared + off);
          } else {
            tmp[u][0] = y_shared[off];
          }
#pragma unroll
          for (int i = 0; i < VEC; ++i) acc[u][i] = __fadd_rn(acc[u][i], to_f32(tmp[u][i]));
        }
#pragma unroll
        for (int i = 0; i < VEC; ++i) tmp[u][i] = from_f32<T>(acc[u][i]);
        if (VEC > 1) {
          *reinterpret_cast<uint4*>(out + off) = *reinterpret_cast<const uint4*>(tmp[u]);
        } else {
          out[off] = tmp[u][0];
        }
      }
    }
    __syncthreads();
  }
}

// bias[e] = fl32(bias[e] + gamma * s), s = sign(target - counts[e]) in {-1, 0, +1}.
__global__ void bias_update_kernel(int E, const int32_t* __restrict__ counts, float target, float gamma,
                                   float* __restrict__ bias) {
  int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  float c = (float)counts[e];
  float s = (target > c) ? 1.f : ((target < c) ? -1.f : 0.f);
  bias[e] = __fadd_rn(bias[e], __fmul_rn(s, gamma));
}

// Load statistics of one routing: routed = N*k slots, kept = offsets[E],
// dropped = routed - kept, the largest pre-capacity count, and its ratio to
// the mean load fl32(N*k) / fl32(E), each division rounded to nearest.
__global__ void __launch_bounds__(256) load_stats_kernel(int slots, int E, const int32_t* __restrict__ counts,
                                                         const int32_t* __restrict__ offsets,
                                                         moe_load_stats* __restrict__ stats) {
  __shared__ int warp_max[8];
  int m = 0;
  if (slots > 0)
    for (int e = threadIdx.x; e < E; e += blockDim.x) m = max(m, counts[e]);
  m = __reduce_max_sync(0xffffffffu, m);
  if (lane_id() == 0) warp_max[warp_id()] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    int mx = 0;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) mx = max(mx, warp_max[w]);
    const int kept = slots > 0 ? offsets[E] : 0;
    const float mean = __fdiv_rn((float)slots, (float)E);
    stats->routed = slots;
    stats->kept = kept;
    stats->dropped = slots - kept;
    stats->max_count = mx;
    stats->max_over_mean = slots > 0 ? __fdiv_rn((float)mx, mean) : 0.f;
  }
}

}  // namespace moe

namespace moe_host {

template <typename T, int VEC>
static void launch_combine_t(const void* h, const void* y_perm, const int32_t* slot_row, const float* topk_gate,
                             const void* y_shared, void* out, int n, int d, int k, const int32_t* shared_offsets,
                             int e, dim3 grid, cudaStream_t s) {
#define MOE_COMBINE(KC)                                                                                    \
  moe::combine_kernel<T, VEC, KC><<<grid, 128, 0, s>>>((const T*)h, (const T*)y_perm, slot_row, topk_gate, \
                                                       (const T*)y_shared, (T*)out, n, d, k, shared_offsets, e)
#define MOE_COMBINE_COLS(KC)                                                                                  \
  moe::combine_cols_kernel<T, VEC, KC, 2><<<grid, 128, 0, s>>>((const T*)h, (const T*)y_perm, slot_row,      \
                                                               topk_gate, (const T*)y_shared, (T*)out, n, d, k, \
                                                               shared_offsets, e)
  // measured on B200: two column blocks in flight pay off for k <= 4 (the
  // Mixtral-shaped combine 37 -> 29 us); at k = 8 the extra registers cost more
  if (k <= 2) MOE_COMBINE_COLS(2);
  else if (k <= 4) MOE_COMBINE_COLS(4);
  else MOE_COMBINE(8);
#undef MOE_COMBINE_COLS
#undef MOE_COMBINE
}

moe_status launch_combine(int dtype, const void* h, const void* y_perm, const int32_t* slot_row,
                          const float* topk_gate, const void* y_shared, void* out, int n, int d, int k,
                          cudaStream_t s, const int32_t* shared_offsets, int e) {
  if (n == 0) return MOE_OK;
  const dim3 grid = row_split_grid(n, d, dtype == MOE_BF16 ? 8 : 4);
  const uintptr_t addr = (uintptr_t)h | (uintptr_t)y_perm | (uintptr_t)y_shared | (uintptr_t)out;
  if (dtype == MOE_BF16) {
    if (d % 8 == 0 && addr % 16 == 0)
      launch_combine_t<moe::bf16, 8>(h, y_perm, slot_row, topk_gate, y_shared, out, n, d, k, shared_offsets, e, grid, s);
    else
      launch_combine_t<moe::bf16, 1>(h, y_perm, slot_row, topk_gate, y_shared, out, n, d, k, shared_offsets, e, grid, s);
  } else {
    if (d % 4 == 0 && addr % 16 == 0)
      launch_combine_t<float, 4>(h, y_perm, slot_row, topk_gate, y_shared, out, n, d, k, shared_offsets, e, grid, s);
    else
      launch_combine_t<float, 1>(h, y_perm, slot_row, topk_gate, y_shared, out, n, d, k, shared_offsets, e, grid, s);
  }
  return launch_status();
}

moe_status launch_load_stats(int slots, int e, const int32_t* counts, const int32_t* offsets, moe_load_stats* stats,
                             cudaStream_t s) {
  moe::load_stats_kernel<<<1, 256, 0, s>>>(slots, e, counts, offsets, stats);
  return launch_status();
}

moe_status launch_bias_update(int e, const int32_t* counts, float target, float gamma, float* bias,
                              cudaStream_t s) {
  if (e == 0) return MOE_OK;
  moe::bias_update_kernel<<<(e + 255) / 256, 256, 0, s>>>(e, counts, target, gamma, bias);
  return launch_status();
}

}  // namespace moe_host
