// Grouped GEMM on the CUDA cores with fp32 FFMA accumulation.
//
// Serves the fp32 layers (tensor-core TF32 cannot hold a 1e-4 output error)
// and the router of layers with few experts, where the product is a thin
// N x E matrix and the kernel only streams xn.  Step a2 (router logits,
// "Mixture of Experts (MoE)" lesson, "Step 1: the router": one linear layer
// scores every expert) and steps a6-a7 (SwiGLU experts, same lesson, "The
// concept": each expert an independent FFN, usually SwiGLU).
//
// Tiles of 64 rows x 64 columns, K in steps of 16, 256 threads with a 4x4
// register tile each.  blockIdx.x walks the m-tiles of all groups (the group
// of a tile is found from the device offsets), blockIdx.y the n-tiles.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

constexpr int SB_M = 64, SB_N = 64, SB_K = 16;

__device__ __forceinline__ float silu_f32(float z) { return __fdiv_rn(z, __fadd_rn(1.f, expf(-z))); }

template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ B,
                                                        const T* __restrict__ B2,
                                                        const int32_t* __restrict__ offsets, int G,
                                                        int max_rows, int nout, int K, void* __restrict__ C,
                                                        int ldc) {
  __shared__ float As[SB_K][SB_M + 4];
  __shared__ float Bs[SB_K][SB_N + 4];
  __shared__ float B2s[(EPI == moe_host::EPI_SWIGLU) ? SB_K : 1][SB_N + 4];
  __shared__ int tile_info[3];  // group, row_begin, row_end

  if (threadIdx.x == 0) {
    int g = -1, rb = 0, re = 0;
    if (offsets == nullptr) {
      if ((int)blockIdx.x * SB_M < max_rows) {
        g = 0;
        rb = blockIdx.x * SB_M;
        re = min(max_rows, rb + SB_M);
      }
    } else {
      int seen = 0;
      for (int i = 0; i < G; ++i) {
        int b = offsets[i], e = offsets[i + 1];
        int mt = (e - b + SB_M - 1) / SB_M;
        if ((int)blockIdx.x < seen + mt) {
          g = i;
          rb = b + (blockIdx.x - seen) * SB_M;
          re = min(e, rb + SB_M);
          break;
        }
        seen += mt;
      }
    }
    tile_info[0] = g;
    tile_info[1] = rb;
    tile_info[2] = re;
  }
  __syncthreads();
  const int g = tile_info[0];
  if (g < 0) return;
  const int rb = tile_info[1], re = tile_info[2];
  const int n0 = blockIdx.y * SB_N;
  const T* Bg = B + (size_t)g * nout * K;
  const T* B2g = (EPI == moe_host::EPI_SWIGLU) ? B2 + (size_t)g * nout * K : nullptr;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  float acc2[4][4] = {};

  for (int k0 = 0; k0 < K; k0 += SB_K) {
    // 64 x 16 tiles: 1024 elements, 4 per thread; element (r, kk) with kk fastest
    for (int i = threadIdx.x; i < SB_M * SB_K; i += 256) {
      int r = i / SB_K, kk = i % SB_K;
      int row = rb + r, col = k0 + kk;
      As[kk][r] = (row < re && col < K) ? to_f32(A[(size_t)row * K + col]) : 0.f;
      int nr = n0 + r;
      Bs[kk][r] = (nr < nout && col < K) ? to_f32(Bg[(size_t)nr * K + col]) : 0.f;
      if (EPI == moe_host::EPI_SWIGLU)
        B2s[kk][r] = (nr < nout && col < K) ? to_f32(B2g[(size_t)nr * K + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SB_K; ++kk) {
      float a[4], b[4], b2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
        if (EPI == moe_host::EPI_SWIGLU) b2[i] = B2s[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
          if (EPI == moe_host::EPI_SWIGLU) acc2[i][j] = __fmaf_rn(a[i], b2[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int row = rb + ty * 4 + i;
    if (row >= re) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int col = n0 + tx * 4 + j;
      if (col >= nout) continue;
      size_t o = (size_t)row * ldc + col;
      if (EPI == moe_host::EPI_F32) {
        ((float*)C)[o] = acc[i][j];
      } else if (EPI == moe_host::EPI_SWIGLU) {
        ((T*)C)[o] = from_f32<T>(__fmul_rn(silu_f32(acc[i][j]), acc2[i][j]));
      } else {
        ((T*)C)[o] = from_f32<T>(acc[i][j]);
      }
    }
  }
}

}  // namespace moe

namespace moe_host {

template <typename T>
static void launch_simt_t(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                          int groups, int max_rows, int nout, int k, void* c, int ldc, cudaStream_t s) {
  dim3 grid((max_rows + moe::SB_M - 1) / moe::SB_M + (offsets ? groups : 0), (nout + moe::SB_N - 1) / moe::SB_N);
  const T* A = (const T*)a;
  const T* B = (const T*)b;
  const T* B2 = (const T*)b2;
  if (epi == EPI_F32)
    moe::gemm_simt_kernel<T, EPI_F32><<<grid, 256, 0, s>>>(A, B, B2, offsets, groups, max_rows, nout, k, c, ldc);
  else if (epi == EPI_SWIGLU)
    moe::gemm_simt_kernel<T, EPI_SWIGLU><<<grid, 256, 0, s>>>(A, B, B2, offsets, groups, max_rows, nout, k, c,
                                                              ldc);
  else
    moe::gemm_simt_kernel<T, EPI_STORE><<<grid, 256, 0, s>>>(A, B, B2, offsets, groups, max_rows, nout, k, c,
                                                             ldc);
}

moe_status launch_gemm_simt(int dtype, int epi, const void* a, const void* b, const void* b2,
                            const int32_t* offsets, int groups, int max_rows, int nout, int k, void* c,
                            int ldc, cudaStream_t s) {
  if (max_rows == 0 || nout == 0) return MOE_OK;
  if (dtype == MOE_BF16)
    launch_simt_t<moe::bf16>(epi, a, b, b2, offsets, groups, max_rows, nout, k, c, ldc, s);
  else
    launch_simt_t<float>(epi, a, b, b2, offsets, groups, max_rows, nout, k, c, ldc, s);
  return launch_status();
}

}  // namespace moe_host
