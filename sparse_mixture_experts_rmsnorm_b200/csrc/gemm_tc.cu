// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by
// TMA, persistent over the SMs.  bf16 operands, fp32 accumulation.
//
// Computes, for every group g (an expert) and every row r in
// [offsets[g], offsets[g+1]) of A:
//   EPI_SWIGLU: C[r][n] = bf16(silu(A[r] . Bg[g][n]) * (A[r] . Bu[g][n]))    (step a6)
//   EPI_STORE:  C[r][n] = bf16(A[r] . B[g][n])                               (step a7)
//   EPI_F32:    C[r][n] = A[r] . B[g][n] in fp32                             (router logits, a2)
// Sources: "Mixture of Experts (MoE)" lesson (AI Engineering from Scratch,
// Phase 07), "The concept" (each expert an independent FFN, usually
// SwiGLU; the router a single linear layer); "Expert parallelism for MoE
// serving", "Future" section (GEMM units that batch many experts into one).
//
// Design (one CTA per SM, 192 threads, warp-specialised):
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 per stage,
//               128-byte swizzle, 4-stage ring (48 KiB per stage);
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma
//               (M = 128, N = 256, K = 16, both operands K-major from shared
//               memory) into one of two 256-column fp32 accumulators;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp owns the
//               32 TMEM lanes = rows its rank allows), SwiGLU or plain
//               conversion, masked stores of the rows inside the group.
// The two accumulators let the epilogue of one tile overlap the main loop
// of the next.  For SwiGLU, B holds 128 gate rows then 128 up rows of the
// same hidden units, so one N = 256 MMA produces both halves.
// Tiles are numbered group-major, then n-tile, then m-tile, so CTAs working
// at the same time share weight tiles through L2.
// Every mbarrier wait is bounded: on time-out the block records
// MOE_ERR_DEVICE_TIMEOUT in the workspace header, stops issuing work, drains
// its copies and MMAs (again with a bound), frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BN = 256;  // MMA N (accumulator columns per tile)
constexpr int TC_BK = 64;   // 128 bytes of bf16: one swizzle row
constexpr int TC_STAGES = 4;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;     // 16 KiB
constexpr int TC_B_HALF_BYTES = 128 * TC_BK * 2;  // 16 KiB (one TMA box of 128 rows)
constexpr int TC_STAGE_BYTES = TC_A_BYTES + 2 * TC_B_HALF_BYTES;
constexpr int TC_SMEM_BYTES = TC_STAGES * TC_STAGE_BYTES + 1024;  // + alignment slack
constexpr int TC_THREADS = 192;
constexpr int TC_MAX_GROUPS = 1024;
constexpr uint32_t TC_TMEM_COLS = 512;

// wait sites (word 3 of the error record)
enum { SITE_EMPTY = 1, SITE_FULL = 2, SITE_TMEM_EMPTY = 3, SITE_TMEM_FULL = 4, SITE_DRAIN = 5 };

struct TcArgs {
  const int32_t* offsets;  // [G+1] device, or nullptr: one group of max_rows rows
  int groups;
  int max_rows;
  int nout;        // output columns per group (H, d or E)
  int K;
  int n_tiles;     // n-tiles per group
  int out_cols;    // output columns per tile: 128 (SwiGLU) or 256
  void* C;
  int ldc;
  int32_t* hdr;
  uint64_t wait_ns;
};

// ---- PTX wrappers -----------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Fields: start address >> 4 (bits 0-13), leading byte offset (unused by
// swizzled K-major layouts, 1), stride byte offset 1024 >> 4 (bits 32-45),
// descriptor version 1 (bits 46-47), swizzle mode 2 = 128 B (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bit 17,
// M >> 4 at bit 24.
constexpr uint32_t tc_idesc(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

#define MOE_TMEM_LD32(taddr, r)                                                                                   \
  asm volatile(                                                                                                   \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, " \
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"              \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),           \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),     \
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),   \
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])    \
      : "r"(taddr))

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float silu_tc(float z) { return __fdiv_rn(z, __fadd_rn(1.f, expf(-z))); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x = lo (lower address), .y = hi
  return *reinterpret_cast<uint32_t*>(&p);
}

// Store 32 consecutive columns [col, col + 32) of one output row as bf16,
// masked to col < nout; 16-byte stores when the row allows them.
__device__ __forceinline__ void store_row32_bf16(bf16* out, int col, int nout, bool vec_ok, const float (&v)[32]) {
  if (vec_ok && col + 32 <= nout) {
    uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                          pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (col + i < nout) out[col + i] = __float2bfloat16_rn(v[i]);
  }
}

// ---- tile schedule -----------------------------------------------------------
struct Tile {
  int group, row0, row_end, n0;
};

__device__ __forceinline__ Tile decode_tile(int t, const int* prefix, const int* offs, int groups, int n_tiles,
                                            int out_cols) {
  int lo = 0, hi = groups - 1;  // last g with prefix[g] <= t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int rows = offs[g + 1] - offs[g];
  const int mt = (rows + TC_BM - 1) / TC_BM;
  const int local = t - prefix[g];
  Tile tl;
  tl.group = g;
  tl.row0 = offs[g] + (local % mt) * TC_BM;
  tl.row_end = offs[g + 1];
  tl.n0 = (local / mt) * out_cols;
  return tl;
}

template <int EPI>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_b2, const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[TC_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[TC_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int offs_sh[TC_MAX_GROUPS + 1];
  __shared__ int prefix_sh[TC_MAX_GROUPS + 1];

  const int warp = warp_id(), lane = lane_id();
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;

  // ---- group table: offsets and the tile prefix (n_tiles tiles per m-tile)
  const int G = args.groups;
  for (int i = threadIdx.x; i <= G; i += blockDim.x)
    offs_sh[i] = args.offsets ? args.offsets[i] : (i == 0 ? 0 : args.max_rows);
  if (threadIdx.x == 0) abort_flag = 0;
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      int g = base + lane;
      int v = 0;
      if (g < G) v = ((offs_sh[g + 1] - offs_sh[g] + TC_BM - 1) / TC_BM) * args.n_tiles;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (g < G) prefix_sh[g] = carry + x - v;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) prefix_sh[G] = carry;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 4);
    }
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(TC_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  const int total_tiles = prefix_sh[G];
  const int nk = (args.K + TC_BK - 1) / TC_BK;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_map(&map_a);
      tma_prefetch_map(&map_b);
      tma_prefetch_map(&map_b2);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile(t, prefix_sh, offs_sh, G, args.n_tiles, args.out_cols);
        const int brow = tl.group * args.nout + tl.n0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_base + stage * TC_STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], TC_STAGE_BYTES);
          tma_load_2d(sa, &map_a, &full_bar[stage], kb * TC_BK, tl.row0);
          if (EPI == moe_host::EPI_SWIGLU) {
            tma_load_2d(sa + TC_A_BYTES, &map_b, &full_bar[stage], kb * TC_BK, brow);
            tma_load_2d(sa + TC_A_BYTES + TC_B_HALF_BYTES, &map_b2, &full_bar[stage], kb * TC_BK, brow);
          } else {
            tma_load_2d(sa + TC_A_BYTES, &map_b, &full_bar[stage], kb * TC_BK, brow);
            tma_load_2d(sa + TC_A_BYTES + TC_B_HALF_BYTES, &map_b, &full_bar[stage], kb * TC_BK, brow + 128);
          }
          ++issued;
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the last (up to TC_STAGES) loads must have landed before exit.
      long n_drain = issued < TC_STAGES ? issued : TC_STAGES;
      int s = stage;
      uint32_t ph = phase;
      for (long i = 0; i < n_drain; ++i) {
        if (--s < 0) {
          s = TC_STAGES - 1;
          ph ^= 1u;
        }
        mbar_wait_bounded(&full_bar[s], ph, args.wait_ns, nullptr, args.hdr, KID_GEMM_TC, SITE_DRAIN);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc = tc_idesc(TC_BM, TC_BN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(&tempty_bar[buf], bphase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_EMPTY))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * TC_BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * TC_STAGE_BYTES;
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + TC_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk)  // K = 16 per MMA: 32 bytes further along the row
            tc_mma(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc, (kb | kk) != 0);
          tc_commit(&empty_bar[stage]);
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[buf]);
        if (++buf == 2) {
          buf = 0;
          bphase ^= 1u;
        }
      }
      // Drain: every MMA issued by this thread completes before TMEM is freed.
      tc_commit(&drain_bar);
      mbar_wait_bounded(&drain_bar, 0, args.wait_ns, nullptr, args.hdr, KID_GEMM_TC, SITE_DRAIN);
    }
  } else {
    // ======================= epilogue (warps 2..5) =======================
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r_local = quarter * 32 + lane;
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const Tile tl = decode_tile(t, prefix_sh, offs_sh, G, args.n_tiles, args.out_cols);
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait_bounded(&tfull_bar[buf], bphase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_FULL);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * TC_BN);
      const int row = tl.row0 + r_local;
      const bool row_ok = row < tl.row_end;
      if (EPI == moe_host::EPI_SWIGLU) {
        bf16* out = reinterpret_cast<bf16*>(args.C) + (size_t)row * args.ldc;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t g[32], u[32];
          MOE_TMEM_LD32(tbase + c, g);
          MOE_TMEM_LD32(tbase + 128 + c, u);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(silu_tc(__uint_as_float(g[i])), __uint_as_float(u[i]));
          if (row_ok) store_row32_bf16(out, tl.n0 + c, args.nout, (args.ldc & 7) == 0, v);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < TC_BN; c += 32) {
          uint32_t a[32];
          MOE_TMEM_LD32(tbase + c, a);
          tmem_wait_ld();
          const int col = tl.n0 + c;
          if (row_ok) {
            if (EPI == moe_host::EPI_F32) {
              float* out = reinterpret_cast<float*>(args.C) + (size_t)row * args.ldc;
              if (col + 32 <= args.nout && (args.ldc & 3) == 0) {
                uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = make_uint4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col + i < args.nout) out[col + i] = __uint_as_float(a[i]);
              }
            } else {
              float v[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(a[i]);
              store_row32_bf16(reinterpret_cast<bf16*>(args.C) + (size_t)row * args.ldc, col, args.nout,
                               (args.ldc & 7) == 0, v);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[buf]);
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TC_TMEM_COLS)
                 : "memory");
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// completes; the wait must give up and record MOE_ERR_DEVICE_TIMEOUT.
__global__ void selftest_wait_kernel(int32_t* hdr, uint64_t wait_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait_bounded(&bar, 0, wait_ns, &abort_flag, hdr, KID_SELFTEST, 1);
  }
}

}  // namespace moe

namespace moe_host {

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 map over a row-major [rows][k] matrix, box 128 rows x 64 columns,
// 128-byte swizzle, zero fill outside the matrix.
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int k) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)k * 2};
  cuuint32_t box[2] = {(cuuint32_t)moe::TC_BK, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI>
static moe_status launch_tc_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                              const moe::TcArgs& args, int grid, cudaStream_t s) {
  static bool attr_done[64] = {};
  int dev = current_device();
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(moe::gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             moe::TC_SMEM_BYTES) != cudaSuccess)
      return MOE_ERR_CUDA;
    attr_done[dev] = true;
  }
  moe::gemm_tc_kernel<EPI><<<grid, moe::TC_THREADS, moe::TC_SMEM_BYTES, s>>>(ma, mb, mb2, args);
  return launch_status();
}

moe_status launch_gemm_tc(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                          int groups, int max_rows, int nout, int k, void* c, int ldc, int32_t* hdr,
                          cudaStream_t s) {
  if (max_rows == 0 || nout == 0 || groups == 0) return MOE_OK;
  if (groups > moe::TC_MAX_GROUPS || (k % 8) != 0) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)a | (uintptr_t)b | (uintptr_t)(b2 ? b2 : b)) % 16 != 0) return MOE_ERR_UNSUPPORTED;
  CUtensorMap ma, mb, mb2;
  const int64_t b_rows = (int64_t)groups * nout;
  if (!make_map(&ma, a, max_rows, k) || !make_map(&mb, b, b_rows, k)) return MOE_ERR_CUDA;
  if (epi == EPI_SWIGLU) {
    if (!make_map(&mb2, b2, b_rows, k)) return MOE_ERR_CUDA;
  } else {
    mb2 = mb;
  }
  moe::TcArgs args;
  args.offsets = offsets;
  args.groups = offsets ? groups : 1;
  args.max_rows = max_rows;
  args.nout = nout;
  args.K = k;
  args.out_cols = (epi == EPI_SWIGLU) ? 128 : moe::TC_BN;
  args.n_tiles = (nout + args.out_cols - 1) / args.out_cols;
  args.C = c;
  args.ldc = ldc;
  args.hdr = hdr;
  args.wait_ns = wait_limit_ns();
  // Upper bound on the number of tiles; the exact count lives on the device.
  const int64_t m_tiles = (int64_t)(max_rows + moe::TC_BM - 1) / moe::TC_BM + (offsets ? groups : 0);
  const int64_t bound = m_tiles * args.n_tiles;
  const int grid = (int)(bound < sm_count() ? bound : sm_count());
  if (epi == EPI_SWIGLU) return launch_tc_t<EPI_SWIGLU>(ma, mb, mb2, args, grid, s);
  if (epi == EPI_STORE) return launch_tc_t<EPI_STORE>(ma, mb, mb2, args, grid, s);
  return launch_tc_t<EPI_F32>(ma, mb, mb2, args, grid, s);
}

moe_status launch_selftest_wait(int32_t* hdr, cudaStream_t s) {
  moe::selftest_wait_kernel<<<1, 32, 0, s>>>(hdr, wait_limit_ns());
  return launch_status();
}

}  // namespace moe_host
