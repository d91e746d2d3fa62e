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
//               conversion, masked stores of the rows inside the group; the
//               plain bf16 store sends a warp's whole 32-row blocks out
//               through a 4 KiB shared-memory stage and a TMA store.
// The two accumulators let the epilogue of one tile overlap the main loop
// of the next.  A tile of at most 64 rows (a ragged expert's last tile, or
// every tile of a decode step) runs as M = 64 MMAs; its accumulator keeps row
// r in TMEM lane (r / 16) * 32 + r % 16, the first 16 lanes of each quarter.
// For SwiGLU, B holds 128 gate rows then 128 up rows of the same hidden
// units, so one N = 256 MMA produces both halves.  A plain-store launch with
// too few tiles to fill the SMs uses 128-column tiles: one B box per stage
// and N = 128 MMAs.
// The fp32 epilogue (router logits) runs 128-column tiles (256-column ones
// when those take fewer waves) and accumulates in K-chunks.  The tensor cores' fp32 accumulator loses more
// per step than a round-to-nearest add: measured on B200 against a float64
// router with K = 7168 and 256 experts, one accumulator per tile put the
// selection keys (softmax score + bias) off by up to 1.2e-5, enough to swap
// two experts whose keys differ by 1.1e-6; chunks of 256 (or 128) along K
// bring that to 6.6e-7, and chunks of 512 to 8.9e-7.  So each chunk of
// TC_F32_CHUNK_KB k-blocks starts a fresh accumulator in one of four
// 128-column (or two 256-column) TMEM slots, and eight epilogue warps, two
// per TMEM lane quarter and each with half the columns, add the chunks in
// order in fp32 registers (round-to-nearest) before the single store of the
// row.
// Tiles are numbered group-major, then n-tile, then m-tile, so CTAs working
// at the same time share weight tiles through L2.
// Every mbarrier wait is bounded: on time-out the block records
// MOE_ERR_DEVICE_TIMEOUT in the workspace header, stops issuing work, drains
// its copies and MMAs (again with a bound), frees its TMEM and returns.
#include <cudaTypedefs.h>

#include <algorithm>

#include "tcgen05.cuh"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BN = 256;  // MMA N (accumulator columns per tile)
constexpr int TC_STAGES = 4;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;     // 16 KiB
constexpr int TC_B_HALF_BYTES = 128 * TC_BK * 2;  // 16 KiB (one TMA box of 128 rows)
constexpr int TC_STAGE_BYTES = TC_A_BYTES + 2 * TC_B_HALF_BYTES;
constexpr int TC_EPI_STAGE_BYTES = 32 * 128;  // one warp's 32 x 64 bf16 output block (TMA-store epilogue)
constexpr int TC_SMEM_BYTES = TC_STAGES * TC_STAGE_BYTES + 4 * TC_EPI_STAGE_BYTES + 1024;  // + alignment slack
constexpr int TC_THREADS = 192;
// The fp32 epilogue runs eight epilogue warps, two per TMEM lane quarter,
// each summing half of a tile's columns, so that a 256-column tile keeps at
// most 128 partial sums per thread.
template <int EPI>
constexpr int tc_threads() {
  return EPI == moe_host::EPI_F32 ? 320 : TC_THREADS;
}
constexpr int TC_F32_CHUNK_KB = 4;  // k-blocks (of 64) per fp32 partial accumulator: K = 256

// tcgen05.ld of 16 columns of the warp's 32 TMEM lanes (16 registers a thread).
#define MOE_TMEM_LD16(taddr, r)                                                                                   \
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, " \
               "%13, %14, %15}, [%16];"                                                                         \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),  \
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),         \
                 "=r"(r[15])                                                                                      \
               : "r"(taddr))

// Writes `ncols` (a multiple of 4, at most 128) fp32 values of one row from
// column n0 on, masked to columns < nout.
__device__ __forceinline__ void store_row_f32(const TcArgs& args, int row, int n0, int ncols, const float (&v)[128]) {
  float* out = reinterpret_cast<float*>(args.C) + (size_t)row * args.ldc;
  const bool vec = (args.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(args.C) & 15) == 0;
#pragma unroll
  for (int c = 0; c < 128; c += 4) {
    if (c >= ncols) break;
    const int col = n0 + c;
    if (vec && col + 4 <= args.nout) {
      *reinterpret_cast<float4*>(out + col) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (col + i < args.nout) out[col + i] = v[c + i];
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(tc_threads<EPI>(), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_b2, const __grid_constant__ CUtensorMap map_sb,
                   const __grid_constant__ CUtensorMap map_sb2, const __grid_constant__ CUtensorMap map_sa,
                   const __grid_constant__ CUtensorMap map_c, const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[TC_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[TC_STAGES];
  // accumulator slots: two of 256 columns (one per tile); for the fp32
  // epilogue one per K-chunk, four of 128 columns (128-column tiles) or two
  // of 256 (256-column tiles)
  constexpr bool F32 = EPI == moe_host::EPI_F32;
  constexpr int NBUF = F32 ? 4 : 2;
  __shared__ __align__(8) uint64_t tfull_bar[NBUF];
  __shared__ __align__(8) uint64_t tempty_bar[NBUF];
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
  if (args.pick != 0) {
    // both tilings were launched: the one not picked for these groups ends here
    __shared__ int picked_sh;
    if (warp == 0) {
      const bool pairs = pairs_picked(offs_sh, G, args.n_tiles, args.pick_pairs, args.pick_ctas);
      if (lane == 0) picked_sh = pairs ? 2 : 1;
    }
    __syncthreads();
    if (picked_sh != args.pick) return;
  }
  if (warp == 0) build_prefix<TC_BM>(offs_sh, prefix_sh, G, args.n_tiles);
  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], F32 ? 8 : 4);  // one arrival per epilogue warp
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
  const uint32_t slot_cols = (F32 && args.narrow) ? 128u : (uint32_t)TC_BN;
  const int nbuf = (F32 && args.narrow) ? 4 : 2;
  // k-blocks per accumulator and accumulators per tile
  const int chunk_kb = F32 ? TC_F32_CHUNK_KB : nk;
  const int n_chunks = F32 ? (nk + TC_F32_CHUNK_KB - 1) / TC_F32_CHUNK_KB : 1;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_map(&map_a);
      tma_prefetch_map(&map_b);
      tma_prefetch_map(&map_b2);
      if (args.shared_a) tma_prefetch_map(&map_sa);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile<TC_BM>(t, prefix_sh, offs_sh, G, args.out_cols);
        // the shared expert (when folded in as the last group) has its own weights
        const bool sh = tl.group == args.shared_group;
        const CUtensorMap* mb = sh ? &map_sb : &map_b;
        const CUtensorMap* mb2 = sh ? &map_sb2 : &map_b2;
        const int brow = (sh ? 0 : tl.group * args.nout) + tl.n0;
        // ... and, when given its own A map, reads its rows from there
        const bool sa_own = sh && args.shared_a;
        const CUtensorMap* ma = sa_own ? &map_sa : &map_a;
        const int arow = sa_own ? tl.row0 - offs_sh[tl.group] : tl.row0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_base + stage * TC_STAGE_BYTES;
          const bool narrow = EPI != moe_host::EPI_SWIGLU && args.narrow;
          mbar_arrive_expect_tx(&full_bar[stage], narrow ? TC_A_BYTES + TC_B_HALF_BYTES : TC_STAGE_BYTES);
          tma_load_2d(sa, ma, &full_bar[stage], kb * TC_BK, arow);
          if (EPI == moe_host::EPI_SWIGLU) {
            tma_load_2d(sa + TC_A_BYTES, mb, &full_bar[stage], kb * TC_BK, brow);
            tma_load_2d(sa + TC_A_BYTES + TC_B_HALF_BYTES, mb2, &full_bar[stage], kb * TC_BK, brow);
          } else {
            tma_load_2d(sa + TC_A_BYTES, mb, &full_bar[stage], kb * TC_BK, brow);
            if (!narrow)
              tma_load_2d(sa + TC_A_BYTES + TC_B_HALF_BYTES, mb, &full_bar[stage], kb * TC_BK, brow + 128);
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
      // 128-column tiles (the fp32 epilogue, and plain stores with few tiles) run N = 128 MMAs
      const int bn = (EPI != moe_host::EPI_SWIGLU && args.narrow) ? 128 : TC_BN;
      const uint32_t idesc = tc_idesc(TC_BM, bn);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile<TC_BM>(t, prefix_sh, offs_sh, G, args.out_cols);
        // a tile of at most 64 rows runs as M = 64 MMAs (half the rows of work)
        const uint32_t id = (tl.row_end - tl.row0 <= 64) ? tc_idesc(64, bn) : idesc;
        for (int c = 0; c < n_chunks && ok; ++c) {
          if (!mbar_wait_bounded(&tempty_bar[buf], bphase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_TMEM_EMPTY)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)buf * slot_cols;
          const int kb0 = c * chunk_kb;
          const int kb1 = kb0 + chunk_kb < nk ? kb0 + chunk_kb : nk;
          for (int kb = kb0; kb < kb1; ++kb) {
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
              tc_mma(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), id, ((kb - kb0) | kk) != 0);
            tc_commit(&empty_bar[stage]);
            if (++stage == TC_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit(&tfull_bar[buf]);
          if (++buf == nbuf) {
            buf = 0;
            bphase ^= 1u;
          }
        }
      }
      // Drain: every MMA issued by this thread completes before TMEM is freed.
      tc_commit(&drain_bar);
      mbar_wait_bounded(&drain_bar, 0, args.wait_ns, nullptr, args.hdr, KID_GEMM_TC, SITE_DRAIN);
    }
  } else {
    // ============ epilogue (warps 2..5; for the fp32 epilogue 2..9) ============
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r_local = quarter * 32 + lane;
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const Tile tl = decode_tile<TC_BM>(t, prefix_sh, offs_sh, G, args.out_cols);
      if constexpr (F32) {
        // the tile's K-chunks, summed in order in fp32 registers
        const bool half = tl.row_end - tl.row0 <= 64;
        const int row = half ? tl.row0 + quarter * 16 + (lane & 15) : tl.row0 + r_local;
        // warps 2..5 take the first half of the tile's columns, warps 6..9 the second
        const int my_cols = (int)slot_cols / 2;  // 64 or 128
        const int col0 = ((warp - 2) >> 2) * my_cols;
        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
        bool ok = true;
        for (int c = 0; c < n_chunks; ++c) {
          if (lane == 0)
            ok = mbar_wait_bounded(&tfull_bar[buf], bphase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                   SITE_TMEM_FULL);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          const uint32_t tb =
              tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)buf * slot_cols + (uint32_t)col0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {  // 16 columns at a time, so the sums and a load fit the registers
            if (16 * j >= my_cols) break;
            uint32_t a[16];
            MOE_TMEM_LD16(tb + 16 * j, a);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[16 * j + i] = __fadd_rn(acc[16 * j + i], __uint_as_float(a[i]));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[buf]);
          if (++buf == nbuf) {
            buf = 0;
            bphase ^= 1u;
          }
        }
        if (!ok) break;
        if (row < tl.row_end && (!half || lane < 16)) store_row_f32(args, row, tl.n0 + col0, my_cols, acc);
        continue;
      }
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait_bounded(&tfull_bar[buf], bphase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_FULL);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)buf * slot_cols;
      // M = 64 accumulators keep row r in lane (r / 16) * 32 + r % 16: lanes
      // 0..15 of each warp's quarter
      const bool half = tl.row_end - tl.row0 <= 64;
      const int ncols = args.narrow ? 128 : 256;
      if (EPI == moe_host::EPI_STORE && args.tma_store && !half && tl.row0 + quarter * 32 + 32 <= tl.row_end) {
        // a whole warp of rows: 32 x 64 blocks through shared memory and TMA
        const uint32_t stage_w = smem_base + TC_STAGES * TC_STAGE_BYTES + (uint32_t)(quarter * TC_EPI_STAGE_BYTES);
        epilogue_warp_store_tma(&map_c, tbase, stage_w, tl.row0 + quarter * 32, tl.n0, ncols);
      } else {
        const int row = half ? tl.row0 + quarter * 16 + (lane & 15) : tl.row0 + r_local;
        epilogue_row<EPI>(args, tbase, row, row < tl.row_end && (!half || lane < 16), tl.n0, ncols);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[buf]);
      if (++buf == nbuf) {
        buf = 0;
        bphase ^= 1u;
      }
    }
    // the TMA stores of this warp have written global memory before the block ends
    if (EPI == moe_host::EPI_STORE && args.tma_store && lane == 0) bulk_wait_all();
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

// The driver's tensor-map encoder, looked up once (a function-local static, so the first calls of several host
// threads are safe); nullptr when the driver does not export it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

bool make_store_map(CUtensorMap* m, void* base, int64_t rows, int cols, int ldc) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ldc * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tc_map(CUtensorMap* m, const void* base, int64_t rows, int k) { return make_tc_map_rows(m, base, rows, k, 128); }

bool make_tc_map_rows(CUtensorMap* m, const void* base, int64_t rows, int k, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)k * 2};
  cuuint32_t box[2] = {(cuuint32_t)moe::TC_BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI>
static moe_status launch_tc_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                              const CUtensorMap& msb, const CUtensorMap& msb2, const CUtensorMap& msa,
                              const CUtensorMap& mc, const moe::TcArgs& args, int grid, cudaStream_t s) {
  static SmemLimit lim;
  const moe_status st = ensure_smem_limit(moe::gemm_tc_kernel<EPI>, moe::TC_SMEM_BYTES, lim);
  if (st != MOE_OK) return st;
  moe::gemm_tc_kernel<EPI><<<grid, moe::tc_threads<EPI>(), moe::TC_SMEM_BYTES, s>>>(ma, mb, mb2, msb, msb2, msa, mc,
                                                                                    args);
  return launch_status();
}

moe_status launch_gemm_tc(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                          int groups, int max_rows, int nout, int k, void* c, int ldc, int32_t* hdr, cudaStream_t s,
                          const void* sb, const void* sb2, const void* sa, int sa_rows) {
  if (max_rows == 0 || nout == 0 || groups == 0) return MOE_OK;
  if (groups > moe::TC_MAX_GROUPS || (k % 8) != 0) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)a | (uintptr_t)b | (uintptr_t)(b2 ? b2 : b) | (uintptr_t)(sb ? sb : b) |
       (uintptr_t)(sb2 ? sb2 : b) | (uintptr_t)(sa ? sa : a)) % 16 != 0)
    return MOE_ERR_UNSUPPORTED;
  CUtensorMap ma, mb, mb2, msb, msb2, msa;
  // the routed weights hold one [nout][k] block per routed group only: a
  // folded shared expert (the last group) has its own tensor, so the map must
  // end at the routed allocation for TMA to zero-fill past it
  const int routed_groups = (sb != nullptr && offsets) ? groups - 1 : groups;
  const int64_t b_rows = (int64_t)routed_groups * nout;
  // with its own A map the shared group's rows are not in `a`, which then
  // holds the routed rows only
  const bool shared_a = sb != nullptr && offsets && sa != nullptr && sa_rows > 0;
  // (no routed rows at all: the map is never read, but must hold a row)
  const int64_t a_rows = shared_a ? std::max<int64_t>((int64_t)max_rows - sa_rows, 1) : max_rows;
  if (!make_tc_map(&ma, a, a_rows, k) || !make_tc_map(&mb, b, b_rows, k)) return MOE_ERR_CUDA;
  if (epi == EPI_SWIGLU) {
    if (!make_tc_map(&mb2, b2, b_rows, k)) return MOE_ERR_CUDA;
  } else {
    mb2 = mb;
  }
  // the shared expert folded in as the last group: its own [nout][k] weights
  if (sb != nullptr) {
    if (!make_tc_map(&msb, sb, nout, k)) return MOE_ERR_CUDA;
    if (epi == EPI_SWIGLU) {
      if (!make_tc_map(&msb2, sb2, nout, k)) return MOE_ERR_CUDA;
    } else {
      msb2 = msb;
    }
  } else {
    msb = mb;
    msb2 = mb2;
  }
  // the folded shared expert's input rows, when they are not in `a`
  if (shared_a) {
    if (!make_tc_map(&msa, sa, sa_rows, k)) return MOE_ERR_CUDA;
  } else {
    msa = ma;
  }
  moe::TcArgs args;
  args.offsets = offsets;
  args.groups = offsets ? groups : 1;
  args.max_rows = max_rows;
  args.nout = nout;
  args.K = k;
  args.out_cols = (epi == EPI_SWIGLU) ? 128 : moe::TC_BN;
  args.n_tiles = (nout + args.out_cols - 1) / args.out_cols;
  args.narrow = 0;
  args.tma_store = 0;
  args.pick = 0;
  args.pick_pairs = 1;
  args.pick_ctas = 1;
  args.C = c;
  args.ldc = ldc;
  args.hdr = hdr;
  args.wait_ns = wait_limit_ns();
  args.shared_group = (sb != nullptr && offsets) ? groups - 1 : -1;
  args.shared_a = shared_a ? 1 : 0;
  // The plain bf16 store writes whole warps' 32 x 64 blocks through TMA: one
  // box per block instead of 16-byte pieces of 32 rows, which otherwise crowd
  // the operand loads when K is short (measured on B200: the DeepSeek-V3-shaped
  // down projection, K = 2048, 2.46 -> 2.32 ms; the SwiGLU epilogue writes half
  // as much per tile and did not gain).
  CUtensorMap mc = ma;
  if (epi == EPI_STORE && (ldc % 8) == 0 && ((uintptr_t)c % 16) == 0) {
    if (!make_store_map(&mc, c, max_rows, nout, ldc)) return MOE_ERR_CUDA;
    args.tma_store = 1;
  }
  const int rows_per_group = max_rows / (offsets ? groups : 1);
  const int forced = tc_pairing();
  // Operands swapped on SM pairs (gemm_swap.cu): weight rows on M, the
  // group's rows on N in chunks of at most 256 padded to 16 (K a multiple of
  // 64).  Measured on B200 (same box, interleaved processes):
  //  - the SwiGLU projection is fastest this way on every grouped workload:
  //    DeepSeek-V3-shaped prefill 4.54 against 4.66 ms, Mixtral-shaped
  //    (8 groups of 1024) 1.58-1.61 against 1.70-1.71 ms, load-imbalance
  //    1.09-1.10 against 1.18-1.19 ms, decode (2 rows a group) 1.94 against
  //    2.00 ms;
  //  - the down projection when groups average >= 64 rows: DeepSeek-V3-shaped
  //    2.25 against 2.47 ms, Mixtral-shaped 0.67 against 0.74 ms (and 0.88
  //    with SM pairs), load-imbalance 0.53 against 0.56 ms; decode keeps the
  //    M = 64 tiles (0.97 ms either way).
  const bool swap_auto = forced == 0 && offsets != nullptr &&
                         (epi == EPI_SWIGLU || (epi == EPI_STORE && rows_per_group >= 64));
  if ((forced == 3 || swap_auto) && swap_supported(epi, nout, k, ldc))
    return launch_gemm_swap(epi, a, b, b2, offsets, groups, max_rows, nout, k, c, ldc, hdr, s, sb, sb2, sa, sa_rows);
  // Upper bound on the number of tiles; the exact count lives on the device.
  const int64_t m_tiles = (int64_t)(max_rows + moe::TC_BM - 1) / moe::TC_BM + (offsets ? groups : 0);
  if (epi == EPI_F32) {
    // fp32 outputs (the router's logits) take single-SM tiles accumulated in
    // K-chunks, whatever the tiling setting: 128 columns wide, or 256 when
    // that takes fewer waves.  A 256-column tile loads 1.5 times the bytes of
    // a 128-column one per k-block (A once, B twice), and the router's loads
    // set its pace, so it counts as 1.5 narrow tiles.
    const int64_t sms = sm_count();
    const int64_t narrow_waves = (m_tiles * ((nout + 127) / 128) + sms - 1) / sms;
    const int64_t wide_waves = (m_tiles * ((nout + 255) / 256) + sms - 1) / sms;
    const bool wide = 3 * wide_waves < 2 * narrow_waves;
    args.narrow = wide ? 0 : 1;
    args.out_cols = wide ? 256 : 128;
    args.n_tiles = (nout + args.out_cols - 1) / args.out_cols;
    const int64_t tiles = m_tiles * args.n_tiles;
    return launch_tc_t<EPI_F32>(ma, mb, mb2, msb, msb2, msa, mc, args, (int)(tiles < sms ? tiles : sms), s);
  }
  const int mode = forced == 3 ? 0 : forced;
  // A plain-store launch that would leave more than half the SMs idle runs
  // 128-column tiles on single SMs instead, twice as many.
  const bool few = epi == EPI_STORE && mode != 2 && nout > 128 && m_tiles * args.n_tiles < sm_count() / 2;
  // Measured on B200: SM pairs help the plain-store epilogue of large groups
  // (down projection) by a few percent when both tilings take the same number
  // of waves; for the SwiGLU projection the extra padding of 256-row tiles
  // outweighs the saved operand traffic.  The group sizes live on the device,
  // so for the grouped down projection both kernels are launched and each
  // keeps or drops itself from the offsets (pairs_picked); a single group
  // keeps the host rule.
  const bool pair_rule = mode == 2 || (mode == 0 && rows_per_group >= 512 && epi != EPI_SWIGLU && !few);
  const bool device_pick = mode == 0 && pair_rule && epi == EPI_STORE && offsets != nullptr;
  if (pair_rule && !device_pick)
    return launch_gemm_tc2(epi, ma, mb, mb2, msb, msb2, msa, mc, args, max_rows, offsets ? groups : 0, s);
  if (few) {
    args.narrow = 1;
    args.out_cols = 128;
    args.n_tiles = (nout + 127) / 128;
  }
  const int64_t bound = m_tiles * args.n_tiles;
  const int grid = (int)(bound < sm_count() ? bound : sm_count());
  if (device_pick) {
    args.pick_pairs = (int)tc2_pairs_launched(epi, max_rows, groups, args.n_tiles);
    args.pick_ctas = grid;
    args.pick = 2;
    const moe_status st = launch_gemm_tc2(epi, ma, mb, mb2, msb, msb2, msa, mc, args, max_rows, groups, s);
    if (st != MOE_OK) return st;
    args.pick = 1;
  }
  if (epi == EPI_SWIGLU) return launch_tc_t<EPI_SWIGLU>(ma, mb, mb2, msb, msb2, msa, mc, args, grid, s);
  return launch_tc_t<EPI_STORE>(ma, mb, mb2, msb, msb2, msa, mc, args, grid, s);
}

static std::atomic<int> g_pairing{0};
void set_tc_pairing(int mode) { g_pairing.store(mode, std::memory_order_relaxed); }
int tc_pairing() { return g_pairing.load(std::memory_order_relaxed); }

moe_status launch_selftest_wait(int32_t* hdr, cudaStream_t s) {
  moe::selftest_wait_kernel<<<1, 32, 0, s>>>(hdr, wait_limit_ns());
  return launch_status();
}

}  // namespace moe_host
