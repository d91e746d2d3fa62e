// Grouped GEMM on SM pairs: tcgen05.mma.cta_group::2 over a 2-CTA cluster.
//
// Same products and epilogues as gemm_tc.cu (steps a2, a6, a7; see there
// for the sources), with 256-row tiles split over the two SMs of a cluster:
// each CTA holds 128 rows of A and half (128 rows) of the 256-row B tile,
// and one MMA (M = 256, N = 256, K = 16) issued by the even CTA multiplies
// both halves.  Per SM a k-block then costs 32 KiB of operands instead of
// 48 KiB, so six stages fit where the single-SM kernel holds four, and each
// weight tile crosses L2 -> SM once per 256 rows.  Each CTA keeps its own
// 128 rows x 2 x 256 fp32 accumulators in TMEM (double-buffered).
//
// Roles (192 threads per CTA):
//   warp 0      TMA producer in both CTAs: waits for its own free stage and
//               loads its A and B halves; the loads complete on the even
//               CTA's full barrier, which alone posts the expected bytes;
//   warp 1      TMEM allocation (both CTAs, cta_group::2); in the even CTA
//               lane 0 issues the MMAs and commits to the stage and
//               accumulator barriers of both CTAs at once (multicast commit);
//   warps 2..5  epilogue of the CTA's own 128 rows (the plain bf16 store
//               through shared memory and TMA stores, as in the single-SM
//               kernel), then one arrival per warp on the even CTA's
//               accumulator-empty barrier.
// No TMA load uses cluster multicast.  Every mbarrier wait is bounded as in
// the single-SM kernel; both CTAs always meet at the final cluster barrier.
#include <cudaTypedefs.h>

#include "tcgen05_pair.cuh"

namespace moe {

constexpr int P_BM = 256;  // rows per pair tile (128 per CTA)
constexpr int P_BN = 256;  // MMA N
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = 128 * TC_BK * 2;              // 16 KiB: this CTA's rows of A
constexpr int P_B_BYTES = 128 * TC_BK * 2;              // 16 KiB: this CTA's half of B
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;    // 32 KiB
constexpr int P_EPI_STAGE_BYTES = 32 * 128;  // one warp's 32 x 64 bf16 output block (TMA-store epilogue)
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + 4 * P_EPI_STAGE_BYTES + 1024;
constexpr int P_THREADS = 192;

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ CUtensorMap map_b2, const __grid_constant__ CUtensorMap map_sb,
                    const __grid_constant__ CUtensorMap map_sb2, const __grid_constant__ CUtensorMap map_sa,
                    const __grid_constant__ CUtensorMap map_c, const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[P_STAGES];   // used in the even CTA
  __shared__ __align__(8) uint64_t empty_bar[P_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];        // used in the even CTA
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int offs_sh[TC_MAX_GROUPS + 1];
  __shared__ int prefix_sh[TC_MAX_GROUPS + 1];

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int first = (int)cluster_index(), step = (int)cluster_count();
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;

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
  if (warp == 0) build_prefix<P_BM>(offs_sh, prefix_sh, G, args.n_tiles);
  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(TC_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  const int total_tiles = prefix_sh[G];
  const int nk = (args.K + TC_BK - 1) / TC_BK;

  if (warp == 0) {
    // ======================= TMA producer (both CTAs) =======================
    if (lane == 0) {
      tma_prefetch_map(&map_a);
      if (args.shared_a) tma_prefetch_map(&map_sa);
      const bool second = rank == 1 && EPI == moe_host::EPI_SWIGLU;  // the up half of a SwiGLU tile
      tma_prefetch_map(second ? &map_b2 : &map_b);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = first; t < total_tiles && ok; t += step) {
        const Tile tl = decode_tile<P_BM>(t, prefix_sh, offs_sh, G, args.out_cols);
        const bool sh = tl.group == args.shared_group;  // the folded shared expert has its own weights
        const CUtensorMap* bmap = sh ? (second ? &map_sb2 : &map_sb) : (second ? &map_b2 : &map_b);
        // the folded shared expert's rows may come from their own A map, from row 0
        const bool sa_own = sh && args.shared_a;
        const CUtensorMap* amap = sa_own ? &map_sa : &map_a;
        const int a_row = (sa_own ? tl.row0 - offs_sh[tl.group] : tl.row0) + (int)rank * 128;
        const int b_row = (sh ? 0 : tl.group * args.nout) + tl.n0 + (EPI == moe_host::EPI_SWIGLU ? 0 : (int)rank * 128);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_base + stage * P_STAGE_BYTES;
          const uint32_t full_leader = map_to_rank(&full_bar[stage], 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * P_STAGE_BYTES);
          tma_load_2d_pair(sa, amap, full_leader, kb * TC_BK, a_row);
          tma_load_2d_pair(sa + P_A_BYTES, bmap, full_leader, kb * TC_BK, b_row);
          ++issued;
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain (even CTA, which owns the full barriers): the last loads of
      // both CTAs have landed before exit.
      if (leader) {
        long n_drain = issued < P_STAGES ? issued : P_STAGES;
        int s = stage;
        uint32_t ph = phase;
        for (long i = 0; i < n_drain; ++i) {
          if (--s < 0) {
            s = P_STAGES - 1;
            ph ^= 1u;
          }
          mbar_wait_bounded(&full_bar[s], ph, args.wait_ns, nullptr, args.hdr, KID_GEMM_TC, SITE_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer (even CTA) =======================
    if (leader && lane == 0) {
      constexpr uint32_t idesc = tc_idesc(P_BM, P_BN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      for (int t = first; t < total_tiles && ok; t += step) {
        if (!mbar_wait_bounded(&tempty_bar[buf], bphase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_EMPTY))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * P_BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * P_STAGE_BYTES;
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + P_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk)
            tc2_mma(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc, (kb | kk) != 0);
          tc2_commit_both(&empty_bar[stage]);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc2_commit_both(&tfull_bar[buf]);
        if (++buf == 2) {
          buf = 0;
          bphase ^= 1u;
        }
      }
      // Drain: every MMA issued here completes before TMEM is freed and
      // before the odd CTA (whose shared memory they read) may exit.
      tc2_commit_own(&drain_bar);
      mbar_wait_bounded(&drain_bar, 0, args.wait_ns, nullptr, args.hdr, KID_GEMM_TC, SITE_DRAIN);
    }
  } else {
    // ======================= epilogue (warps 2..5, both CTAs) =======================
    const int quarter = warp & 3;
    const int r_local = (int)rank * 128 + quarter * 32 + lane;
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = first; t < total_tiles; t += step) {
      const Tile tl = decode_tile<P_BM>(t, prefix_sh, offs_sh, G, args.out_cols);
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait_bounded(&tfull_bar[buf], bphase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_FULL);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * P_BN);
      const int row = tl.row0 + r_local;
      const int wrow0 = tl.row0 + (int)rank * 128 + quarter * 32;
      if (EPI == moe_host::EPI_STORE && args.tma_store && wrow0 + 32 <= tl.row_end) {
        // a whole warp of rows: 32 x 64 blocks through shared memory and TMA
        const uint32_t stage_w = smem_base + P_STAGES * P_STAGE_BYTES + (uint32_t)(quarter * P_EPI_STAGE_BYTES);
        epilogue_warp_store_tma(&map_c, tbase, stage_w, wrow0, tl.n0, 256);
      } else {
        epilogue_row<EPI>(args, tbase, row, row < tl.row_end, tl.n0);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(&tempty_bar[buf], 0));
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
    // the TMA stores of this warp have written global memory before the block ends
    if (EPI == moe_host::EPI_STORE && args.tma_store && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TC_TMEM_COLS)
                 : "memory");
}

}  // namespace moe

namespace moe_host {

// Clusters of two that can be resident at once (one CTA per SM), per device.
template <int EPI>
static int resident_pairs() {
  static std::atomic<int> cache[64] = {};
  const int dev = current_device();
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sm_count() & ~1));
  cfg.blockDim = dim3(moe::P_THREADS);
  cfg.dynamicSmemBytes = moe::P_SMEM_BYTES;
  if (cudaOccupancyMaxActiveClusters(&n, moe::gemm_tc2_kernel<EPI>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  if (n > sm_count() / 2) n = sm_count() / 2;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

static int resident_pairs_of(int epi) {
  if (epi == EPI_SWIGLU) return resident_pairs<EPI_SWIGLU>();
  return resident_pairs<EPI_STORE>();
}

// Upper bound on the pair tiles (the exact count lives on the device).
static int64_t pair_tile_bound(int64_t max_rows, int groups_bound, int n_tiles) {
  return ((max_rows + moe::P_BM - 1) / moe::P_BM + groups_bound) * n_tiles;
}

int64_t tc2_pairs_launched(int epi, int64_t max_rows, int groups_bound, int n_tiles) {
  const int64_t bound = pair_tile_bound(max_rows, groups_bound, n_tiles);
  const int64_t res = resident_pairs_of(epi);
  return bound < res ? bound : res;
}

template <int EPI>
static moe_status launch_tc2_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                               const CUtensorMap& msb, const CUtensorMap& msb2, const CUtensorMap& msa,
                               const CUtensorMap& mc, const moe::TcArgs& args, int64_t pair_bound, cudaStream_t s) {
  static SmemLimit lim;
  const moe_status st = ensure_smem_limit(moe::gemm_tc2_kernel<EPI>, moe::P_SMEM_BYTES, lim);
  if (st != MOE_OK) return st;
  const int64_t pairs = pair_bound < resident_pairs<EPI>() ? pair_bound : resident_pairs<EPI>();
  moe::gemm_tc2_kernel<EPI><<<(unsigned)(2 * pairs), moe::P_THREADS, moe::P_SMEM_BYTES, s>>>(ma, mb, mb2, msb, msb2,
                                                                                          msa, mc, args);
  return launch_status();
}

// Launch of the SM-pair kernel; maps and arguments come from launch_gemm_tc.
moe_status launch_gemm_tc2(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                           const CUtensorMap& msb, const CUtensorMap& msb2, const CUtensorMap& msa,
                           const CUtensorMap& mc, const moe::TcArgs& args, int64_t max_rows, int groups_bound,
                           cudaStream_t s) {
  const int64_t bound = pair_tile_bound(max_rows, groups_bound, args.n_tiles);
  if (epi == EPI_SWIGLU) return launch_tc2_t<EPI_SWIGLU>(ma, mb, mb2, msb, msb2, msa, mc, args, bound, s);
  if (epi == EPI_STORE) return launch_tc2_t<EPI_STORE>(ma, mb, mb2, msb, msb2, msa, mc, args, bound, s);
  return MOE_ERR_UNSUPPORTED;  // fp32 outputs run on the single-SM kernel only
}

}  // namespace moe_host
