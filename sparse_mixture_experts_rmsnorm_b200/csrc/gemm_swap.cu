// Grouped GEMM with the operands swapped, on SM pairs (tcgen05.mma.cta_group::2).
//
// Same products as gemm_tc.cu (steps a6 and a7; see there for the sources):
//   EPI_SWIGLU: C[r][n] = bf16(silu(X[r] . Wg[g][n]) * (X[r] . Wu[g][n]))
//   EPI_STORE:  C[r][n] = bf16(X[r] . W[g][n])
// for the rows r of group (expert) g, computed transposed,
//   D^T[n][r] = sum_k W[g][n][k] * X[r][k],
// with the expert's weight rows on the MMA's M side (256 per SM pair, 128 per
// CTA) and up to 256 of the group's rows on its N side.  A group of m rows is
// cut into ceil(m / 256) equal chunks, each rounded up to 16 rows, so a tile
// carries at most 15 rows of padding, where 128- or 256-row tiles of rows pad
// a group's last tile by up to 127 or 255.  This suits experts of a few
// hundred rows, as in the DeepSeek-V3-shaped prefill layer ("Mixture of
// Experts (MoE)" lesson, "Shared experts": 256 fine-grained routed experts,
// top-8): there each weight tile is streamed from HBM once, by one SM pair,
// while the expert's rows (a few MB) stay in L2 across its weight tiles.
//
// Roles (192 threads per CTA, clusters of two; as in gemm_tc2.cu):
//   warp 0      TMA producer in both CTAs: this CTA's 128 weight rows
//               (SwiGLU: 64 gate rows then the 64 up rows of the same hidden
//               units) and its half of the chunk's rows, in boxes of 128, 64,
//               32, 16 and 8 rows; 6-stage ring of 32 KiB; the loads complete
//               on the even CTA's full barrier;
//   warp 1      TMEM allocation (512 columns, cta_group::2); in the even CTA
//               lane 0 issues M = 256, N = rows of the chunk rounded to 16,
//               K = 16 MMAs into one of two 256-column accumulators and
//               commits to both CTAs' barriers;
//   warps 2..5  epilogue.  TMEM lane = weight row = output column, TMEM
//               column = output row.  Each warp reads 32 x 32 blocks; lanes
//               trade one value with their neighbour so that each store
//               writes two adjacent bf16 columns of one output row.  For
//               SwiGLU the warps holding up rows (lanes 64..127) pass their
//               fp32 blocks through shared memory to the warps holding the
//               gate rows of the same hidden units, which apply
//               silu(gate) * up and store.
// Tiles run group by group; within a group, chunks in runs of eight share
// the walk over the weight tiles, so the SM pairs that hold one weight tile's
// chunks run at the same time.  No TMA load uses cluster multicast.  Every
// mbarrier wait is bounded: on time-out the block records
// MOE_ERR_DEVICE_TIMEOUT, stops issuing work, drains and returns; both CTAs
// always meet at the final cluster barrier.
#include <cudaTypedefs.h>

#include <algorithm>

#include "tcgen05_pair.cuh"

namespace moe {

constexpr int S_STAGES = 6;
constexpr int S_A_BYTES = 128 * TC_BK * 2;           // 16 KiB: this CTA's 128 weight rows
constexpr int S_B_BYTES = 128 * TC_BK * 2;           // 16 KiB: up to 128 rows of the chunk
constexpr int S_STAGE_BYTES = S_A_BYTES + S_B_BYTES;  // 32 KiB
constexpr int S_XCH_BYTES = 32 * 32 * 4;              // one 32 x 32 fp32 block of up values
constexpr int S_SMEM_BYTES = S_STAGES * S_STAGE_BYTES + 4 * S_XCH_BYTES + 1024;
constexpr int S_THREADS = 192;
constexpr int S_CHUNK = 256;  // most rows of a group in one tile (the MMA's largest N)
constexpr int S_RUN = 8;      // chunks that walk a group's weight tiles together
constexpr int S_BOXES = 5;    // row boxes of 128, 64, 32, 16 and 8 rows

struct SwapMaps {
  CUtensorMap w[2];            // routed weights: gate and up (64-row boxes) or down (128-row box, w[1] = w[0])
  CUtensorMap ws[2];           // the folded shared expert's weights, the same boxes
  CUtensorMap x[S_BOXES];      // the rows: boxes of 128 >> i rows
  CUtensorMap xs[S_BOXES];     // the shared group's rows when they come from their own tensor
};

struct SwapArgs {
  const int32_t* offsets;  // [G+1] device, or nullptr: one group of max_rows rows
  int groups;
  int max_rows;
  int nout;          // output columns per group (H or d)
  int K;
  int n_o;           // weight tiles per group: ceil(H / 128) (SwiGLU) or ceil(d / 256)
  void* C;
  int ldc;
  int32_t* hdr;
  uint64_t wait_ns;
  int shared_group;  // group whose weights come from ws (-1: none)
  int shared_a;      // 1: that group's rows come from xs, from row 0
};

struct SwapTile {
  int group, row0, rows, n, o;  // rows [row0, row0 + rows) of C; n = rows rounded up to 16; weight tile o
};

// Chunks of a group of m rows, and their common size (a multiple of 16).
__device__ __forceinline__ int swap_chunks(int m) { return (m + S_CHUNK - 1) / S_CHUNK; }
__device__ __forceinline__ int swap_chunk_rows(int m, int ch) { return ((m + ch - 1) / ch + 15) & ~15; }

// One warp: prefix[g] = first tile of group g (n_o tiles per chunk).
__device__ __forceinline__ void swap_prefix(const int* offs, int* prefix, int groups, int n_o) {
  const int lane = lane_id();
  int carry = 0;
  for (int base = 0; base < groups; base += 32) {
    const int g = base + lane;
    const int v = (g < groups) ? swap_chunks(offs[g + 1] - offs[g]) * n_o : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (g < groups) prefix[g] = carry + x - v;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) prefix[groups] = carry;
}

// Tile t: its group, then within the group runs of S_RUN chunks, each run
// walking the weight tiles with its chunks innermost.
__device__ __forceinline__ SwapTile swap_decode(int t, const int* prefix, const int* offs, int groups, int n_o) {
  int lo = 0, hi = groups - 1;  // last g with prefix[g] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int m = offs[g + 1] - offs[g];
  const int ch = swap_chunks(m);
  const int nc = swap_chunk_rows(m, ch);
  const int local = t - prefix[g];
  const int run = local / (n_o * S_RUN);
  const int rem = local - run * n_o * S_RUN;
  const int in_run = min(S_RUN, ch - run * S_RUN);
  const int c = run * S_RUN + rem % in_run;
  SwapTile tl;
  tl.group = g;
  tl.o = rem / in_run;
  tl.row0 = offs[g] + c * nc;
  tl.rows = min(nc, m - c * nc);
  tl.n = (tl.rows + 15) & ~15;
  return tl;
}

// Warp-uniform bounded wait: lane 0 waits with the bound, the outcome goes to
// every lane, and each lane then observes the completed phase itself (which
// returns at once: the phase cannot move on without this warp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const SwapArgs& a, volatile int* abort,
                                          int site) {
  bool ok = true;
  if (lane_id() == 0) ok = mbar_wait_bounded(bar, parity, a.wait_ns, abort, a.hdr, KID_GEMM_TC, site);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok)
    for (int i = 0; i < (1 << 20) && !mbar_try_wait(bar, parity); ++i) {
    }
  return ok;
}

// Store 32 accumulator columns of this lane's output column `col` (lane =
// column; the block is rows row0 .. row0 + 31 of C, the first `valid` of them
// real).  Neighbouring lanes trade one value, so each lane stores two adjacent
// bf16 columns of one row: the even lane of a pair rows j, the odd lane rows
// j + 1.  nout is a multiple of 8, so a pair is inside or outside it whole.
__device__ __forceinline__ void store_cols_bf16x2(bf16* C, int ldc, int row0, int valid, int col, int nout,
                                                  const float (&v)[32]) {
  const bool odd = lane_id() & 1;
  const int c = odd ? col - 1 : col;
  const bool col_ok = c < nout;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float send = odd ? v[j] : v[j + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const int r = odd ? j + 1 : j;
    const float lo = odd ? recv : v[j];
    const float hi = odd ? v[j + 1] : recv;
    if (col_ok && r < valid)
      *reinterpret_cast<uint32_t*>(C + (size_t)(row0 + r) * ldc + c) = pack_bf16x2(lo, hi);
  }
}

enum { SITE_XFULL = 6, SITE_XEMPTY = 7 };

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(S_THREADS, 1)
    gemm_swap_kernel(const __grid_constant__ SwapMaps maps, const SwapArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S_STAGES];   // used in the even CTA
  __shared__ __align__(8) uint64_t empty_bar[S_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];        // used in the even CTA
  __shared__ __align__(8) uint64_t xfull_bar[2][2];      // SwiGLU: up block of warp pair p, buffer b, written
  __shared__ __align__(8) uint64_t xempty_bar[2][2];     //         ... and read
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
  if (warp == 0) swap_prefix(offs_sh, prefix_sh, G, args.n_o);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);  // 4 epilogue warps in each CTA
      for (int p = 0; p < 2; ++p) {
        mbar_init(&xfull_bar[p][b], 32);
        mbar_init(&xempty_bar[p][b], 32);
      }
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
      for (int i = 0; i < 2; ++i) tma_prefetch_map(&maps.w[i]);
      for (int i = 0; i < S_BOXES; ++i) tma_prefetch_map(&maps.x[i]);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = first; t < total_tiles && ok; t += step) {
        const SwapTile tl = swap_decode(t, prefix_sh, offs_sh, G, args.n_o);
        const bool sh = tl.group == args.shared_group;  // the folded shared expert has its own weights
        const CUtensorMap* w0 = sh ? &maps.ws[0] : &maps.w[0];
        const CUtensorMap* w1 = sh ? &maps.ws[1] : &maps.w[1];
        const bool own_rows = sh && args.shared_a;       // ... and may read its rows from xn, from row 0
        const CUtensorMap* xm = own_rows ? maps.xs : maps.x;
        const int half = tl.n >> 1;                      // rows of the chunk in each CTA (8 .. 128)
        const int x_row = (own_rows ? tl.row0 - offs_sh[tl.group] : tl.row0) + (int)rank * half;
        const int w_base = sh ? 0 : tl.group * args.nout;
        const int w_row = EPI == moe_host::EPI_SWIGLU ? w_base + tl.o * 128 + (int)rank * 64
                                                      : w_base + tl.o * 256 + (int)rank * 128;
        const uint32_t tx = 2u * (uint32_t)(S_A_BYTES + half * TC_BK * 2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_base + stage * S_STAGE_BYTES;
          const uint32_t full_leader = map_to_rank(&full_bar[stage], 0);
          const int kc = kb * TC_BK;
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], tx);
          if (EPI == moe_host::EPI_SWIGLU) {
            tma_load_2d_pair(sa, w0, full_leader, kc, w_row);                   // 64 gate rows
            tma_load_2d_pair(sa + S_A_BYTES / 2, w1, full_leader, kc, w_row);   // 64 up rows
          } else {
            tma_load_2d_pair(sa, w0, full_leader, kc, w_row);                   // 128 weight rows
          }
          // this CTA's rows of the chunk, in boxes of 128 or 64 / 32 / 16 / 8 rows
          uint32_t dst = sa + S_A_BYTES;
          if (half == 128) {
            tma_load_2d_pair(dst, &xm[0], full_leader, kc, x_row);
          } else {
            int r = x_row;
#pragma unroll
            for (int i = 1; i < S_BOXES; ++i) {
              const int h = 128 >> i;
              if (half & h) {
                tma_load_2d_pair(dst, &xm[i], full_leader, kc, r);
                dst += (uint32_t)(h * TC_BK * 2);
                r += h;
              }
            }
          }
          ++issued;
          if (++stage == S_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain (even CTA, which owns the full barriers): the last loads of
      // both CTAs have landed before exit.
      if (leader) {
        const long n_drain = issued < S_STAGES ? issued : S_STAGES;
        int s = stage;
        uint32_t ph = phase;
        for (long i = 0; i < n_drain; ++i) {
          if (--s < 0) {
            s = S_STAGES - 1;
            ph ^= 1u;
          }
          mbar_wait_bounded(&full_bar[s], ph, args.wait_ns, nullptr, args.hdr, KID_GEMM_TC, SITE_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer (even CTA) =======================
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      for (int t = first; t < total_tiles && ok; t += step) {
        const SwapTile tl = swap_decode(t, prefix_sh, offs_sh, G, args.n_o);
        const uint32_t idesc = tc_idesc(256, tl.n);
        if (!mbar_wait_bounded(&tempty_bar[buf], bphase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_EMPTY))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * 256);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * S_STAGE_BYTES;
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + S_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk)
            tc2_mma(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc, (kb | kk) != 0);
          tc2_commit_both(&empty_bar[stage]);
          if (++stage == S_STAGES) {
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
    const int quarter = warp & 3;  // TMEM lanes 32 * quarter .. + 31
    const int pair = quarter & 1;  // SwiGLU: gate quarter `pair`, up quarter `pair + 2`
    const bool up_warp = EPI == moe_host::EPI_SWIGLU && quarter >= 2;
    const uint32_t xch = smem_base + S_STAGES * S_STAGE_BYTES;
    bf16* C = reinterpret_cast<bf16*>(args.C);
    int buf = 0;
    uint32_t bphase = 0;
    uint32_t xcnt = 0;  // SwiGLU blocks this warp pair has passed so far
    bool ok = true;
    for (int t = first; t < total_tiles && ok; t += step) {
      const SwapTile tl = swap_decode(t, prefix_sh, offs_sh, G, args.n_o);
      if (!warp_wait(&tfull_bar[buf], bphase, args, &abort_flag, SITE_TMEM_FULL)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * 256);
      if (EPI == moe_host::EPI_STORE) {
        const int col = tl.o * 256 + (int)rank * 128 + quarter * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < tl.rows; c0 += 32) {
          uint32_t a[32];
          MOE_TMEM_LD32(tbase + c0, a);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(a[i]);
          store_cols_bf16x2(C, args.ldc, tl.row0 + c0, tl.rows - c0, col, args.nout, v);
        }
      } else {
        const int col = tl.o * 128 + (int)rank * 64 + pair * 32 + lane;  // hidden unit
#pragma unroll 1
        for (int c0 = 0; c0 < tl.rows; c0 += 32, ++xcnt) {
          const int b = (int)(xcnt & 1u);
          const uint32_t ph = (xcnt >> 1) & 1u;
          const uint32_t blk = xch + (uint32_t)((pair * 2 + b) * S_XCH_BYTES) + (uint32_t)lane * 4u;
          uint32_t a[32];
          MOE_TMEM_LD32(tbase + c0, a);
          tmem_wait_ld();
          if (up_warp) {
            // hand the up values (fp32, [column][lane]) to the gate warp
            if (!warp_wait(&xempty_bar[pair][b], ph ^ 1u, args, &abort_flag, SITE_XEMPTY)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j)
              asm volatile("st.shared.b32 [%0], %1;" ::"r"(blk + (uint32_t)(j * 128)), "r"(a[j]) : "memory");
            mbar_arrive(&xfull_bar[pair][b]);
          } else {
            if (!warp_wait(&xfull_bar[pair][b], ph, args, &abort_flag, SITE_XFULL)) {
              ok = false;
              break;
            }
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              uint32_t u;
              asm volatile("ld.shared.b32 %0, [%1];" : "=r"(u) : "r"(blk + (uint32_t)(j * 128)) : "memory");
              v[j] = __fmul_rn(silu_tc(__uint_as_float(a[j])), __uint_as_float(u));
            }
            mbar_arrive(&xempty_bar[pair][b]);
            store_cols_bf16x2(C, args.ldc, tl.row0 + c0, tl.rows - c0, col, args.nout, v);
          }
        }
        if (!ok) break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(&tempty_bar[buf], 0));
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
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
static int swap_resident_pairs() {
  static std::atomic<int> cache[64] = {};
  const int dev = current_device();
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sm_count() & ~1));
  cfg.blockDim = dim3(moe::S_THREADS);
  cfg.dynamicSmemBytes = moe::S_SMEM_BYTES;
  if (cudaOccupancyMaxActiveClusters(&n, moe::gemm_swap_kernel<EPI>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  if (n > sm_count() / 2) n = sm_count() / 2;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int EPI>
static moe_status launch_swap_t(const moe::SwapMaps& maps, const moe::SwapArgs& args, int64_t tile_bound,
                                cudaStream_t s) {
  static SmemLimit lim;
  const moe_status st = ensure_smem_limit(moe::gemm_swap_kernel<EPI>, moe::S_SMEM_BYTES, lim);
  if (st != MOE_OK) return st;
  const int64_t pairs = std::min<int64_t>(tile_bound, swap_resident_pairs<EPI>());
  moe::gemm_swap_kernel<EPI><<<(unsigned)(2 * pairs), moe::S_THREADS, moe::S_SMEM_BYTES, s>>>(maps, args);
  return launch_status();
}

moe_status launch_gemm_swap(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                            int groups, int max_rows, int nout, int k, void* c, int ldc, int32_t* hdr,
                            cudaStream_t s, const void* sb, const void* sb2, const void* sa, int sa_rows) {
  if (max_rows == 0 || nout == 0 || groups == 0) return MOE_OK;
  if (epi == EPI_F32 || groups > moe::TC_MAX_GROUPS || (k % 8) != 0 || (nout % 8) != 0 || (ldc % 8) != 0)
    return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)a | (uintptr_t)b | (uintptr_t)(b2 ? b2 : b) | (uintptr_t)(sb ? sb : b) |
       (uintptr_t)(sb2 ? sb2 : b) | (uintptr_t)(sa ? sa : a) | (uintptr_t)c) % 16 != 0)
    return MOE_ERR_UNSUPPORTED;
  const bool swiglu = epi == EPI_SWIGLU;
  const int wbox = swiglu ? 64 : 128;
  moe::SwapMaps maps;
  // the routed weights hold one [nout][k] block per routed group only; a
  // folded shared expert (the last group) has its own tensors
  const int routed_groups = (sb != nullptr && offsets) ? groups - 1 : groups;
  const int64_t w_rows = std::max<int64_t>((int64_t)routed_groups * nout, 1);
  const bool shared_a = sb != nullptr && offsets && sa != nullptr && sa_rows > 0;
  const int64_t x_rows = shared_a ? std::max<int64_t>((int64_t)max_rows - sa_rows, 1) : max_rows;
  if (!make_tc_map_rows(&maps.w[0], b, w_rows, k, wbox)) return MOE_ERR_CUDA;
  maps.w[1] = maps.w[0];
  if (swiglu && !make_tc_map_rows(&maps.w[1], b2, w_rows, k, wbox)) return MOE_ERR_CUDA;
  if (sb != nullptr) {
    if (!make_tc_map_rows(&maps.ws[0], sb, nout, k, wbox)) return MOE_ERR_CUDA;
    maps.ws[1] = maps.ws[0];
    if (swiglu && !make_tc_map_rows(&maps.ws[1], sb2, nout, k, wbox)) return MOE_ERR_CUDA;
  } else {
    maps.ws[0] = maps.w[0];
    maps.ws[1] = maps.w[1];
  }
  for (int i = 0; i < moe::S_BOXES; ++i) {
    if (!make_tc_map_rows(&maps.x[i], a, x_rows, k, 128 >> i)) return MOE_ERR_CUDA;
    if (shared_a) {
      if (!make_tc_map_rows(&maps.xs[i], sa, sa_rows, k, 128 >> i)) return MOE_ERR_CUDA;
    } else {
      maps.xs[i] = maps.x[i];
    }
  }
  moe::SwapArgs args;
  args.offsets = offsets;
  args.groups = offsets ? groups : 1;
  args.max_rows = max_rows;
  args.nout = nout;
  args.K = k;
  args.n_o = swiglu ? (nout + 127) / 128 : (nout + 255) / 256;
  args.C = c;
  args.ldc = ldc;
  args.hdr = hdr;
  args.wait_ns = wait_limit_ns();
  args.shared_group = (sb != nullptr && offsets) ? groups - 1 : -1;
  args.shared_a = shared_a ? 1 : 0;
  // upper bound on the tiles; the exact count lives on the device
  const int64_t chunks = (int64_t)(max_rows + moe::S_CHUNK - 1) / moe::S_CHUNK + args.groups;
  const int64_t bound = chunks * args.n_o;
  if (swiglu) return launch_swap_t<EPI_SWIGLU>(maps, args, bound, s);
  return launch_swap_t<EPI_STORE>(maps, args, bound, s);
}

}  // namespace moe_host
