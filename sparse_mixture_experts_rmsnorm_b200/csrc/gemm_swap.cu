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
// Loads: every operand comes through a 3-D view of its row-major [rows][K]
// matrix, {64 columns, rows, K / 64 k-blocks} with the k-block stride 128
// bytes, so that ONE TMA instruction brings S_KB consecutive k-blocks of a
// box of rows (the views need K % 64 == 0).  A stage holds S_KB k-blocks; per
// stage each CTA issues one weight load and one load of its half of the
// chunk's rows, the latter through the map whose box is exactly that many
// rows (16 maps, 8 .. 128 rows).  TMA instructions are issued at a limited
// rate per SM, and one or two of them per k-block left the tensor pipe
// waiting; two per S_KB k-blocks do not.
//
// Roles (192 threads per CTA, clusters of two; as in gemm_tc2.cu):
//   warp 0      TMA producer in both CTAs; 3-stage ring of 64 KiB; the loads
//               complete on the even CTA's full barrier;
//   warp 1      TMEM allocation (512 columns, cta_group::2); in the even CTA
//               lane 0 issues M = 256, N = rows of the chunk rounded to 16,
//               K = 16 MMAs into one of two 256-column accumulators and
//               commits to both CTAs' barriers;
//   warps 2..5  epilogue.  TMEM lane = weight row = output column, TMEM
//               column = output row.  Each warp reads 32 x 32 blocks; lanes
//               trade one value with their neighbour so that each store
//               writes two adjacent bf16 columns of one output row.  For
//               SwiGLU the even CTA holds the gate rows and the odd CTA the up
//               rows of the same 128 hidden units.  Of every 32 output rows
//               the even CTA finishes the first 16 and the odd CTA the last
//               16: each warp writes the other 16 columns of its fp32 block
//               into its partner warp's shared memory in the other CTA
//               (distributed shared memory, two buffers per warp), takes the
//               partner's values for its own 16, applies silu(gate) * up and
//               stores.
// Tiles run group by group; within a group, chunks in runs of eight share
// the walk over the weight tiles, so the SM pairs that hold one weight tile's
// chunks run at the same time.  Each pair claims its next tile from a
// per-launch counter and hands the index to the other roles through a ring.
// Data that crosses to the other CTA (ring entries, SwiGLU halves) travels by
// st.async, counted on the receiving barrier, and slots are handed back with
// relaxed arrivals: a cluster-scope release would hold the arriving thread
// until its earlier memory operations are performed at cluster scope, about
// 1.4 k cycles each time on B200.  No TMA load uses cluster multicast.  Every
// mbarrier wait is bounded: on time-out the block records
// MOE_ERR_DEVICE_TIMEOUT, stops issuing work, drains and returns; both CTAs
// always meet at the final cluster barrier.
#include <cudaTypedefs.h>

#include <algorithm>

#include "tcgen05_pair.cuh"

namespace moe {

constexpr int S_KB = 2;                                // k-blocks per stage (per TMA instruction)
constexpr int S_STAGES = 3;
constexpr int S_KBLK_BYTES = 128 * TC_BK * 2;         // one k-block of 128 rows: 16 KiB
constexpr int S_A_BYTES = S_KB * S_KBLK_BYTES;        // this CTA's 128 weight rows
constexpr int S_B_BYTES = S_KB * S_KBLK_BYTES;        // up to 128 rows of the chunk
constexpr int S_STAGE_BYTES = S_A_BYTES + S_B_BYTES;  // 64 KiB
constexpr int S_XCH_PITCH = 20;                       // words per row of an exchange block (16 + pad)
constexpr int S_XCH_BYTES = 32 * S_XCH_PITCH * 4;     // one warp's 32 rows x 16 fp32 columns
constexpr int S_SMEM_BYTES = S_STAGES * S_STAGE_BYTES + 8 * S_XCH_BYTES + 1024;  // 4 warps x 2 buffers
constexpr int S_THREADS = 192;
constexpr int S_CHUNK = 256;  // most rows of a group in one tile (the MMA's largest N)
constexpr int S_RUN = 8;      // chunks that walk a group's weight tiles together
constexpr int S_XMAPS = 16;   // row boxes of 8, 16, ..., 128 rows
constexpr int S_TRING = 8;    // tile indices published ahead of the roles that read them
// readers of each published tile index: the even CTA's MMA thread and 4 epilogue
// warps, the odd CTA's producer and 4 epilogue warps
constexpr int S_TRING_READERS = 10;

struct SwapMaps {
  CUtensorMap w[2];            // routed weights: gate and up (SwiGLU) or down (w[1] = w[0]); 128-row boxes
  CUtensorMap ws[2];           // the folded shared expert's weights
  CUtensorMap x[S_XMAPS];      // the rows: x[i] has boxes of 8 (i + 1) rows
  CUtensorMap xs[S_XMAPS];     // the shared group's rows when they come from their own tensor
};

struct SwapArgs {
  const int32_t* offsets;  // [G+1] device, or nullptr: one group of max_rows rows
  int groups;
  int max_rows;
  int nout;          // output columns per group (H or d)
  int K;             // a multiple of 64
  int n_o;           // weight tiles per group: ceil(H / 128) (SwiGLU) or ceil(d / 256)
  void* C;
  int ldc;
  int32_t* hdr;
  uint64_t wait_ns;
  int shared_group;  // group whose weights come from ws (-1: none)
  int shared_a;      // 1: that group's rows come from xs, from row 0
  int* tile_counter; // zeroed before the launch: tiles claimed past the first one of each pair (nullptr: static)
};

enum { SITE_XFULL = 6, SITE_XEMPTY = 7, SITE_RING = 8 };  // wait sites of this kernel (error record word 3)

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

// TMA load of S_KB k-blocks of a box of rows through a 3-D view, into this
// CTA's shared memory, completing on the even CTA's barrier; no multicast.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int row,
                                                 int kb) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(0), "r"(row), "r"(kb)
      : "memory");
}

// Wait on a barrier that the other CTA of the pair arrives on (acquire at
// cluster scope), with the bounded-wait rules of mbar_wait_bounded.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One thread's bounded wait on a barrier that the other CTA of the pair may
// arrive on (acquire at cluster scope).
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, const SwapArgs& a, volatile int* abort);

// Warp-uniform bounded wait: lane 0 waits with the bound, the outcome goes to
// every lane, and each lane then observes the completed phase itself (which
// returns at once: the phase cannot move on without this warp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const SwapArgs& a, volatile int* abort,
                                          int site, bool cluster_scope) {
  bool ok = true;
  if (lane_id() == 0) {
    if (cluster_scope) {
      ok = mbar_try_wait_cluster(bar, parity);
      if (!ok) {
        const uint64_t t0 = global_timer_ns();
        for (uint32_t polls = 1; !(ok = mbar_try_wait_cluster(bar, parity)); ++polls) {
          if ((polls & 63u) == 0u) {
            if (*abort) break;
            if (global_timer_ns() - t0 >= a.wait_ns) {
              record_error(a.hdr, MOE_ERR_DEVICE_TIMEOUT, KID_GEMM_TC, blockIdx.x, site);
              *abort = 1;
              break;
            }
          }
        }
      }
    } else {
      ok = mbar_wait_bounded(bar, parity, a.wait_ns, abort, a.hdr, KID_GEMM_TC, site);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok)
    for (int i = 0; i < (1 << 20); ++i)
      if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) break;
  return ok;
}

__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, const SwapArgs& a, volatile int* abort) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t polls = 1;; ++polls) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((polls & 63u) == 0u) {
      if (*abort) return false;
      if (global_timer_ns() - t0 >= a.wait_ns) {
        record_error(a.hdr, MOE_ERR_DEVICE_TIMEOUT, KID_GEMM_TC, blockIdx.x, SITE_RING);
        *abort = 1;
        return false;
      }
    }
  }
}

// Store ROWS accumulator columns of this lane's output column `col` (lane =
// column; the block is rows row0 .. row0 + ROWS - 1 of C, the first `valid` of
// them real).  Neighbouring lanes trade one value, so each lane stores two
// adjacent bf16 columns of one row: the even lane of a pair rows j, the odd
// lane rows j + 1.  nout is a multiple of 8, so a pair is inside or outside
// it whole.
template <int ROWS>
__device__ __forceinline__ void store_cols_bf16x2(bf16* C, int ldc, int row0, int valid, int col, int nout,
                                                  const float (&v)[ROWS]) {
  const bool odd = lane_id() & 1;
  const int c = odd ? col - 1 : col;
  const bool col_ok = c < nout;
#pragma unroll
  for (int j = 0; j < ROWS; j += 2) {
    const float send = odd ? v[j] : v[j + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const int r = odd ? j + 1 : j;
    const float lo = odd ? recv : v[j];
    const float hi = odd ? v[j + 1] : recv;
    if (col_ok && r < valid)
      *reinterpret_cast<uint32_t*>(C + (size_t)(row0 + r) * ldc + c) = pack_bf16x2(lo, hi);
  }
}



// silu(z) = z / (1 + e^-z) with the fast exp and divide intrinsics: about 1e-6
// relative error in fp32, far below the bf16 rounding of the activation that
// follows; z -> -inf gives -0, z -> +inf gives z.
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.f + __expf(-z)); }

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(S_THREADS, 1)
    gemm_swap_kernel(const __grid_constant__ SwapMaps maps, const SwapArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S_STAGES];   // used in the even CTA
  __shared__ __align__(8) uint64_t empty_bar[S_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];        // used in the even CTA
  __shared__ __align__(8) uint64_t xfull_bar[4][2];      // SwiGLU: the partner's block for warp q, buffer b, arrived
  __shared__ __align__(8) uint64_t xempty_bar[4][2];     //         ... this CTA's block in the partner has been read
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t tr_full[S_TRING];   // a tile index is in tile_ring[j] (both CTAs)
  __shared__ __align__(8) uint64_t tr_empty[S_TRING];  // every reader has taken it (even CTA)
  __shared__ volatile int tile_ring[S_TRING];
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
    }
    for (int q = 0; q < 4; ++q)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&xfull_bar[q][b], 1);   // lane 0 of the partner warp (plus its st.async bytes)
        mbar_init(&xempty_bar[q][b], 1);
      }
    for (int j = 0; j < S_TRING; ++j) {
      mbar_init(&tr_full[j], 1);
      mbar_init(&tr_empty[j], S_TRING_READERS);
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
  const int nk = args.K / TC_BK;
  const int n_stage_tiles = (nk + S_KB - 1) / S_KB;  // stages per tile

  if (warp == 0) {
    // ======================= TMA producer (both CTAs) =======================
    if (lane == 0) {
      // SwiGLU: the even CTA loads gate rows, the odd CTA the up rows of the same units
      const int wsel = (EPI == moe_host::EPI_SWIGLU) ? (int)rank : 0;
      tma_prefetch_map(&maps.w[wsel]);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      // Tiles: each pair starts with tile `first`; the even CTA's producer then
      // claims the next unclaimed tile from the launch's counter and publishes
      // every index (and finally one past the last tile) to the other roles of
      // both CTAs through tile_ring.  The odd CTA's producer reads the ring too.
      // A tile's successor is published right after the tile's first stage is
      // issued, so both producers already hold it when the tile's last stage
      // is out, and the claim behind it was made a whole tile earlier (the
      // atomic's round trip and the cross-CTA publish stay off the boundary).
      int rs = 0;
      uint32_t rph = 0;
      auto publish = [&](int v) -> bool {
        if (!mbar_wait_bounded(&tr_empty[rs], rph ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_RING))
          return false;
        tile_ring[rs] = v;
        mbar_arrive(&tr_full[rs]);
        // the odd CTA's copy: the word and its barrier's completion travel together
        const uint32_t peer_full = map_to_rank(&tr_full[rs], 1);
        mbar_arrive_expect_tx_cluster(peer_full, 4);
        st_async_b32(map_to_rank((const void*)&tile_ring[rs], 1), (uint32_t)v, peer_full);
        if (++rs == S_TRING) {
          rs = 0;
          rph ^= 1u;
        }
        return true;
      };
      auto take = [&](int& v) -> bool {
        if (!ring_wait(&tr_full[rs], rph, args, &abort_flag)) return false;
        v = tile_ring[rs];
        mbar_arrive_cluster_relaxed(map_to_rank(&tr_empty[rs], 0) + depend_zero((uint32_t)v));
        if (++rs == S_TRING) {
          rs = 0;
          rph ^= 1u;
        }
        return true;
      };
      // the tile after `prev` in the launch's order: the counter's next, else the pair's static successor
      auto claim = [&](int prev) -> int { return args.tile_counter ? step + atomicAdd(args.tile_counter, 1) : prev + step; };
      int t = first;
      int pending = 0;  // even CTA: the claimed successor of the next tile
      if (leader) {
        ok = publish(t);
        if (ok && t < total_tiles) pending = claim(t);
      } else {
        ok = take(t);
      }
      while (ok && t < total_tiles) {
        const SwapTile tl = swap_decode(t, prefix_sh, offs_sh, G, args.n_o);
        const bool sh = tl.group == args.shared_group;  // the folded shared expert has its own weights
        const CUtensorMap* wm = sh ? &maps.ws[wsel] : &maps.w[wsel];
        const bool own_rows = sh && args.shared_a;       // ... and may read its rows from xn, from row 0
        const int half = tl.n >> 1;                      // rows of the chunk in each CTA (8 .. 128)
        const CUtensorMap* xm = own_rows ? &maps.xs[half / 8 - 1] : &maps.x[half / 8 - 1];
        const int x_row = (own_rows ? tl.row0 - offs_sh[tl.group] : tl.row0) + (int)rank * half;
        const int w_base = sh ? 0 : tl.group * args.nout;
        const int w_row = EPI == moe_host::EPI_SWIGLU ? w_base + tl.o * 128 : w_base + tl.o * 256 + (int)rank * 128;
        const uint32_t tx = 2u * (uint32_t)(S_A_BYTES + S_KB * half * TC_BK * 2);
        int next = 0;
        bool sent = !leader;  // the even CTA still owes the ring this tile's successor
        for (int ks = 0; ks < n_stage_tiles; ++ks) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_base + stage * S_STAGE_BYTES;
          const uint32_t full_leader = map_to_rank(&full_bar[stage], 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], tx);
          tma_load_3d_pair(sa, wm, full_leader, w_row, ks * S_KB);
          tma_load_3d_pair(sa + S_A_BYTES, xm, full_leader, x_row, ks * S_KB);
          ++issued;
          if (++stage == S_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (!sent) {
            sent = true;
            next = pending;
            if (!publish(next)) {
              ok = false;
              break;
            }
            if (next < total_tiles) pending = claim(next);
          }
        }
        if (!ok) break;
        if (leader) {
          t = next;
        } else if (!take(t)) {
          break;
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
      int rs = 0;
      uint32_t rph = 0;
      while (ok) {
        if (!ring_wait(&tr_full[rs], rph, args, &abort_flag)) break;
        const int t = tile_ring[rs];
        mbar_arrive(&tr_empty[rs]);
        if (++rs == S_TRING) {
          rs = 0;
          rph ^= 1u;
        }
        if (t >= total_tiles) break;
        const SwapTile tl = swap_decode(t, prefix_sh, offs_sh, G, args.n_o);
        const uint32_t idesc = tc_idesc(256, tl.n);
        const uint32_t b_kblk = (uint32_t)((tl.n >> 1) * TC_BK * 2);  // bytes of one k-block of this CTA's rows
        if (!mbar_wait_bounded(&tempty_bar[buf], bphase ^ 1u, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                               SITE_TMEM_EMPTY))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * 256);
        for (int ks = 0; ks < n_stage_tiles; ++ks) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, args.wait_ns, &abort_flag, args.hdr, KID_GEMM_TC,
                                 SITE_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * S_STAGE_BYTES;
          const int kb_n = min(S_KB, nk - ks * S_KB);  // k-blocks of this stage inside K
          for (int j = 0; j < kb_n; ++j) {
            const uint64_t adesc = sw128_desc(sa + (uint32_t)(j * S_KBLK_BYTES));
            const uint64_t bdesc = sw128_desc(sa + S_A_BYTES + (uint32_t)j * b_kblk);
#pragma unroll
            for (int kk = 0; kk < TC_BK / 16; ++kk)
              tc2_mma(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc, (ks | j | kk) != 0);
          }
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
    const uint32_t peer = rank ^ 1u;
    // SwiGLU exchange: buffer b of this warp's row `lane` (16 fp32), here and in the partner CTA
    const uint32_t xrow = smem_base + S_STAGES * S_STAGE_BYTES + (uint32_t)(quarter * 2 * S_XCH_BYTES) +
                          (uint32_t)(lane * S_XCH_PITCH * 4);
    bf16* C = reinterpret_cast<bf16*>(args.C);
    int buf = 0;
    uint32_t bphase = 0;
    uint32_t xi = 0;  // SwiGLU: 32-row blocks this warp has handled (buffer xi & 1, phase (xi >> 1) & 1)
    bool ok = true;
    int rs = 0;
    uint32_t rph = 0;
    while (ok) {
      if (!warp_wait(&tr_full[rs], rph, args, &abort_flag, SITE_RING, true)) break;
      const int t = tile_ring[rs];
      const uint32_t z = depend_zero((uint32_t)t);  // every lane's read has returned ...
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(map_to_rank(&tr_empty[rs], 0) + z);  // ... before the slot is freed
      if (++rs == S_TRING) {
        rs = 0;
        rph ^= 1u;
      }
      if (t >= total_tiles) break;
      const SwapTile tl = swap_decode(t, prefix_sh, offs_sh, G, args.n_o);
      if (!warp_wait(&tfull_bar[buf], bphase, args, &abort_flag, SITE_TMEM_FULL, false)) break;
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
          store_cols_bf16x2<32>(C, args.ldc, tl.row0 + c0, tl.rows - c0, col, args.nout, v);
        }
      } else {
        // Block i of 32 output rows: rows 0..15 are finished by the even CTA,
        // rows 16..31 by the odd one.  Each warp sends its partner the values
        // of the partner's rows of block i + 1 before it waits for the
        // partner's values of block i, so the exchange latency hides behind
        // a block of work.
        const int col = tl.o * 128 + quarter * 32 + lane;  // hidden unit
        const int nblk = (tl.rows + 31) >> 5;
        uint32_t own[16];  // this CTA's values (gate or up) of its own 16 rows of the current block
        // send block j (buffer xi & 1 of the partner) and keep this CTA's half of it in own[]
        auto send_block = [&](int j, uint32_t x) -> bool {
          uint32_t a[32];
          MOE_TMEM_LD32(tbase + (uint32_t)(j * 32), a);
          tmem_wait_ld();
          const int b = (int)(x & 1u);
          if (!warp_wait(&xempty_bar[quarter][b], ((x >> 1) & 1u) ^ 1u, args, &abort_flag, SITE_XEMPTY, true))
            return false;
          uint32_t snd[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            snd[i] = leader ? a[16 + i] : a[i];
            own[i] = leader ? a[i] : a[16 + i];
          }
          // the values and the partner's barrier completion travel together (st.async)
          const uint32_t dst = map_to_rank_addr(xrow + (uint32_t)(b * S_XCH_BYTES), peer);
          const uint32_t peer_full = map_to_rank(&xfull_bar[quarter][b], peer);
          if (lane == 0) mbar_arrive_expect_tx_cluster(peer_full, 32u * 16u * 4u);
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            st_async_v4(dst + (uint32_t)(i * 4), snd[i], snd[i + 1], snd[i + 2], snd[i + 3], peer_full);
          return true;
        };
        if (nblk > 0 && !send_block(0, xi)) {
          ok = false;
          break;
        }
#pragma unroll 1
        for (int j = 0; j < nblk; ++j, ++xi) {
          uint32_t cur[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) cur[i] = own[i];
          if (j + 1 < nblk && !send_block(j + 1, xi + 1)) {
            ok = false;
            break;
          }
          const int b = (int)(xi & 1u);
          if (!warp_wait(&xfull_bar[quarter][b], (xi >> 1) & 1u, args, &abort_flag, SITE_XFULL, true)) {
            ok = false;
            break;
          }
          const uint32_t xb = xrow + (uint32_t)(b * S_XCH_BYTES);
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            uint32_t u[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                         : "r"(xb + (uint32_t)(i * 4))
                         : "memory");
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float mv = __uint_as_float(cur[i + e]), other = __uint_as_float(u[e]);
              const float g = leader ? mv : other, up = leader ? other : mv;
              v[i + e] = __fmul_rn(silu_fast(g), up);
            }
          }
          // every lane's reads of the buffer have returned (v depends on all four loads) before
          // lane 0 lets the partner overwrite it
          const uint32_t z = depend_zero(__float_as_uint(v[3]) ^ __float_as_uint(v[7]) ^ __float_as_uint(v[11]) ^
                                         __float_as_uint(v[15]));
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(map_to_rank(&xempty_bar[quarter][b], peer) + z);
          const int mine = (int)rank * 16;
          store_cols_bf16x2<16>(C, args.ldc, tl.row0 + j * 32 + mine, tl.rows - j * 32 - mine, col, args.nout, v);
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

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();  // gemm_tc.cu

// 3-D view {64 columns, rows, k / 64 k-blocks} of a row-major bf16 [rows][k]
// matrix (k % 64 == 0), the k-block stride 128 bytes: a box of `box_rows`
// rows and S_KB k-blocks, 128-byte swizzle, zero fill outside the matrix.
static bool make_kblock_map(CUtensorMap* m, const void* base, int64_t rows, int k, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)moe::TC_BK, (cuuint64_t)rows, (cuuint64_t)(k / moe::TC_BK)};
  cuuint64_t strides[2] = {(cuuint64_t)k * 2, (cuuint64_t)moe::TC_BK * 2};
  cuuint32_t box[3] = {(cuuint32_t)moe::TC_BK, (cuuint32_t)box_rows, (cuuint32_t)moe::S_KB};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

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

bool swap_supported(int epi, int nout, int k, int ldc) {
  return epi != EPI_F32 && k >= moe::TC_BK && k % moe::TC_BK == 0 && nout % 8 == 0 && ldc % 8 == 0;
}

moe_status launch_gemm_swap(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                            int groups, int max_rows, int nout, int k, void* c, int ldc, int32_t* hdr,
                            cudaStream_t s, const void* sb, const void* sb2, const void* sa, int sa_rows) {
  if (max_rows == 0 || nout == 0 || groups == 0) return MOE_OK;
  if (!swap_supported(epi, nout, k, ldc) || groups > moe::TC_MAX_GROUPS) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)a | (uintptr_t)b | (uintptr_t)(b2 ? b2 : b) | (uintptr_t)(sb ? sb : b) |
       (uintptr_t)(sb2 ? sb2 : b) | (uintptr_t)(sa ? sa : a) | (uintptr_t)c) % 16 != 0)
    return MOE_ERR_UNSUPPORTED;
  const bool swiglu = epi == EPI_SWIGLU;
  moe::SwapMaps maps;
  // the routed weights hold one [nout][k] block per routed group only; a
  // folded shared expert (the last group) has its own tensors
  const int routed_groups = (sb != nullptr && offsets) ? groups - 1 : groups;
  const int64_t w_rows = std::max<int64_t>((int64_t)routed_groups * nout, 1);
  const bool shared_a = sb != nullptr && offsets && sa != nullptr && sa_rows > 0;
  const int64_t x_rows = shared_a ? std::max<int64_t>((int64_t)max_rows - sa_rows, 1) : max_rows;
  if (!make_kblock_map(&maps.w[0], b, w_rows, k, 128)) return MOE_ERR_CUDA;
  maps.w[1] = maps.w[0];
  if (swiglu && !make_kblock_map(&maps.w[1], b2, w_rows, k, 128)) return MOE_ERR_CUDA;
  if (sb != nullptr) {
    if (!make_kblock_map(&maps.ws[0], sb, nout, k, 128)) return MOE_ERR_CUDA;
    maps.ws[1] = maps.ws[0];
    if (swiglu && !make_kblock_map(&maps.ws[1], sb2, nout, k, 128)) return MOE_ERR_CUDA;
  } else {
    maps.ws[0] = maps.w[0];
    maps.ws[1] = maps.w[1];
  }
  for (int i = 0; i < moe::S_XMAPS; ++i) {
    if (!make_kblock_map(&maps.x[i], a, x_rows, k, 8 * (i + 1))) return MOE_ERR_CUDA;
    if (shared_a) {
      if (!make_kblock_map(&maps.xs[i], sa, sa_rows, k, 8 * (i + 1))) return MOE_ERR_CUDA;
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
  // the tile counter lives in the workspace header (word 32), zeroed for every launch
  args.tile_counter = nullptr;
  if (hdr != nullptr) {
    args.tile_counter = hdr + 32;
    if (cudaMemsetAsync(args.tile_counter, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // upper bound on the tiles; the exact count lives on the device
  const int64_t chunks = (int64_t)(max_rows + moe::S_CHUNK - 1) / moe::S_CHUNK + args.groups;
  const int64_t bound = chunks * args.n_o;
  if (swiglu) return launch_swap_t<EPI_SWIGLU>(maps, args, bound, s);
  return launch_swap_t<EPI_STORE>(maps, args, bound, s);
}

}  // namespace moe_host
