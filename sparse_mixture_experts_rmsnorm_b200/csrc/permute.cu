// Steps a4 and a5 of the MoE layer: per-expert counting sort of the N*k
// routing slots with an optional capacity, and the gather of token rows into
// expert-contiguous buffers.
//
// Sources: Ultralytics glossary "Mixture of Experts (MoE)", "Load balancing
// and expert capacity" (tokens per expert; tokens over an expert's limit
// continue on the residual) and its top-2 example (each expert takes the
// tokens that chose it, in token order); "Mixture of Experts (MoE)" lesson,
// "The load-balancing problem" (expert capacity C x N / E, overflow tokens
// pass the layer); "Expert parallelism for MoE serving", "Technical insight"
// (dispatch groups each expert's tokens; capacity keeps GEMM shapes
// predictable).
//
// Slot s = t*k + j.  Its rank within expert e is the number of slots s' < s
// routed to e; with a capacity, ranks >= cap are dropped.  The order is fixed
// by the slot index alone (no atomics decide it), so the result is
// deterministic and equals a stable sort.
//
// Kernels: (1) one warp per chunk of 256 slots counts the chunk's slots per
// expert into hist[e][chunk]; (2) one block scans each expert's row of hist
// (giving every chunk the rank of its first slot within the expert) and
// forms the kept counts and offsets; (3) the chunk warps recompute their
// in-chunk ranks and write slot_row / row_token; (4) the gather copies each
// token's row to its kept slots with 16-byte accesses.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

constexpr int kChunk = 256;        // slots per warp
constexpr int kPermWarps = 4;      // warps per block in kernels (1) and (3)

// In-chunk ranking shared by kernels (1) and (3).  `run` is this warp's
// shared running count per expert (zeroed by the caller).  For each slot of
// the chunk in increasing order, calls f(slot, expert, rank_in_chunk).
template <typename F>
__device__ __forceinline__ void chunk_walk(const int32_t* __restrict__ idx, int64_t slots, int64_t c,
                                           int32_t* run, F f) {
  const int lane = lane_id();
  const unsigned lt = (1u << lane) - 1u;
  for (int step = 0; step < kChunk / 32; ++step) {
    int64_t s = c * kChunk + step * 32 + lane;
    int e = (s < slots) ? idx[s] : -1;
    unsigned same = __match_any_sync(0xffffffffu, e);
    int before = __popc(same & lt);
    int base = (e >= 0) ? run[e] : 0;
    __syncwarp();
    if (e >= 0) {
      f(s, e, base + before);
      if (before == 0) run[e] = base + __popc(same);  // the lowest lane of each group
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kPermWarps * 32) chunk_hist_kernel(const int32_t* __restrict__ idx,
                                                                     int64_t slots, int E, int nchunks,
                                                                     int32_t* __restrict__ hist) {
  extern __shared__ int32_t run_all[];
  int32_t* run = run_all + warp_id() * E;
  int64_t c = (int64_t)blockIdx.x * kPermWarps + warp_id();
  for (int e = lane_id(); e < E; e += 32) run[e] = 0;
  __syncwarp();
  if (c >= nchunks) return;
  chunk_walk(idx, slots, c, run, [](int64_t, int, int) {});
  for (int e = lane_id(); e < E; e += 32) hist[(int64_t)e * nchunks + c] = run[e];
}

// One block of 1024 threads.
//   1. Each warp takes whole experts, kScanExp at a time: the exclusive scan
//      of hist[e][*] over the chunks, in place, gives every chunk the rank of
//      its first slot of expert e; the row total is count_e (also written to
//      `counts` when given).  The warp loads kScanExp rows of 32 * kScanPer
//      chunk counts with coalesced, independent loads, scans them as warp
//      scans in registers and stores them back coalesced: one memory round
//      trip per kScanExp experts and 32 * kScanPer chunks.
//   2. kept_e = min(count_e, cap); offsets = exclusive scan of kept (E+1).
constexpr int kScanPer = 8;
constexpr int kScanExp = 4;

__global__ void __launch_bounds__(1024) hist_scan_kernel(int32_t* __restrict__ hist, int E, int nchunks, int cap,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ offsets_ext, int extra,
                                                         int32_t* __restrict__ counts) {
  __shared__ int32_t kept_sh[1024];
  __shared__ int32_t warp_sum[32];
  const int lane = lane_id(), warp = warp_id();
  for (int e0 = warp; e0 < E; e0 += 32 * kScanExp) {
    int32_t carry[kScanExp];
#pragma unroll
    for (int b = 0; b < kScanExp; ++b) carry[b] = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 32 * kScanPer) {
      int32_t v[kScanExp][kScanPer];
#pragma unroll
      for (int b = 0; b < kScanExp; ++b) {
        const int e = e0 + 32 * b;
#pragma unroll
        for (int i = 0; i < kScanPer; ++i) {
          const int c = c0 + 32 * i + lane;
          v[b][i] = (e < E && c < nchunks) ? hist[(int64_t)e * nchunks + c] : 0;
        }
      }
#pragma unroll
      for (int b = 0; b < kScanExp; ++b) {
#pragma unroll
        for (int i = 0; i < kScanPer; ++i) {
          int32_t x = v[b][i];
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
          }
          v[b][i] = carry[b] + x - v[b][i];
          carry[b] += __shfl_sync(0xffffffffu, x, 31);
        }
      }
#pragma unroll
      for (int b = 0; b < kScanExp; ++b) {
        const int e = e0 + 32 * b;
        if (e >= E) continue;  // uniform across the warp
#pragma unroll
        for (int i = 0; i < kScanPer; ++i) {
          const int c = c0 + 32 * i + lane;
          if (c < nchunks) hist[(int64_t)e * nchunks + c] = v[b][i];
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < kScanExp; ++b) {
        const int e = e0 + 32 * b;
        if (e >= E) continue;
        kept_sh[e] = (cap >= 0 && carry[b] > cap) ? cap : carry[b];
        if (counts != nullptr) counts[e] = carry[b];
      }
    }
  }
  __syncthreads();
  const int tid = threadIdx.x;
  const int32_t k = (tid < E) ? kept_sh[tid] : 0;
  int32_t x = k;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t w = warp_sum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int32_t excl = x - k + (warp > 0 ? warp_sum[warp - 1] : 0);
  if (tid < E) offsets[tid] = excl;
  if (tid == E - 1) offsets[E] = excl + k;
  if (offsets_ext != nullptr) {  // the same offsets plus a trailing group of `extra` rows
    if (tid < E) offsets_ext[tid] = excl;
    if (tid == E - 1) {
      offsets_ext[E] = excl + k;
      offsets_ext[E + 1] = excl + k + extra;
    }
  }
}

__global__ void __launch_bounds__(kPermWarps * 32) chunk_scatter_kernel(
    const int32_t* __restrict__ idx, int64_t slots, int k, int E, int nchunks, int cap,
    const int32_t* __restrict__ hist, const int32_t* __restrict__ offsets, int32_t* __restrict__ slot_row,
    int32_t* __restrict__ row_token) {
  extern __shared__ int32_t run_all[];
  int32_t* run = run_all + warp_id() * E;
  int64_t c = (int64_t)blockIdx.x * kPermWarps + warp_id();
  for (int e = lane_id(); e < E; e += 32) run[e] = 0;
  __syncwarp();
  if (c >= nchunks) return;
  chunk_walk(idx, slots, c, run, [&](int64_t s, int e, int r_in_chunk) {
    int32_t rank = hist[(int64_t)e * nchunks + c] + r_in_chunk;
    if (cap < 0 || rank < cap) {
      int32_t row = offsets[e] + rank;
      slot_row[s] = row;
      row_token[row] = (int32_t)(s / k);
    } else {
      slot_row[s] = -1;
    }
  });
}

// Kernels (1)-(3) in one block of 1024 threads, for up to 32 chunks when
// the histogram and the per-warp running counts fit shared memory
// (decode-sized and Mixtral-sized batches): warp w walks chunk w, the
// histogram stays in shared memory, and the same scans and ranks as above
// follow with block barriers instead of kernel boundaries.
__global__ void __launch_bounds__(1024) permute_fused_kernel(const int32_t* __restrict__ idx, int64_t slots, int k,
                                                             int E, int nchunks, int cap,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ offsets_ext, int extra,
                                                             int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ slot_row,
                                                             int32_t* __restrict__ row_token) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;                         // [E][nchunks]
  int32_t* run = sm + (size_t)E * nchunks + (size_t)warp_id() * E;  // this warp's running counts
  __shared__ int32_t kept_sh[1024];
  __shared__ int32_t offs_sh[1024];
  __shared__ int32_t warp_sum[32];
  const int lane = lane_id(), warp = warp_id();
  const int c = warp;
  for (int e = lane; e < E; e += 32) run[e] = 0;
  __syncwarp();
  if (c < nchunks) {
    chunk_walk(idx, slots, c, run, [](int64_t, int, int) {});
    for (int e = lane; e < E; e += 32) hist[e * nchunks + c] = run[e];
  }
  __syncthreads();
  // exclusive scan of each expert's row over the chunks (nchunks <= 32)
  for (int e = warp; e < E; e += 32) {
    const int32_t v = lane < nchunks ? hist[e * nchunks + lane] : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < nchunks) hist[e * nchunks + lane] = x - v;
    const int32_t total = __shfl_sync(0xffffffffu, x, 31);
    if (lane == 0) {
      kept_sh[e] = (cap >= 0 && total > cap) ? cap : total;
      if (counts != nullptr) counts[e] = total;
    }
  }
  __syncthreads();
  const int tid = threadIdx.x;
  const int32_t kv = (tid < E) ? kept_sh[tid] : 0;
  int32_t x = kv;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t w = warp_sum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sum[lane] = w;
  }
  __syncthreads();
  const int32_t excl = x - kv + (warp > 0 ? warp_sum[warp - 1] : 0);
  if (tid < E) {
    offs_sh[tid] = excl;
    offsets[tid] = excl;
    if (offsets_ext != nullptr) offsets_ext[tid] = excl;
  }
  if (tid == E - 1) {
    offsets[E] = excl + kv;
    if (offsets_ext != nullptr) {
      offsets_ext[E] = excl + kv;
      offsets_ext[E + 1] = excl + kv + extra;
    }
  }
  __syncthreads();
  // ranks: the chunk's first rank per expert plus the in-chunk rank
  for (int e = lane; e < E; e += 32) run[e] = 0;
  __syncwarp();
  if (c < nchunks) {
    chunk_walk(idx, slots, c, run, [&](int64_t s, int e, int r_in_chunk) {
      const int32_t rank = hist[e * nchunks + c] + r_in_chunk;
      if (cap < 0 || rank < cap) {
        const int32_t row = offs_sh[e] + rank;
        slot_row[s] = row;
        row_token[row] = (int32_t)(s / k);
      } else {
        slot_row[s] = -1;
      }
    });
  }
}

// a5 in token order: token t's row of xn is read once and written to each
// of its kept slots, x_perm[slot_row[t * k + j]] = xn[t].  (A folded shared
// expert reads its rows straight from xn.)  Every x_perm row r < R has
// exactly one kept slot pointing at it,
// so this writes the same x_perm as reading x_perm[r] = xn[row_token[r]],
// while each xn row crosses HBM once instead of once per slot.  One block
// per token (grid-stride); VEC elements per 16-byte access when the row
// allows it.
template <typename V>
__global__ void __launch_bounds__(128) scatter_rows_kernel(const V* __restrict__ xn,
                                                           const int32_t* __restrict__ slot_row,
                                                           int n, int k, V* __restrict__ x_perm, int row_vecs) {
  __shared__ int32_t dst[32];
  // block (x, y): tokens x, x + gridDim.x, ..., the y-th column range of each row
  const int w = (row_vecs + (int)gridDim.y - 1) / (int)gridDim.y;
  const int ib = min(row_vecs, (int)blockIdx.y * w);
  const int ie = min(row_vecs, ib + w);
  for (int t = blockIdx.x; t < n; t += gridDim.x) {
    if (threadIdx.x < k) dst[threadIdx.x] = slot_row[(size_t)t * k + threadIdx.x];
    __syncthreads();
    const V* src = xn + (size_t)t * row_vecs;
#pragma unroll 4
    for (int i = ib + threadIdx.x; i < ie; i += blockDim.x) {
      const V v = src[i];
      for (int j = 0; j < k; ++j) {
        const int r = dst[j];
        if (r >= 0) x_perm[(size_t)r * row_vecs + i] = v;
      }
    }
    __syncthreads();
  }
}

// The same scatter with bulk copies (the copy engine moves whole rows, the
// SM only issues them).  One warp per block; lane 0 keeps kBulkRing rows of
// the block's tokens (t = blockIdx.x, + gridDim.x, ...) in flight: each row
// arrives in shared memory by one bulk load completing on that buffer's
// mbarrier, then leaves by one bulk store per kept slot, committed as one
// bulk group.  A buffer is reloaded once the
// group that read it has finished reading (wait_group.read).  Lane j < nd
// holds destination j of the next token, loaded a token ahead.  Rows must be
// 16-byte aligned and a multiple of 16 bytes.
constexpr int kBulkRing = 4;

__global__ void __launch_bounds__(32) scatter_rows_bulk_kernel(const uint8_t* __restrict__ xn,
                                                               const int32_t* __restrict__ slot_row,
                                                               int n, int k, uint8_t* __restrict__ x_perm,
                                                               uint32_t row_bytes, int32_t* __restrict__ hdr,
                                                               uint64_t wait_ns) {
  extern __shared__ __align__(128) uint8_t rows[];
  __shared__ __align__(8) uint64_t full[kBulkRing];
  const int lane = lane_id();
  const int64_t count = (n - (int64_t)blockIdx.x + gridDim.x - 1) / gridDim.x;  // this block's tokens
  if (lane == 0) {
    for (int b = 0; b < kBulkRing; ++b) mbar_init(&full[b], 1);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the copy engine sees the initialised barriers
  }
  __syncwarp();
  auto token = [&](int64_t i) { return (int64_t)blockIdx.x + i * gridDim.x; };
  auto dst_of = [&](int64_t i) -> int {  // this lane's destination of the block's i-th token, or -1
    if (i >= count || lane >= k) return -1;
    return slot_row[token(i) * k + lane];
  };
  auto load = [&](int64_t i) {
    if (lane != 0 || i >= count) return;
    const int b = (int)(i % kBulkRing);
    mbar_arrive_expect_tx(&full[b], row_bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(rows + (size_t)b * row_bytes)),
        "l"(xn + token(i) * row_bytes), "r"(row_bytes), "r"(smem_u32(&full[b]))
        : "memory");
  };
  for (int64_t i = 0; i < kBulkRing - 1; ++i) load(i);
  int d_cur = dst_of(0);
  int64_t i = 0;
  for (; i < count; ++i) {
    const int d_next = dst_of(i + 1);  // in flight while this token is handled
    const int b = (int)(i % kBulkRing);
    bool landed = true;
    if (lane == 0)
      landed = mbar_wait_bounded(&full[b], (uint32_t)((i / kBulkRing) & 1), wait_ns, nullptr, hdr, KID_SCATTER, 1);
    if (!__shfl_sync(0xffffffffu, landed, 0)) break;
    const uint32_t src = smem_u32(rows + (size_t)b * row_bytes);
    for (int j = 0; j < k; ++j) {
      const int r = __shfl_sync(0xffffffffu, d_cur, j);
      if (lane == 0 && r >= 0)
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(x_perm +
                                                                                        (size_t)r * row_bytes),
                     "r"(src), "r"(row_bytes)
                     : "memory");
    }
    if (lane == 0) {
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      // the previous token's stores have read their buffer, which the next load reuses
      asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
    }
    __syncwarp();
    load(i + kBulkRing - 1);
    d_cur = d_next;
  }
  if (lane == 0) {
    // After a failed wait, the loads still in flight land before the block
    // exits (each wait bounded; the first failure is already recorded).
    for (int64_t j = i; j < i + kBulkRing - 1 && j < count; ++j)
      mbar_wait_bounded(&full[j % kBulkRing], (uint32_t)((j / kBulkRing) & 1), wait_ns, nullptr, nullptr,
                        KID_SCATTER, 1);
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
}

}  // namespace moe

namespace moe_host {

static inline int64_t n_chunks(int64_t slots) { return (slots + moe::kChunk - 1) / moe::kChunk; }

size_t permute_hist_ints(int64_t slots, int e) { return (size_t)(n_chunks(slots) > 0 ? n_chunks(slots) : 1) * e; }

moe_status launch_permute(const int32_t* topk_idx, int n, int k, int e, int cap, int32_t* hist,
                          int32_t* offsets, int32_t* slot_row, int32_t* row_token, cudaStream_t s,
                          int32_t* offsets_ext, int extra, int32_t* counts) {
  const int64_t slots = (int64_t)n * k;
  const int64_t nch = n_chunks(slots);
  if (nch == 0) {
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (e + 1), s) != cudaSuccess) return MOE_ERR_CUDA;
    // no slots means no tokens, so the trailing group is empty too (extra == 0)
    if (offsets_ext != nullptr && cudaMemsetAsync(offsets_ext, 0, sizeof(int32_t) * (e + 2), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (counts != nullptr && cudaMemsetAsync(counts, 0, sizeof(int32_t) * e, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  // one block for small batches: histogram and running counts in shared memory
  const size_t fused_smem = sizeof(int32_t) * (size_t)e * (size_t)(nch + 32);
  if (nch <= 32 && fused_smem <= 96 * 1024) {
    static SmemLimit lim;
    const moe_status st = ensure_smem_limit(moe::permute_fused_kernel, 96 * 1024, lim);
    if (st != MOE_OK) return st;
    moe::permute_fused_kernel<<<1, 1024, fused_smem, s>>>(topk_idx, slots, k, e, (int)nch, cap, offsets, offsets_ext,
                                                          extra, counts, slot_row, row_token);
    return launch_status();
  }
  const int blocks = (int)((nch + moe::kPermWarps - 1) / moe::kPermWarps);
  const size_t smem = sizeof(int32_t) * e * moe::kPermWarps;
  moe::chunk_hist_kernel<<<blocks, moe::kPermWarps * 32, smem, s>>>(topk_idx, slots, e, (int)nch, hist);
  moe::hist_scan_kernel<<<1, 1024, 0, s>>>(hist, e, (int)nch, cap, offsets, offsets_ext, extra, counts);
  moe::chunk_scatter_kernel<<<blocks, moe::kPermWarps * 32, smem, s>>>(topk_idx, slots, k, e, (int)nch, cap,
                                                                       hist, offsets, slot_row, row_token);
  return launch_status();
}

moe_status launch_gather(int dtype, const void* xn, const int32_t* slot_row, int n, int k, void* x_perm, int d,
                         cudaStream_t s, int32_t* hdr) {
  if (n == 0) return MOE_OK;
  if (k > 32) return MOE_ERR_UNSUPPORTED;
  const size_t row_bytes = (size_t)d * (dtype == MOE_BF16 ? 2 : 4);
  const uintptr_t addr = (uintptr_t)xn | (uintptr_t)x_perm;
  // Bulk copies once there are enough tokens to keep every SM's copies busy
  // (the block-per-token kernel below splits rows over blocks for fewer).
  const size_t bulk_smem = moe::kBulkRing * row_bytes;
  if (row_bytes % 16 == 0 && addr % 16 == 0 && n >= 2 * sm_count() && bulk_smem <= 192 * 1024) {
    static SmemLimit lim;
    const moe_status st = ensure_smem_limit(moe::scatter_rows_bulk_kernel, 192 * 1024, lim);
    if (st != MOE_OK) return st;
    const int per_sm = (int)std::max<size_t>(1, (160 * 1024) / bulk_smem);
    const int grid = (int)std::min<int64_t>(n, (int64_t)sm_count() * std::min(per_sm, 8));
    moe::scatter_rows_bulk_kernel<<<grid, 32, bulk_smem, s>>>((const uint8_t*)xn, slot_row, n, k, (uint8_t*)x_perm,
                                                             (uint32_t)row_bytes, hdr, wait_limit_ns());
    return launch_status();
  }
  // columns counted in 16-byte vectors, or elements for the narrower forms
  const int vec_elems = (row_bytes % 16 == 0 && addr % 16 == 0) ? (dtype == MOE_BF16 ? 8 : 4) : 1;
  const dim3 grid = row_split_grid(n, d, vec_elems);
  if (row_bytes % 16 == 0 && addr % 16 == 0)
    moe::scatter_rows_kernel<uint4><<<grid, 128, 0, s>>>((const uint4*)xn, slot_row, n, k,
                                                         (uint4*)x_perm, (int)(row_bytes / 16));
  else if (row_bytes % 4 == 0 && addr % 4 == 0)
    moe::scatter_rows_kernel<uint32_t><<<grid, 128, 0, s>>>((const uint32_t*)xn, slot_row, n, k,
                                                            (uint32_t*)x_perm, (int)(row_bytes / 4));
  else
    moe::scatter_rows_kernel<uint16_t><<<grid, 128, 0, s>>>((const uint16_t*)xn, slot_row, n, k,
                                                            (uint16_t*)x_perm, (int)(row_bytes / 2));
  return launch_status();
}

}  // namespace moe_host
