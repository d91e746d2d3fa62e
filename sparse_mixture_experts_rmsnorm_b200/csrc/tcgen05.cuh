// tcgen05 / TMA building blocks shared by the grouped GEMM kernels
// (single-SM tiles in gemm_tc.cu, SM-pair tiles in gemm_tc2.cu): argument
// block, PTX wrappers, shared-memory and instruction descriptors, the TMEM
// load, the work schedule and the epilogue of one accumulator row.
#pragma once

#include <cuda.h>

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

constexpr int TC_BK = 64;  // k-block: 128 bytes of bf16, one 128-byte swizzle row
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
  int shared_group;  // group whose weights come from the second map pair (-1: none)
  int shared_a;      // 1: that group's A rows come from their own map, from row 0
  int narrow;        // 1: 128-column tiles (one B box, N = 128), plain epilogues only
  int tma_store;     // 1: the plain-store epilogue writes whole warps' blocks through TMA
  // Tiling picked on the device from the group sizes (both kernels are
  // launched; the one not picked returns at once): 0 = always run,
  // 1 = run if single-SM tiles are picked, 2 = run if SM-pair tiles are.
  int pick;
  int pick_pairs;    // SM pairs resident for the pair kernel
  int pick_ctas;     // CTAs of the single-SM kernel
};

// The device-side tiling choice of the plain-store epilogue (down
// projection): with persistent CTAs taking tiles in turn, a launch lasts
// about ceil(tiles / workers) tile times; an SM-pair tile does one SM's
// share of work about 3 % faster than a single-SM tile (measured on B200),
// so pairs are picked when 97 * their waves <= 100 * the single-SM waves.
// Called by one whole warp; every lane returns the same answer.
__device__ __forceinline__ bool pairs_picked(const int* offs, int groups, int n_tiles, int pairs, int ctas) {
  int tp = 0, ts = 0;
  for (int g = lane_id(); g < groups; g += 32) {
    const int m = offs[g + 1] - offs[g];
    tp += (m + 255) / 256;
    ts += (m + 127) / 128;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tp += __shfl_xor_sync(0xffffffffu, tp, o);
    ts += __shfl_xor_sync(0xffffffffu, ts, o);
  }
  const long wp = ((long)tp * n_tiles + pairs - 1) / pairs;
  const long wsg = ((long)ts * n_tiles + ctas - 1) / ctas;
  return 97 * wp <= 100 * wsg;
}

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

// TMA store of one box from shared memory (bulk-group completion), and the
// bulk-group waits that guard the shared-memory buffer and the global writes.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// generic-proxy writes to shared memory become visible to the TMA (async proxy)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
// Tiles of BM rows; a group of r rows has ceil(r / BM) m-tiles and n_tiles
// n-tiles; prefix[g] is the first tile of group g.
struct Tile {
  int group, row0, row_end, n0;
};

template <int BM>
__device__ __forceinline__ void build_prefix(const int* offs, int* prefix, int groups, int n_tiles) {
  // one warp: exclusive scan of the tile counts
  const int lane = lane_id();
  int carry = 0;
  for (int base = 0; base < groups; base += 32) {
    const int g = base + lane;
    const int v = (g < groups) ? ((offs[g + 1] - offs[g] + BM - 1) / BM) * n_tiles : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (g < groups) prefix[g] = carry + x - v;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) prefix[groups] = carry;
}

template <int BM>
__device__ __forceinline__ Tile decode_tile(int t, const int* prefix, const int* offs, int groups, int out_cols) {
  int lo = 0, hi = groups - 1;  // last g with prefix[g] <= t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int rows = offs[g + 1] - offs[g];
  const int mt = (rows + BM - 1) / BM;
  const int local = t - prefix[g];
  Tile tl;
  tl.group = g;
  tl.row0 = offs[g] + (local % mt) * BM;
  tl.row_end = offs[g + 1];
  tl.n0 = (local / mt) * out_cols;
  return tl;
}

// ---- plain-store epilogue of one warp's 32 rows through TMA --------------------
// The warp's 32 rows (lane = row) of `ncols` accumulator columns go out in
// blocks of 32 rows x 64 bf16 columns: each lane converts and writes its 128
// bytes into `stage` (4 KiB, 1024-byte aligned) in the 128-byte-swizzled
// layout (16-byte chunk j of row r at chunk j ^ (r % 8)), and lane 0 stores
// the block with one TMA box at (n0 + c, row0).  Columns past the tensor are
// clipped by the TMA.  All 32 lanes must call it.
__device__ __forceinline__ void epilogue_warp_store_tma(const CUtensorMap* map_c, uint32_t tbase, uint32_t stage,
                                                        int row0, int n0, int ncols) {
  const int lane = lane_id();
  const uint32_t my_row = stage + (uint32_t)lane * 128u;
#pragma unroll 1
  for (int c = 0; c < ncols; c += 64) {
    uint32_t a[32], b[32];
    MOE_TMEM_LD32(tbase + c, a);
    MOE_TMEM_LD32(tbase + c + 32, b);
    tmem_wait_ld();
    if (lane == 0) bulk_wait_read_all();  // the previous block has left the stage
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t* v = j < 4 ? a + 8 * j : b + 8 * (j - 4);
      const uint32_t p0 = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
      const uint32_t p1 = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
      const uint32_t p2 = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
      const uint32_t p3 = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
      const uint32_t dst = my_row + ((uint32_t)(j ^ (lane & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(p0), "r"(p1), "r"(p2), "r"(p3)
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(map_c, stage, n0 + c, row0);
      bulk_commit();
    }
  }
}

// ---- epilogue of one accumulator row -----------------------------------------
// The calling thread owns TMEM lane `tbase` (row `row` of the output) and
// drains 256 accumulator columns starting at tbase's column:
//   EPI_SWIGLU: columns c and 128 + c are the gate and up halves of hidden
//               unit n0 + c; writes silu(gate) * up for 128 units;
//   EPI_STORE / EPI_F32: writes `ncols` (256 or 128) columns n0 .. n0 + ncols - 1.
// Stores are masked to row_ok and to columns < nout.  All 32 lanes of the
// warp must call it (tcgen05.ld is warp-wide).
template <int EPI>
__device__ __forceinline__ void epilogue_row(const TcArgs& args, uint32_t tbase, int row, bool row_ok, int n0,
                                             int ncols = 256) {
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
      if (row_ok) store_row32_bf16(out, n0 + c, args.nout, (args.ldc & 7) == 0, v);
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < ncols; c += 32) {
      uint32_t a[32];
      MOE_TMEM_LD32(tbase + c, a);
      tmem_wait_ld();
      const int col = n0 + c;
      if (!row_ok) continue;
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

}  // namespace moe

namespace moe_host {
// 2-D bf16 tensor map over a row-major [rows][k] matrix: box 128 rows x 64
// columns, 128-byte swizzle, zero fill outside the matrix.
bool make_tc_map(CUtensorMap* m, const void* base, int64_t rows, int k);
// The same with a box of `box_rows` rows (8 .. 256) x 64 columns.
bool make_tc_map_rows(CUtensorMap* m, const void* base, int64_t rows, int k, int box_rows);
// 2-D bf16 tensor map over the [rows][ldc] output (cols used), box 32 rows x 64
// columns, 128-byte swizzle: the TMA-store epilogue's map.
bool make_store_map(CUtensorMap* m, void* base, int64_t rows, int cols, int ldc);

// The SM-pair kernel (gemm_tc2.cu) on maps and arguments prepared by
// launch_gemm_tc; groups_bound = groups when offsets are given, else 0.
moe_status launch_gemm_tc2(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                           const CUtensorMap& msb, const CUtensorMap& msb2, const CUtensorMap& msa,
                           const CUtensorMap& mc, const moe::TcArgs& args, int64_t max_rows, int groups_bound,
                           cudaStream_t s);

// The swapped-operand SM-pair kernel (gemm_swap.cu), same arguments as
// launch_gemm_tc; SwiGLU and plain-store epilogues, bf16 only, for the shapes
// swap_supported accepts (K a positive multiple of 64, nout and ldc multiples of 8).
bool swap_supported(int epi, int nout, int k, int ldc);
moe_status launch_gemm_swap(int epi, const void* a, const void* b, const void* b2, const int32_t* offsets,
                            int groups, int max_rows, int nout, int k, void* c, int ldc, int32_t* hdr,
                            cudaStream_t s, const void* sb, const void* sb2, const void* sa, int sa_rows);

// SM pairs that launch_gemm_tc2 launches for these sizes.
int64_t tc2_pairs_launched(int epi, int64_t max_rows, int groups_bound, int n_tiles);

// 0: choose per launch: the swapped-operand SM-pair kernel, where it supports
//    the shape, for every grouped SwiGLU launch and for the grouped plain store
//    of groups averaging >= 64 rows; otherwise single-SM tiles, except that a
//    plain store averaging >= 512 rows a group takes SM-pair tiles (when
//    grouped, both kernels are launched and the device picks from the group
//    sizes, pairs_picked);
// 1: single-SM tiles only; 2: SM-pair tiles only; 3: the swapped-operand
//    kernel for the expert GEMMs it supports (the rest take 0's choice).
// The fp32 logits (the router) always take single-SM tiles (128 or 256
// columns) with K-chunked accumulation, whatever the mode.
void set_tc_pairing(int mode);
int tc_pairing();
}  // namespace moe_host
