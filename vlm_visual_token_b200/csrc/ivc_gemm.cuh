// ivc_gemm.cuh — the connector / projection GEMM for sm_100a.
//
//   out[m, n] = epilogue( sum_k A[m, k] * B[n, k] )      (B = nn.Linear weight [N, K])
//
// Persistent, warp-specialised tcgen05 kernel. Each CTA loops over output
// tiles of 128 x BN (static round-robin over tile index, n fastest). TMA
// streams 128 x 64 A tiles and BN x 64 B tiles (128-byte swizzle) through a
// STAGES-deep shared-memory ring; one thread issues tcgen05.mma (M=128, N=BN,
// K=16) into one of two TMEM accumulators; four epilogue warps drain the other
// accumulator with tcgen05.ld, apply the fused epilogue (LayerNorm fold or
// bias, optional GELU) and store bf16 or fp32, so a tile's epilogue overlaps
// the next tile's mainloop.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
//
// CG = 2 runs the same roles on a CTA pair (a cluster of 2) with
// tcgen05.mma.cta_group::2: the pair computes 256 x BN tiles, each CTA loads
// its own 128 rows of A and BN/2 rows of B into its own shared memory (TMA
// transaction bytes complete on the leader's barrier), the leader issues the
// MMAs and commits them to both CTAs' barriers, and each CTA drains its own
// 128 accumulator rows from its TMEM. Per SM this halves the B traffic into
// shared memory. No load uses cluster multicast.
//
// A operand. pixel_shuffle ("Pixel Shuffle 源码逐行解析" of the
// InternVL3-14B-Instruct connector article; table "三档 Token 规模" of the
// InternVL3_5-2B-Flash article) is not materialised: the GEMM row of
// token (tile, a, b) and the column block of grid offset (di, dj) are
// addressed directly in the [T, 32, 32, C] feature tensor through a 5-D TMA
// tensor map, so every A tile is one TMA box:
//   PS_HALF    (factor 0.5):  dims {C, dj:2, b:16, di:2, tile*16+a}, box {64,1,16,1,8}
//   PS_QUARTER (factor 0.25): dims {C, r:4, b:8, q:4, tile*8+a},     box {64,1,8,1,16}
// Column m of the shuffled row is (block*C + c) with block = 2di+dj
// (4q+r for the quarter), so k-step kk loads block kk/(C/64), channels
// 64*(kk%(C/64)).. of each of the 128 tokens of the tile.
//
// B operand. K-major (nn.Linear weights, 2-D or batched 3-D with the batch
// chosen by the tile's row: batch = m0 / b_batch_rows), or MN-major batched
// 3-D (B[n, k] stored with n contiguous, e.g. a [tokens, channels] feature
// block used as B = X^T): then each stage holds BN/64 boxes of 64 k-rows x
// 64 n-columns and the UMMA descriptor walks them MN-major.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ivc_ptx.cuh"

namespace ivc {

enum AMode : int { A_PLAIN = 0, A_PS_HALF = 1, A_PS_QUARTER = 2, A_PS_QUARTER_TWICE = 3 };
enum BMode : int { B_K2D = 0, B_K3D = 1, B_MN3D = 2 };
enum EpiMode : int { EPI_BIAS = 0, EPI_LNFOLD = 1 };

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_MAX_GROUPS = 8;
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_EPI_BAR = 1;  // named barrier of the 4 epilogue warps

struct alignas(64) GemmMaps {
  CUtensorMap a;
  CUtensorMap b[GEMM_MAX_GROUPS];
};

struct GemmArgs {
  int M, N, K;
  int groups;                    // blockIdx-independent group count (tile index space)
  int a_mode;
  int b_mode;
  int b_batch_rows;              // B_K3D / B_MN3D: rows of A per B batch
  int c_blocks;                  // C / 64 for the pixel_shuffle modes
  int b_prefetch;                // >0: prefetch B (K2D) this many k-steps ahead into L2
  int epi_mode;
  int gelu;
  int remap;                     // 0: none; 1: transpose 16x16 token grid; 2: 8x8
  int out_f32;                   // 1: store fp32 instead of bf16
  int m_valid;                   // >0: store only rows with (row % 128) < m_valid
  void* out;
  long long ldo;                 // elements
  int group_col_stride;          // output column offset per group
  const __nv_bfloat16* bias[GEMM_MAX_GROUPS];  // EPI_BIAS, per group (may be null)
  const float* colsum;           // EPI_LNFOLD
  const float* fbias;            // EPI_LNFOLD
  const float* row_mean;         // EPI_LNFOLD
  const float* row_rstd;         // EPI_LNFOLD
  // Routed rows (router-first flow). With list_count set, the row count is
  // *list_count * item_rows (read on the device, at most M): the rows of the
  // listed tiles in list order. The pixel_shuffle A modes then address tile
  // list[row / item_rows]; stats_remap reads the LN statistics of that tile's
  // row; out_base (if set) stores row r at out_base[r / item_rows] + r % item_rows
  // (after the v1 remap inside the tile) instead of at r.
  const int* list;
  const int* list_count;
  const int* out_base;
  int item_rows;
  int stats_remap;
  // Split-K of the last round (split_max > 1). The output tiles that fill
  // whole rounds of the persistent grid run unsplit; the rem < units tiles
  // left for the last round are each cut into S = min(split_max, units / rem,
  // KT / 4) k-slices, so that round keeps every CTA busy. A slice unit stores
  // its raw fp32 tile at split_part[((tail tile) * S + slice)][TILE_M][BN];
  // splitk_epilogue_kernel sums the slices and applies the epilogue. CTA 0
  // writes split_s[0..2] = {S, first split tile, split tiles}.
  int split_max;
  int split_min;
  float* split_part;
  int* split_s;
  // A and B are not written by the previous kernel in the stream (only the
  // epilogue's inputs may be): only the epilogue warps wait for it, the
  // mainloop starts as soon as the CTA is resident
  int epi_dep_only;
};

// Number of k-slices for `tiles` output tiles on `units` CTAs (or pairs).
// The split-K scratch holds units x TILE_M x BN values: S * tiles <= units.
// Fewer than split_min slices do not pay for the partial traffic and the
// finishing launch (measured on the connector GEMMs: 4 for 256-wide tiles,
// 2 for the 512-wide ones, which exist to be split).
__host__ __device__ __forceinline__ int split_count(int split_max, int units, int tiles, int KT,
                                                    int split_min = 4) {
  if (split_max <= 1 || tiles <= 0) return 1;
  int s = units / tiles;
  if (s > split_max) s = split_max;
  if (s > KT / 4) s = KT / 4;  // at least 4 k-steps per slice
  return s < split_min ? 1 : s;
}

// Output column of TMEM column c. A 512-wide pair tile is two N = 256 pair
// MMAs; CTA r of the pair holds weight rows [256 r, 256 r + 256) of the tile,
// and MMA m reads rows [128 m, 128 m + 128) of both CTAs' blocks, so TMEM
// column 256 m + 128 h + i is output column 128 m + 256 h + i.
template <int BN>
__host__ __device__ __forceinline__ int tmem_col_to_n(int c) {
  if constexpr (BN > 256) {
    const int m = c >> 8, h = (c >> 7) & 1, i = c & 127;
    return 128 * m + 256 * h + i;
  } else {
    return c;
  }
}

template <int BN, int STAGES, int CG = 1>
struct GemmSmem {
  static constexpr uint32_t A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr uint32_t B_ROWS = BN / CG;  // rows of B this CTA loads
  static constexpr uint32_t B_BYTES = B_ROWS * GEMM_BK * 2;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  static constexpr uint32_t RING = STAGES * STAGE;
  static constexpr uint32_t BARS = (2 * STAGES + 4) * 8 + 16;
  static constexpr uint32_t COLS = 2 * BN * 4;
  static constexpr uint32_t TOTAL = 1024 + RING + BARS + COLS;
  // double-buffered accumulator, except for 512-wide pair tiles, whose one
  // accumulator fills the 512 columns of TMEM
  static constexpr int ACC_BUFS = BN > 256 ? 1 : 2;
  static constexpr uint32_t TMEM_COLS = ACC_BUFS * BN;
};

__device__ __forceinline__ float gelu_erf(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync %0, 128;" ::"n"(GEMM_EPI_BAR) : "memory");
}

// Tile index -> (group, m-tile, n-tile), n fastest.
struct TileCoord {
  int g, m0, n0;
};
__device__ __forceinline__ TileCoord tile_coord(int idx, int m_tiles, int n_tiles, int tile_m,
                                                int BN) {
  const int n = idx % n_tiles;
  const int rest = idx / n_tiles;
  const int m = rest % m_tiles;
  return {rest / m_tiles, m * tile_m, n * BN};
}

template <int BN, int STAGES, int CG>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_sm100_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args,
                      int* __restrict__ status) {
  using L = GemmSmem<BN, STAGES, CG>;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 512, "BN");
  static_assert(CG == 1 ? BN <= 256 : (BN == 256 || BN == 512),
                "CTA pairs use 256- or 512-wide tiles, single CTAs up to 256");
  constexpr int TILE_M = GEMM_BM * CG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::RING);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;   // [2] accumulator ready
  uint64_t* tempty_bar = tfull_bar + 2;       // [2] accumulator drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + 2);
  float* s_col0 = reinterpret_cast<float*>(smem + L::RING + L::BARS);
  float* s_col1 = s_col0 + BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = CG == 2 ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit = blockIdx.x / CG;     // this CTA (pair) in the persistent grid
  const int n_units = gridDim.x / CG;
  const int n_tiles = (args.N + BN - 1) / BN;
  const int KT = args.K / GEMM_BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4 * CG);  // one arrival per epilogue warp of the group
    }
    fence_mbar_init();
    tma_prefetch_desc(&maps.a);
    for (int g = 0; g < args.groups; ++g) tma_prefetch_desc(&maps.b[g]);
  }
  if constexpr (CG == 2) cluster_sync();  // peer barriers initialised before any remote use
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, L::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;
  // operands and outputs may belong to the previous kernel in the stream
  if (!args.epi_dep_only || warp >= 2) pdl_wait();
  pdl_trigger();
  int M = args.M;
  if (args.list_count != nullptr) {
    const int c = *args.list_count;
    const long long rows = static_cast<long long>(c < 0 ? 0 : c) * args.item_rows;
    M = rows < M ? static_cast<int>(rows) : M;
  }
  const int m_tiles = (M + TILE_M - 1) / TILE_M;
  const int n_out = m_tiles * n_tiles * args.groups;  // output tiles
  const int rem = n_out % n_units;
  const int S = rem > 0 ? split_count(args.split_max, n_units, rem, KT, args.split_min) : 1;
  const int n_full = S > 1 ? n_out - rem : n_out;     // tiles computed whole
  const int n_total = n_full + (n_out - n_full) * S;  // work units
  const int n_listed = args.list_count != nullptr ? M / args.item_rows : 0;
  if (args.split_s != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    args.split_s[0] = S;
    args.split_s[1] = n_full;
    args.split_s[2] = n_out - n_full;
  }
  // work unit -> output tile and k-block range [kb0, kb1); slice < 0: whole tile
  auto unit_of = [&](int idx, int& tile, int& slice, int& kb0, int& kb1) {
    if (idx < n_full) {
      tile = idx;
      slice = -1;
      kb0 = 0;
      kb1 = KT;
    } else {
      const int j = idx - n_full;
      tile = n_full + j / S;
      slice = j % S;
      kb0 = slice * KT / S;
      kb1 = (slice + 1) * KT / S;
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int it = 0;
      for (int idx = unit; idx < n_total && ok; idx += n_units) {
        int tile, slice, kb0, kb1;
        unit_of(idx, tile, slice, kb0, kb1);
        const TileCoord tc = tile_coord(tile, m_tiles, n_tiles, TILE_M, BN);
        const int my_m0 = tc.m0 + GEMM_BM * rank;
        const int my_n0 = tc.n0 + static_cast<int>(L::B_ROWS) * rank;
        const int bb = args.b_batch_rows > 0 ? tc.m0 / args.b_batch_rows : 0;
        if (args.b_prefetch > 0 && args.b_mode == B_K2D) {
          for (int kk = kb0; kk < kb0 + args.b_prefetch && kk < kb1; ++kk)
            tma_prefetch_2d(&maps.b[tc.g], kk * GEMM_BK, my_n0);
        }
        for (int kk = kb0; kk < kb1; ++kk, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (args.b_prefetch > 0 && args.b_mode == B_K2D && kk + args.b_prefetch < kb1)
            tma_prefetch_2d(&maps.b[tc.g], (kk + args.b_prefetch) * GEMM_BK, my_n0);
          if (!mbar_wait(&empty_bar[s], ph ^ 1)) { ok = false; break; }
          // the leader's barrier counts the bytes of both CTAs of a pair
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], L::STAGE * CG);
          uint8_t* a_dst = ring + s * L::STAGE;
          uint8_t* b_dst = a_dst + L::A_BYTES;
          int ac[5];
          int a_rank = 2;
          int ac4b = -1;  // routed factor 0.25: outer coordinate of the second 64-row box
          if (args.a_mode == A_PLAIN) {
            ac[0] = kk * GEMM_BK;
            ac[1] = my_m0;
          } else {
            const int blk = kk / args.c_blocks;
            const int c0 = (kk - blk * args.c_blocks) * GEMM_BK;
            a_rank = 5;
            if (args.a_mode == A_PS_HALF) {
              ac[0] = c0; ac[1] = blk & 1; ac[2] = 0; ac[3] = blk >> 1; ac[4] = my_m0 >> 4;
              if (args.list != nullptr)  // 128 rows = half of listed tile my_m0 / 256
                ac[4] = args.list[my_m0 >> 8] * 16 + ((my_m0 >> 4) & 15);
            } else {
              int q, r;
              if (args.a_mode == A_PS_QUARTER) {
                q = blk >> 2;
                r = blk & 3;
              } else {  // two successive factor-0.5 shuffles: blk = 8ei + 4ej + 2di + dj
                q = 2 * (blk >> 3) + ((blk >> 1) & 1);
                r = 2 * ((blk >> 2) & 1) + (blk & 1);
              }
              ac[0] = c0; ac[1] = r; ac[2] = 0; ac[3] = q; ac[4] = my_m0 >> 3;
              if (args.list != nullptr) {
                // 128 rows = listed tiles j and j + 1 (64 rows each, one box
                // apiece); past the last one, j again (rows >= M, not stored)
                const int j = my_m0 >> 6;
                ac[4] = args.list[j < n_listed ? j : (n_listed > 0 ? n_listed - 1 : 0)] * 8;
                ac4b = args.list[j + 1 < n_listed ? j + 1 : (n_listed > 0 ? n_listed - 1 : 0)] * 8;
              }
            }
          }
          if constexpr (CG == 2) {
            const uint32_t lb = pair_leader_addr(&full_bar[s]);
            if (a_rank == 2) {
              tma_load_2d_pair(a_dst, &maps.a, lb, ac[0], ac[1]);
            } else {
              tma_load_5d_pair(a_dst, &maps.a, lb, ac[0], ac[1], ac[2], ac[3], ac[4]);
              if (ac4b >= 0)
                tma_load_5d_pair(a_dst + L::A_BYTES / 2, &maps.a, lb, ac[0], ac[1], ac[2], ac[3],
                                 ac4b);
            }
            tma_load_2d_pair(b_dst, &maps.b[tc.g], lb, kk * GEMM_BK, my_n0);
            continue;
          }
          if (a_rank == 2) {
            tma_load_2d(a_dst, &maps.a, &full_bar[s], ac[0], ac[1]);
          } else {
            tma_load_5d(a_dst, &maps.a, &full_bar[s], ac[0], ac[1], ac[2], ac[3], ac[4]);
            if (ac4b >= 0)
              tma_load_5d(a_dst + L::A_BYTES / 2, &maps.a, &full_bar[s], ac[0], ac[1], ac[2], ac[3],
                          ac4b);
          }
          const CUtensorMap* bm = &maps.b[tc.g];
          if (args.b_mode == B_K2D) {
            tma_load_2d(b_dst, bm, &full_bar[s], kk * GEMM_BK, tc.n0);
          } else if (args.b_mode == B_K3D) {
            tma_load_3d(b_dst, bm, &full_bar[s], kk * GEMM_BK, tc.n0, bb);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_3d(b_dst + j * (64 * GEMM_BK * 2), bm, &full_bar[s], tc.n0 + 64 * j,
                          kk * GEMM_BK, bb);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr int MMA_N = BN > 256 ? 256 : BN;
      const uint32_t idesc = idesc_bf16_f32(TILE_M, MMA_N) |
                             (args.b_mode == B_MN3D ? (1u << 16) : 0u);  // B MN-major
      int it = 0, local = 0;
      for (int idx = unit; idx < n_total && ok; idx += n_units, ++local) {
        const int acc = local % L::ACC_BUFS;
        const uint32_t use = static_cast<uint32_t>(local / L::ACC_BUFS);
        int tile, slice, kb0, kb1;
        unit_of(idx, tile, slice, kb0, kb1);
        if (!mbar_wait(&tempty_bar[acc], (use & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kk = kb0; kk < kb1; ++kk, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&full_bar[s], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(ring + s * L::STAGE);
          const uint64_t ad = sw128_kmajor_desc(a_addr);
          const uint64_t bd = args.b_mode == B_MN3D
                                  ? sw128_mnmajor_desc(a_addr + L::A_BYTES, 64 * GEMM_BK * 2)
                                  : sw128_kmajor_desc(a_addr + L::A_BYTES);
          const uint64_t bstep = args.b_mode == B_MN3D ? (16 * 128) >> 4 : 2;
#pragma unroll
          for (int k = 0; k < GEMM_BK / 16; ++k) {
            // K-major: advance 16 bf16 = 32 bytes inside the swizzle atom;
            // MN-major: advance 16 k-rows of 128 bytes.
            const uint32_t accum = (kk != kb0 || k != 0) ? 1u : 0u;
            if constexpr (CG == 2) {
              umma_bf16_pair(d_tmem, ad + 2 * k, bd + bstep * k, idesc, accum);
              if constexpr (BN > 256)  // rows 128..255 of each CTA's weight block (+16 KB)
                umma_bf16_pair(d_tmem + 256, ad + 2 * k, bd + ((128 * 128) >> 4) + bstep * k,
                               idesc, accum);
            } else {
              umma_bf16(d_tmem, ad + 2 * k, bd + bstep * k, idesc, accum);
            }
          }
          if constexpr (CG == 2)
            umma_commit_pair(&empty_bar[s]);
          else
            umma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        if constexpr (CG == 2)
          umma_commit_pair(&tfull_bar[acc]);
        else
          umma_commit(&tfull_bar[acc]);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127
    int local = 0;
    for (int idx = unit; idx < n_total; idx += n_units, ++local) {
      int tile, slice, kb0, kb1;
      unit_of(idx, tile, slice, kb0, kb1);
      const TileCoord tc = tile_coord(tile, m_tiles, n_tiles, TILE_M, BN);
      const int acc = local % L::ACC_BUFS;
      const uint32_t use = static_cast<uint32_t>(local / L::ACC_BUFS);
      // per-column epilogue vectors of this tile, by TMEM column
      epi_bar_sync();
      for (int i = et; i < BN; i += 128) {
        const int n = tc.n0 + tmem_col_to_n<BN>(i);
        float c0 = 0.f, c1 = 0.f;
        if (n < args.N) {
          if (args.epi_mode == EPI_LNFOLD) {
            c0 = args.colsum[n];
            c1 = args.fbias[n];
          } else if (args.bias[tc.g] != nullptr) {
            c1 = __bfloat162float(args.bias[tc.g][n]);
          }
        }
        s_col0[i] = c0;
        s_col1[i] = c1;
      }
      epi_bar_sync();
      // After a timed-out wait the warp keeps looping (the named barrier above
      // counts all four epilogue warps every tile) but does no more work.
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], use & 1));
      if (!ok) continue;
      tc_fence_after();
      const int row = tc.m0 + GEMM_BM * rank + quad * 32 + lane;
      float mean = 0.f, rstd = 1.f;
      if (args.epi_mode == EPI_LNFOLD && row < M) {
        const int sr = args.stats_remap
                           ? args.list[row / args.item_rows] * args.item_rows + row % args.item_rows
                           : row;
        mean = args.row_mean[sr];
        rstd = args.row_rstd[sr];
      }
      const float nms = -mean * rstd;
      long long out_row = row;
      if (args.remap == 1) {
        const int t = row & 255;
        out_row = (row & ~255) | ((t & 15) << 4) | (t >> 4);
      } else if (args.remap == 2) {
        const int t = row & 63;
        out_row = (row & ~63) | ((t & 7) << 3) | (t >> 3);
      }
      if (args.out_base != nullptr && row < M)  // item_rows is 256 / 64, as the remaps
        out_row = args.out_base[row / args.item_rows] + out_row % args.item_rows;
      const long long out_off =
          out_row * args.ldo + static_cast<long long>(tc.g) * args.group_col_stride + tc.n0;
      const uint32_t t_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                              static_cast<uint32_t>(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        const int cn = tmem_col_to_n<BN>(c);  // output column of this 32-column chunk
        uint32_t r[32];
        tmem_ld32(t_base + c, r);
        tmem_ld_wait();
        if (c + 32 == BN) {
          // accumulator fully read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (CG == 2)
              mbar_arrive_cluster(pair_leader_addr(&tempty_bar[acc]));
            else
              mbar_arrive(&tempty_bar[acc]);
          }
        }
        if (slice >= 0) {
          // raw sums of this k-slice (the whole TILE_M x BN tile, in bounds
          // of its slot); splitk_epilogue_kernel finishes the tile
          float4* dst = reinterpret_cast<float4*>(
              args.split_part +
              ((static_cast<long long>(tile - n_full) * S + slice) * TILE_M + (row - tc.m0)) * BN +
              cn);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          continue;
        }
        if (row < M && tc.n0 + cn < args.N && (args.m_valid == 0 || (row & 127) < args.m_valid)) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float t = __uint_as_float(r[i]);
            if (args.epi_mode == EPI_LNFOLD)
              t = fmaf(rstd, t, nms * s_col0[c + i]) + s_col1[c + i];
            else
              t += s_col1[c + i];
            v[i] = args.gelu ? gelu_erf(t) : t;
          }
          if (args.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.out) + out_off + cn);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + out_off + cn);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                                  pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                  pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                  pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          }
        }
      }
    }
  }

  if (!ok && status != nullptr) atomicOr(status, 4 /* IVC_DEV_WAIT_TIMEOUT */);
  tc_fence_before();
  __syncthreads();
  // a pair stays resident until neither CTA touches the other's barriers
  if constexpr (CG == 2) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2)
      tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

}  // namespace ivc
