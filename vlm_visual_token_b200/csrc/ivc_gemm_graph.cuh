// ivc_gemm_graph.cuh — several connector Linears in one persistent launch.
//
// The connector's Linears are small next to the GPU: on one 13-tile image
// (InternVL3_5-2B-Flash dims) mlp2's first Linear has 64 output tiles of
// 256 x 256, its second and third 32 each, and mlp1's 104 and 104. Launched
// one after another, each leaves SMs idle in its last round and in the gap to
// the next launch, and the 32-tile launches fill only half the GPU. Here one
// persistent launch runs every Linear of both MLPs ("problems"): a CTA pair
// works through a list of output tiles drawn from all problems, and a tile of
// a problem that reads another problem's output (fc2 reads fc1's hidden rows)
// starts as soon as that problem's 256-row block is complete, not when the
// whole previous Linear is.
//
// Row-block counters in global memory carry the dependency. After a CTA has
// stored its 128 rows of a tile, one epilogue thread makes the stores visible
// at GPU scope and increments done[problem][row block] (each CTA of the pair
// once, so a block is complete at 2 * n_tiles). A producer thread that needs
// the block polls the counter with acquire loads (bounded: after about a
// second it gives up and sets the status word), then orders its following
// TMA (async-proxy) reads after them with a proxy fence.
//
// Each pair's tile list is either a host-computed list schedule carried in
// the launch arguments (small problems, where the order decides how full the
// GPU stays) or a round-robin over the tiles in problem order. Both are
// deadlock-free: every list is in increasing global order, and a tile only
// waits for tiles earlier in that order, so the earliest unfinished tile can
// always run.
//
// Tiles are 256 x 256 on CTA pairs (tcgen05.mma.cta_group::2), two TMEM
// accumulators so that a tile's epilogue overlaps the next tile's mainloop:
// the roles and the epilogue of gemm_sm100_kernel (ivc_gemm.cuh), with the
// problem's own A view, weights and epilogue. Operands are staged two k-blocks
// (128 channels) at a time: every TMA request is one 32 KB box, A or B, 128
// rows x 2 chunks of 64 channels, the chunk being the outermost box dimension
// so that each chunk lands as its own 128-row, 128-byte-swizzled block. On
// B200 one such request per operand streams about twice as fast per SM as
// two 16 KB requests (measured with all SMs loading, A and B together: ~175
// against ~90 GB/s per SM). The ring holds six 32 KB boxes: three stages of
// an A and a B box, one full and one empty barrier per stage.
//
// A "wide" problem has 256 x 512 tiles: per stage one A box and two B boxes
// (the two 256-column halves, each split between the CTAs of the pair), two
// MMAs per k-step into both TMEM accumulators. A CTA then loads 48 KB per
// 2 x 256 x 256 x 128 MACs instead of 64 KB, 25% fewer operand bytes per MAC,
// which pays where the operand stream bounds a long run of tiles (the first
// Linear of the InternViT-6B connector, K = 12800, 8320 tiles). A wide tile
// holds both accumulators, so its epilogue does not overlap the next tile's
// mainloop past its first half. Launches with wide problems use the ring as
// six slots with a full and an empty barrier each (SLOT_RING), a stage taking
// the next two or three slots in turn; the others keep the three fixed
// stages, whose single barrier pair per stage measured faster on the small
// images.
//
// Operand views (all 128-byte swizzled, box 64 x rows x ... x 2 chunks):
//   plain rows [M, K]:      {64, M, K/64}, strides {2K, 128} bytes
//   weights [N, K]:         the same with N rows
//   pixel_shuffle block (qb, rb) at factor 1/f, g = 32/f grid columns:
//     {64, b: g, tile*g + a, C/64} over the pixels (f a + qb, f b + rb),
//     strides {2fC, 64fC, 128} bytes from the block's first pixel; one box is
//     the 128 rows (a, b) of 128/g grid rows, so row m of the shuffled
//     matrix and channel chunk c of block (qb, rb) is one box coordinate.
#pragma once
#include "ivc_gemm.cuh"
#include "ivc_graph_schedule.h"

namespace ivc {

constexpr int GG_MAX_PROBLEMS = 5;
constexpr int GG_MAX_AMAPS = 24;   // up to 16 per factor-0.25 problem, 4 per factor-0.5
constexpr int GG_MAX_SCHED = 1024;  // tiles a host schedule can list
constexpr int GG_MAX_PAIRS = 80;
constexpr int GG_BN = 256;        // accumulator width (a wide tile spans two)
constexpr int GG_SLOTS = 6;        // ring slots of one 32 KB box
constexpr int GG_STAGES = 3;       // fixed stages of an A and a B box (no wide problems)
constexpr int GG_KPER = 2;          // k-blocks of 64 per stage (one box per operand)
constexpr int GG_TILE_M = 2 * GEMM_BM;

// Shared memory of one CTA: the ring (slots of 2 x 16 KB: 128 rows of A or
// of B for two k-blocks), barriers, per-column epilogue vectors.
struct GraphSmem {
  static constexpr uint32_t CHUNK = GEMM_BM * GEMM_BK * 2;  // 128 rows x 64 bf16
  static constexpr uint32_t SLOT = GG_KPER * CHUNK;
  static constexpr uint32_t RING = GG_SLOTS * SLOT;
  static constexpr uint32_t BARS = (2 * GG_SLOTS + 4) * 8 + 16;
  static constexpr uint32_t COLS = 2 * GG_BN * 4;
  static constexpr uint32_t TOTAL = 1024 + RING + BARS + COLS;
  static constexpr uint32_t TMEM_COLS = 2 * GG_BN;
};

struct GraphProblem {
  int M, N, K;
  int a_mode;          // AMode
  int a_map;           // first A map of this problem in GraphMaps::a
  int a_views;         // 1 (plain rows) or f*f (one view per pixel_shuffle block)
  int c_blocks;        // C / 64 (pixel_shuffle modes)
  int m_tiles, n_tiles;
  int epi_mode, gelu, remap;
  int dep;             // problem whose output rows this one reads, or -1
  int dep_target;      // that problem's counter value of a complete row block
  int done_base;       // this problem's first row-block counter in done[]
  const __nv_bfloat16* bias;  // EPI_BIAS (may be null)
  const float* colsum;
  const float* fbias;
  const float* row_mean;
  const float* row_rstd;
  void* out;           // bf16 [M, ldo]
  long long ldo;
  int wide;            // 1: 256 x 512 tiles (n_tiles counts 512-column blocks)
  int group_m;         // > 0: tiles in groups of group_m row blocks (tile_coords)
};

struct alignas(64) GraphMaps {
  CUtensorMap a[GG_MAX_AMAPS];
  CUtensorMap b[GG_MAX_PROBLEMS];
};

struct GraphArgs {
  int n_problems;
  int n_amaps;
  GraphProblem p[GG_MAX_PROBLEMS];
  int unit_begin[GG_MAX_PROBLEMS + 1];  // global tile index of each problem's first tile
  int* done;                            // row-block counters, zero at launch
  int n_pairs;
  int scheduled;                        // 1: per-pair lists below; 0: round-robin
  unsigned short sched_off[GG_MAX_PAIRS + 1];
  unsigned short sched[GG_MAX_SCHED];
};

struct GraphTile {
  int p, m, n;
};

__device__ __forceinline__ GraphTile graph_tile(const GraphArgs& g, int u) {
  int p = 0;
  while (p + 1 < g.n_problems && u >= g.unit_begin[p + 1]) ++p;
  GraphTile t{p, 0, 0};
  tile_coords(u - g.unit_begin[p], g.p[p].m_tiles, g.p[p].n_tiles, g.p[p].group_m, &t.m, &t.n);
  return t;
}

// Bounded acquire poll of a row-block counter (one thread).
__device__ __forceinline__ bool wait_counter(const int* ctr, int target) {
  const long long t0 = clock64();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (clock64() - t0 > IVC_WAIT_CYCLES) return false;
    __nanosleep(64);
  }
}

__device__ __forceinline__ void graph_fence_proxy_async() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <bool SLOT_RING>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_graph_kernel(const __grid_constant__ GraphMaps maps, const __grid_constant__ GraphArgs g,
                      int* __restrict__ status) {
  using L = GraphSmem;
  constexpr int BN = GG_BN;
  constexpr int SLOTS = GG_SLOTS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::RING);
  uint64_t* empty_bar = full_bar + SLOTS;
  uint64_t* tfull_bar = empty_bar + SLOTS;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + 2);
  float* s_col0 = reinterpret_cast<float*>(smem + L::RING + L::BARS);
  float* s_col1 = s_col0 + BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int q = blockIdx.x / 2;  // this pair
  const int units_total = g.unit_begin[g.n_problems];
  int n_my;
  if (g.scheduled)
    n_my = g.sched_off[q + 1] - g.sched_off[q];
  else
    n_my = q < units_total ? (units_total - q + g.n_pairs - 1) / g.n_pairs : 0;
  auto unit_at = [&](int i) -> int {
    return g.scheduled ? static_cast<int>(g.sched[g.sched_off[q] + i]) : q + i * g.n_pairs;
  };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < SLOTS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);  // 4 epilogue warps of each CTA of the pair
    }
    fence_mbar_init();
    for (int i = 0; i < g.n_amaps; ++i) tma_prefetch_desc(&maps.a[i]);
    for (int p = 0; p < g.n_problems; ++p) tma_prefetch_desc(&maps.b[p]);
  }
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;
  // The first problems' epilogues read the LayerNorm statistics of the
  // previous kernel in the stream; A and B of every tile are either inputs of
  // the call or written inside this launch.
  if (warp >= 2) pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t sc = 0;  // slot ring: boxes issued (box sc goes to slot sc % SLOTS)
      uint32_t it = 0;  // fixed stages: stages issued
      uint8_t* st_base = ring;
      uint32_t st_lb = 0;
      // Box b (0: A, 1 + h: B half h) of the next stage, once the box that
      // last used its place has been consumed; the pair leader's full barrier
      // expects it from both CTAs.
      auto claim = [&](int b, uint8_t*& dst, uint32_t& lb) -> bool {
        if constexpr (SLOT_RING) {
          const int s = static_cast<int>(sc % SLOTS);
          const uint32_t ph = (sc / SLOTS) & 1;
          ++sc;
          if (!mbar_wait(&empty_bar[s], ph ^ 1)) return false;
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], L::SLOT * 2);
          dst = ring + s * L::SLOT;
          lb = pair_leader_addr(&full_bar[s]);
          return true;
        } else {
          if (b == 0) {
            const int s = static_cast<int>(it % GG_STAGES);
            const uint32_t ph = (it / GG_STAGES) & 1;
            ++it;
            if (!mbar_wait(&empty_bar[s], ph ^ 1)) return false;
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * L::SLOT * 2);
            st_base = ring + s * 2 * L::SLOT;
            st_lb = pair_leader_addr(&full_bar[s]);
          }
          dst = st_base + b * L::SLOT;
          lb = st_lb;
          return true;
        }
      };
      for (int i = 0; i < n_my && ok; ++i) {
        const GraphTile t = graph_tile(g, unit_at(i));
        const GraphProblem& P = g.p[t.p];
        if (P.dep >= 0) {
          if (!wait_counter(g.done + g.p[P.dep].done_base + t.m, P.dep_target)) {
            ok = false;
            break;
          }
          graph_fence_proxy_async();
        }
        const int m0 = t.m * GG_TILE_M + GEMM_BM * rank;
        const int wide = SLOT_RING ? P.wide : 0;  // (no wide problems on fixed stages)
        const int n0 = t.n * (BN << wide) + (BN / 2) * rank;
        const int KT = P.K / GEMM_BK;
        const CUtensorMap* bm = &maps.b[t.p];
        for (int kk = 0; kk < KT; kk += GG_KPER) {
          uint8_t* a_dst;
          uint32_t lb;
          if (!claim(0, a_dst, lb)) { ok = false; break; }
          if (P.a_mode == A_PLAIN) {
            tma_load_3d_pair(a_dst, &maps.a[P.a_map], lb, 0, m0, kk);
          } else {
            // both k-blocks of the stage lie in one pixel_shuffle block
            // (C / 64 is even)
            const int blk = kk / P.c_blocks;
            const int chunk = kk - blk * P.c_blocks;
            int qb, rb;  // pixel_shuffle block: (di, dj) of factor 0.5 or (q, r) of 0.25
            if (P.a_mode == A_PS_HALF) {
              qb = blk >> 1;
              rb = blk & 1;
            } else if (P.a_mode == A_PS_QUARTER) {
              qb = blk >> 2;
              rb = blk & 3;
            } else {  // two successive factor-0.5 shuffles: blk = 8ei + 4ej + 2di + dj
              qb = 2 * (blk >> 3) + ((blk >> 1) & 1);
              rb = 2 * ((blk >> 2) & 1) + (blk & 1);
            }
            const int f = P.a_mode == A_PS_HALF ? 2 : 4;
            tma_load_4d_pair(a_dst, &maps.a[P.a_map + qb * f + rb], lb, 0, 0, m0 / (32 / f),
                             chunk);
          }
          for (int h = 0; h <= wide; ++h) {
            uint8_t* b_dst;
            if (!claim(1 + h, b_dst, lb)) { ok = false; break; }
            tma_load_3d_pair(b_dst, bm, lb, 0, n0 + h * BN, kk);
          }
          if (!ok) break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(GG_TILE_M, BN);
      uint32_t sc = 0;            // slot ring: boxes consumed, in the producer's order
      uint32_t it = 0;            // fixed stages: stages consumed
      int st = 0;                 // fixed stages: the current stage
      int nxt = 0;                // accumulator of the next 256-wide tile
      uint32_t uses[2] = {0, 0};  // tiles (or halves) each accumulator has held
      // the ring place (in boxes) of box b of the next stage, once it has landed
      auto take = [&](int b, int& s) -> bool {
        if constexpr (SLOT_RING) {
          s = static_cast<int>(sc % SLOTS);
          const uint32_t ph = (sc / SLOTS) & 1;
          ++sc;
          return mbar_wait(&full_bar[s], ph);
        } else {
          if (b == 0) {
            st = static_cast<int>(it % GG_STAGES);
            const uint32_t ph = (it / GG_STAGES) & 1;
            ++it;
            if (!mbar_wait(&full_bar[st], ph)) return false;
          }
          s = 2 * st + b;
          return true;
        }
      };
      for (int i = 0; i < n_my && ok; ++i) {
        const GraphTile t = graph_tile(g, unit_at(i));
        const int wide = SLOT_RING ? g.p[t.p].wide : 0;
        const int KT = g.p[t.p].K / GEMM_BK;
        // half h accumulates in acc[h]: a wide tile takes both
        // (fixed-bound loops over the halves keep these arrays in registers)
        const int acc[2] = {wide ? 0 : nxt, 1};
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (h <= wide && ok) {
            const uint32_t u = acc[h] == 0 ? uses[0] : uses[1];
            ok = mbar_wait(&tempty_bar[acc[h]], (u & 1) ^ 1);
          }
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < KT; kk += GG_KPER) {
          int sa, sb[2] = {0, 0};
          ok = take(0, sa);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (h <= wide && ok) ok = take(1 + h, sb[h]);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < GG_KPER; ++j) {
            const uint64_t ad = sw128_kmajor_desc(smem_u32(ring + sa * L::SLOT + j * L::CHUNK));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (h > wide) break;
              const uint64_t bd =
                  sw128_kmajor_desc(smem_u32(ring + sb[h] * L::SLOT + j * L::CHUNK));
              const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc[h] * BN);
#pragma unroll
              for (int k = 0; k < GEMM_BK / 16; ++k)
                umma_bf16_pair(d_tmem, ad + 2 * k, bd + 2 * k, idesc,
                               (kk != 0 || j != 0 || k != 0) ? 1u : 0u);
            }
          }
          if constexpr (SLOT_RING) {
            umma_commit_pair(&empty_bar[sa]);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              if (h <= wide) umma_commit_pair(&empty_bar[sb[h]]);
          } else {
            umma_commit_pair(&empty_bar[st]);
          }
        }
        if (!ok) break;
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (h <= wide) {
            umma_commit_pair(&tfull_bar[acc[h]]);
            if (acc[h] == 0) ++uses[0]; else ++uses[1];
          }
        if (!wide) nxt ^= 1;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127
    int nxt = 0;  // the MMA issuer's accumulator choice, replayed
    uint32_t uses[2] = {0, 0};
    for (int i = 0; i < n_my; ++i) {
      const GraphTile t = graph_tile(g, unit_at(i));
      const GraphProblem& P = g.p[t.p];
      // a 256-wide tile, or each 256-column half of a wide one in turn
      const int wide = SLOT_RING ? P.wide : 0;
      for (int h = 0; h <= wide; ++h) {
        const int acc = wide ? h : nxt;
        const uint32_t use = acc == 0 ? uses[0]++ : uses[1]++;
        const int tm0 = t.m * GG_TILE_M, tn0 = t.n * (BN << wide) + h * BN;
        epi_bar_sync();
        for (int c = et; c < BN; c += 128) {
          const int n = tn0 + c;
          float c0 = 0.f, c1 = 0.f;
          if (n < P.N) {
            if (P.epi_mode == EPI_LNFOLD) {
              c0 = P.colsum[n];
              c1 = P.fbias[n];
            } else if (P.bias != nullptr) {
              c1 = __bfloat162float(P.bias[n]);
            }
          }
          s_col0[c] = c0;
          s_col1[c] = c1;
        }
        epi_bar_sync();
        // after a timed-out wait the warps keep the named barriers in step
        // (two per accumulator read, one per tile) but do no more work
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], use & 1));
        if (!ok) continue;
        tc_fence_after();
        const int row = tm0 + GEMM_BM * rank + quad * 32 + lane;
        float mean = 0.f, rstd = 1.f;
        if (P.epi_mode == EPI_LNFOLD && row < P.M) {
          mean = P.row_mean[row];
          rstd = P.row_rstd[row];
        }
        const float nms = -mean * rstd;
        long long out_row = row;
        if (P.remap == 1) {
          const int tt = row & 255;
          out_row = (row & ~255) | ((tt & 15) << 4) | (tt >> 4);
        } else if (P.remap == 2) {
          const int tt = row & 63;
          out_row = (row & ~63) | ((tt & 7) << 3) | (tt >> 3);
        }
        const long long out_off = out_row * P.ldo + tn0;
        const uint32_t t_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                static_cast<uint32_t>(acc * BN);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(t_base + c, r);
          tmem_ld_wait();
          if (c + 32 == BN) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(pair_leader_addr(&tempty_bar[acc]));
          }
          if (row < P.M && tn0 + c < P.N) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float x = __uint_as_float(r[j]);
              if (P.epi_mode == EPI_LNFOLD)
                x = fmaf(rstd, x, nms * s_col0[c + j]) + s_col1[c + j];
              else
                x += s_col1[c + j];
              v[j] = P.gelu ? gelu_erf(x) : x;
            }
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.out) + out_off + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                                  pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                  pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                  pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          }
        }
      }
      if (!wide) nxt ^= 1;
      // this CTA's 128 rows of the tile are stored: count them into the row
      // block (GPU-scope release after the four warps' stores)
      epi_bar_sync();
      if (ok && et == 0) {
        __threadfence();
        atomicAdd(g.done + P.done_base + t.m, 1);
      }
    }
  }

  if (!ok && status != nullptr) atomicOr(status, 4 /* IVC_DEV_WAIT_TIMEOUT */);
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
  }
}

}  // namespace ivc
