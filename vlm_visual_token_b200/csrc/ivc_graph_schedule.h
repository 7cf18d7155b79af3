// ivc_graph_schedule.h — host-side list schedule of output tiles over the CTA
// pairs of one persistent multi-Linear launch (ivc_gemm_graph.cuh).
//
// Tiles are numbered in priority order: problem by problem (the problems
// already arranged in priority order, every dependency pointing to an earlier
// problem), then within a problem row block by row block, or in groups of G
// row blocks, column block by column block within a group (tile_coords: a
// weight panel read by the group's rows then comes from DRAM once per group,
// and the group's rows of A stay in L2 across the panels). Greedy list
// scheduling takes them in that order and gives each to the pair that becomes
// free first in a cost model (k-steps of the tile plus a fixed epilogue
// cost); a tile that reads another problem's rows cannot start before the
// model time at which that row block is complete. Every pair's list is then
// in increasing tile order, which is what keeps the launch deadlock-free (the
// earliest unfinished tile never waits for a later one).
//
// Free of CUDA calls, so that it can be unit-tested on a machine without a
// GPU; tile_coords is shared with the kernel.
#pragma once
#include <cstdint>
#include <vector>

#ifdef __CUDACC__
#define IVC_HD __host__ __device__
#else
#define IVC_HD
#endif

namespace ivc {

// Row block m and column block n of tile idx of a problem with m_tiles x
// n_tiles tiles: with group_m > 0 in groups of group_m row blocks (the last
// group may be shorter), column block by column block inside a group;
// otherwise row block by row block.
IVC_HD inline void tile_coords(int idx, int m_tiles, int n_tiles, int group_m, int* m, int* n) {
  if (group_m > 0) {
    const int per_group = group_m * n_tiles;
    const int grp = idx / per_group;
    const int r0 = grp * group_m;
    const int rows = m_tiles - r0 < group_m ? m_tiles - r0 : group_m;
    const int w = idx - grp * per_group;
    *m = r0 + w % rows;
    *n = w / rows;
  } else {
    *m = idx / n_tiles;
    *n = idx % n_tiles;
  }
}

struct SchedProblem {
  int m_tiles;
  int n_tiles;
  int k_steps;      // cost of one tile in the model
  int dep;          // problem (earlier index) whose row block m a tile of row block m reads, or -1
  int group_m = 0;  // > 0: tiles in groups of group_m row blocks (tile_coords)
};

// First global tile id of each problem, and the total in the last entry.
inline std::vector<int> schedule_unit_begin(const std::vector<SchedProblem>& P) {
  std::vector<int> b(P.size() + 1, 0);
  for (size_t i = 0; i < P.size(); ++i) b[i + 1] = b[i] + P[i].m_tiles * P[i].n_tiles;
  return b;
}

// Per-pair tile lists (global ids). Returns false for a dependency that does
// not point to an earlier problem or for row-block counts that differ.
inline bool list_schedule(const std::vector<SchedProblem>& P, int pairs, int epi_cost,
                          std::vector<std::vector<int>>& lists) {
  lists.assign(pairs > 0 ? pairs : 0, {});
  if (pairs <= 0) return false;
  std::vector<std::vector<double>> block_done(P.size());
  std::vector<std::vector<int>> block_left(P.size());
  for (size_t p = 0; p < P.size(); ++p) {
    if (P[p].dep >= static_cast<int>(p)) return false;
    if (P[p].dep >= 0 && P[P[p].dep].m_tiles != P[p].m_tiles) return false;
    block_done[p].assign(P[p].m_tiles, 0.0);
    block_left[p].assign(P[p].m_tiles, P[p].n_tiles);
  }
  std::vector<double> free_at(pairs, 0.0);
  int id = 0;
  for (size_t p = 0; p < P.size(); ++p) {
    for (int idx = 0; idx < P[p].m_tiles * P[p].n_tiles; ++idx, ++id) {
      int m, n;
      tile_coords(idx, P[p].m_tiles, P[p].n_tiles, P[p].group_m, &m, &n);
      int best = 0;
      for (int q = 1; q < pairs; ++q)
        if (free_at[q] < free_at[best]) best = q;
      double start = free_at[best];
      if (P[p].dep >= 0) {
        const double ready = block_done[P[p].dep][m];
        if (ready > start) start = ready;
      }
      const double end = start + P[p].k_steps + epi_cost;
      free_at[best] = end;
      lists[best].push_back(id);
      if (end > block_done[p][m]) block_done[p][m] = end;
    }
  }
  return true;
}

}  // namespace ivc
