// Host-only check of ivc::list_schedule (ivc_graph_schedule.h): every tile is
// assigned to exactly one CTA pair, each pair's list is increasing, and
// running the lists (each pair in order, a tile starting only once the row
// block it reads is complete) finishes every tile: no deadlock, for the
// connector problem sets of both MLPs and for random ones, with tiles numbered
// row block by row block or in groups of row blocks (tile_coords).
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "ivc_graph_schedule.h"

using ivc::SchedProblem;

#define CHECK(cond)                                         \
  do {                                                      \
    if (!(cond)) {                                          \
      std::printf("FAILED line %d: %s\n", __LINE__, #cond); \
      return false;                                         \
    }                                                       \
  } while (0)

static bool check(const std::vector<SchedProblem>& P, int pairs) {
  std::vector<std::vector<int>> lists;
  CHECK(ivc::list_schedule(P, pairs, 4, lists));
  const std::vector<int> ub = ivc::schedule_unit_begin(P);
  const int units = ub.back();
  std::vector<int> seen(units, 0);
  for (const auto& l : lists)
    for (size_t i = 0; i < l.size(); ++i) {
      CHECK(l[i] >= 0 && l[i] < units);
      ++seen[l[i]];
      if (i > 0) CHECK(l[i] > l[i - 1]);
    }
  for (int u = 0; u < units; ++u) CHECK(seen[u] == 1);
  // execute: repeatedly let every pair run its next tile if ready
  std::vector<std::vector<int>> left(P.size());
  for (size_t p = 0; p < P.size(); ++p) left[p].assign(P[p].m_tiles, P[p].n_tiles);
  std::vector<size_t> pos(pairs, 0);
  int done = 0;
  bool progress = true;
  while (done < units && progress) {
    progress = false;
    for (int q = 0; q < pairs; ++q) {
      if (pos[q] >= lists[q].size()) continue;
      const int u = lists[q][pos[q]];
      int p = 0;
      while (u >= ub[p + 1]) ++p;
      // the row block of a tile id, as the graph kernel derives it
      int m, n;
      ivc::tile_coords(u - ub[p], P[p].m_tiles, P[p].n_tiles, P[p].group_m, &m, &n);
      if (P[p].dep >= 0 && left[P[p].dep][m] != 0) continue;
      --left[p][m];
      ++pos[q];
      ++done;
      progress = true;
    }
  }
  CHECK(done == units);
  return true;
}

// tile_coords numbers every (row block, column block) exactly once.
static bool coords_bijective(int mt, int nt, int group) {
  std::vector<int> seen(mt * nt, 0);
  for (int idx = 0; idx < mt * nt; ++idx) {
    int m, n;
    ivc::tile_coords(idx, mt, nt, group, &m, &n);
    CHECK(m >= 0 && m < mt && n >= 0 && n < nt);
    ++seen[m * nt + n];
  }
  for (int v : seen) CHECK(v == 1);
  return true;
}

int main() {
  for (int mt = 1; mt <= 20; ++mt)
    for (int nt = 1; nt <= 7; ++nt)
      for (int group = 0; group <= 9; ++group)
        if (!coords_bijective(mt, nt, group)) return 1;
  // groups of 3 over 7 row blocks: rows 0-2 column by column, then 3-5, then 6
  {
    int m, n;
    ivc::tile_coords(4, 7, 2, 3, &m, &n);  // group 0, column 1, row 1
    if (m != 1 || n != 1) return 1;
    ivc::tile_coords(12, 7, 2, 3, &m, &n);  // last group (row 6 only), column 0
    if (m != 6 || n != 0) return 1;
  }
  // both MLPs of a 13-tile image in priority order: mlp2.fc1, mlp1.fc1,
  // mlp2.fc2 (reads 0), mlp1.fc2 (reads 1), mlp2.fc3 (reads 2)
  std::vector<SchedProblem> flash = {
      {4, 16, 256, -1}, {13, 8, 64, -1}, {4, 8, 64, 0}, {13, 8, 32, 1}, {4, 8, 32, 2}};
  for (int pairs : {1, 7, 64, 74, 80})
    if (!check(flash, pairs)) return 1;
  // the same with mlp2.fc1 in one group (column block by column block)
  flash[0].group_m = 8;
  for (int pairs : {1, 7, 56, 64, 74, 80})
    if (!check(flash, pairs)) return 1;
  // one MLP, fc1 then fc2
  if (!check({{3, 4, 64, -1}, {3, 4, 32, 0}}, 74)) return 1;
  // dependencies must point to earlier problems with the same row blocks
  std::vector<std::vector<int>> lists;
  if (ivc::list_schedule({{2, 2, 8, 1}, {2, 2, 8, -1}}, 4, 1, lists)) return 1;
  if (ivc::list_schedule({{2, 2, 8, -1}, {3, 2, 8, 0}}, 4, 1, lists)) return 1;
  // random problem chains
  std::srand(7);
  for (int trial = 0; trial < 200; ++trial) {
    const int n = 1 + std::rand() % 5;
    std::vector<SchedProblem> P;
    const int mt = 1 + std::rand() % 9;
    for (int i = 0; i < n; ++i) {
      const int dep = i > 0 && std::rand() % 2 ? std::rand() % i : -1;
      P.push_back({mt, 1 + std::rand() % 12, 1 + std::rand() % 300, dep, std::rand() % 4});
    }
    if (!check(P, 1 + std::rand() % 80)) return 1;
  }
  std::printf("graph schedule ok\n");
  return 0;
}
