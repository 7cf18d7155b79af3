// ivc_graph.cu — host side of the multi-Linear persistent launch
// (ivc_gemm_graph.cuh): tensor maps, problem table, list schedule, launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>

#include <vector>

#include "ivc_gemm_graph.cuh"
#include "ivc_graph_schedule.h"
#include "ivc_internal.h"

namespace ivc {

// Two-k-block views (box: 128 rows x 2 chunks of 64 channels, the chunk
// outermost; see ivc_gemm_graph.cuh).
// Row-major [rows, cols] bf16: {64, rows, cols / 64}.
static int map_rows_2k(CUtensorMap* m, const void* base, long long rows, long long cols) {
  const unsigned long long d[3] = {64, static_cast<unsigned long long>(rows),
                                   static_cast<unsigned long long>(cols / 64)};
  const unsigned long long st[2] = {static_cast<unsigned long long>(cols) * 2, 128};
  const unsigned box[3] = {64, static_cast<unsigned>(GEMM_BM), GG_KPER};
  return map_bf16(m, 3, base, d, st, box);
}

// The [T,32,32,C] features at factor 1/f: one view per pixel_shuffle block
// (qb, rb), maps[qb * f + rb] = {64, b: g, tile * g + a, C / 64} over the
// pixels (f a + qb, f b + rb), g = 32 / f.
static int map_ps_2k(CUtensorMap* maps, const void* x, int T, int C, int f) {
  const int g = 32 / f;
  const unsigned long long Cu = static_cast<unsigned long long>(C);
  for (int qb = 0; qb < f; ++qb)
    for (int rb = 0; rb < f; ++rb) {
      const char* base = static_cast<const char*>(x) + (static_cast<size_t>(qb) * 32 + rb) * C * 2;
      const unsigned long long d[4] = {64, static_cast<unsigned long long>(g),
                                       static_cast<unsigned long long>(T) * g, Cu / 64};
      const unsigned long long st[3] = {Cu * f * 2, Cu * 32 * f * 2, 128};
      const unsigned box[4] = {64, static_cast<unsigned>(g), static_cast<unsigned>(GEMM_BM / g),
                               GG_KPER};
      const int rc = map_bf16(&maps[qb * f + rb], 4, base, d, st, box);
      if (rc) return rc;
    }
  return IVC_OK;
}

bool graph_supported(const GraphProblemCall* probs, int n) {
  if (n <= 0 || n > GG_MAX_PROBLEMS) return false;
  int amaps = 0;
  for (int i = 0; i < n; ++i) {
    const GraphProblemCall& c = probs[i];
    if (c.M <= 0 || c.N <= 0 || c.N % 32 != 0 || c.K % (GEMM_BK * GG_KPER) != 0) return false;
    if (c.dep >= i || (c.dep >= 0 && probs[c.dep].M != c.M)) return false;
    if (c.a_mode != A_PLAIN && (c.C % (GEMM_BK * GG_KPER) != 0)) return false;
    amaps += c.a_mode == A_PLAIN ? 1 : (c.a_mode == A_PS_HALF ? 4 : 16);
  }
  return amaps <= GG_MAX_AMAPS;
}

int graph_counters(const GraphProblemCall* probs, int n) {
  int c = 0;
  for (int i = 0; i < n; ++i) c += (probs[i].M + GG_TILE_M - 1) / GG_TILE_M;
  return c;
}

// IVC_GRAPH_GROUP: -1 (unset) for the size rule in launch_gemm_graph, else
// the group height in row blocks for every problem (0: row-block order).
static int graph_group_override() {
  static int v = -2;
  if (v == -2) {
    const char* e = std::getenv("IVC_GRAPH_GROUP");
    v = e && e[0] >= '0' && e[0] <= '9' ? std::atoi(e) : -1;
  }
  return v;
}

int launch_gemm_graph(const GraphProblemCall* probs, int n, int* done, int reserve_sms,
                      const Launch& L) {
  if (done == nullptr) return IVC_EINVAL;
  if (!graph_supported(probs, n)) return IVC_EUNSUPPORTED;
  GraphArgs g{};
  g.n_problems = n;
  g.done = done;
  int max_pairs = (num_sms() - (reserve_sms > 0 ? reserve_sms : 0)) / 2;
  if (max_pairs > GG_MAX_PAIRS) max_pairs = GG_MAX_PAIRS;
  if (max_pairs < 1) max_pairs = 1;
  // 256 x 512 tiles for the problems that allow them (wide == 1) when they
  // have many rounds of 256-wide tiles (at least 8 per pair), where the 25%
  // fewer operand bytes per MAC pay; wide == 2 asks for them in any case.
  bool use_wide = false;
  std::vector<int> wide(n, 0);
  for (int i = 0; i < n; ++i) {
    const GraphProblemCall& c = probs[i];
    const long long tiles256 = static_cast<long long>((c.M + GG_TILE_M - 1) / GG_TILE_M) *
                               ((c.N + GG_BN - 1) / GG_BN);
    wide[i] = c.wide == 2 || (c.wide == 1 && tiles256 >= 8LL * max_pairs) ? 1 : 0;
    use_wide = use_wide || wide[i];
  }
  // A weight matrix larger than half of L2 (128 MB for mlp2.fc1, 131 MB for
  // the InternViT-6B connector's mlp1.fc1) does not stay in L2 while the
  // rows of A stream past it: its tiles run in groups of 8 row blocks, column
  // block by column block, so that each panel comes from DRAM once per group
  // and the group's rows of A (8 x 256 rows) stay in L2 across the panels.
  // IVC_GRAPH_GROUP=0 keeps row-block order, =g sets groups of g everywhere.
  const int group_env = graph_group_override();
  std::vector<int> group(n, 0);
  for (int i = 0; i < n; ++i) {
    const double w_bytes = 2.0 * probs[i].N * probs[i].K;
    group[i] = group_env >= 0 ? group_env : (w_bytes > 64e6 ? 8 : 0);
  }
  std::vector<SchedProblem> sp(n);
  int units = 0;
  for (int i = 0; i < n; ++i) {
    const GraphProblemCall& c = probs[i];
    const int w = wide[i];
    const int mt = (c.M + GG_TILE_M - 1) / GG_TILE_M;
    const int nt = (c.N + (GG_BN << w) - 1) / (GG_BN << w);
    // a wide tile's cost in the model: twice the MACs, 1.5 times the bytes
    sp[i] = {mt, nt, (c.K / GEMM_BK) * (w ? 7 : 4) / 4, c.dep, group[i]};
    units += mt * nt;
  }
  const int pairs = units < max_pairs ? units : max_pairs;
  std::vector<std::vector<int>> lists;
  if (units <= GG_MAX_SCHED && !list_schedule(sp, pairs, 4, lists)) return IVC_EINVAL;
  int amap = 0, ctr = 0;
  GraphMaps m{};
  for (int i = 0; i < n; ++i) {
    const GraphProblemCall& c = probs[i];
    GraphProblem& P = g.p[i];
    P.M = c.M;
    P.N = c.N;
    P.K = c.K;
    P.a_mode = c.a_mode;
    P.a_map = amap;
    P.c_blocks = c.C / GEMM_BK;
    P.m_tiles = (c.M + GG_TILE_M - 1) / GG_TILE_M;
    P.wide = wide[i];
    P.n_tiles = (c.N + (GG_BN << P.wide) - 1) / (GG_BN << P.wide);
    P.epi_mode = c.epi_mode;
    P.gelu = c.gelu;
    P.remap = c.remap;
    P.dep = c.dep;
    P.done_base = ctr;
    P.bias = c.bias;
    P.colsum = c.colsum;
    P.fbias = c.fbias;
    P.row_mean = c.row_mean;
    P.row_rstd = c.row_rstd;
    P.out = c.out;
    P.ldo = c.ldo;
    P.group_m = group[i];
    ctr += P.m_tiles;
    int rc;
    if (c.a_mode == A_PLAIN) {
      rc = map_rows_2k(&m.a[amap], c.a, c.M, c.K);
      P.a_views = 1;
    } else {
      const int f = c.a_mode == A_PS_HALF ? 2 : 4;
      rc = map_ps_2k(&m.a[amap], c.a, c.T, c.C, f);
      P.a_views = f * f;
    }
    if (rc) return rc;
    amap += P.a_views;
    rc = map_rows_2k(&m.b[i], c.B, c.N, c.K);
    if (rc) return rc;
  }
  for (int i = 0; i < n; ++i)
    if (g.p[i].dep >= 0) g.p[i].dep_target = 2 * g.p[g.p[i].dep].n_tiles;
  g.n_amaps = amap;
  const std::vector<int> ub = schedule_unit_begin(sp);
  for (int i = 0; i <= n; ++i) g.unit_begin[i] = ub[i];
  g.n_pairs = pairs;
  g.scheduled = 0;
  if (!lists.empty()) {
    int off = 0;
    for (int q = 0; q < pairs; ++q) {
      g.sched_off[q] = static_cast<unsigned short>(off);
      for (int u : lists[q]) g.sched[off++] = static_cast<unsigned short>(u);
    }
    g.sched_off[pairs] = static_cast<unsigned short>(off);
    g.scheduled = 1;
  }
  using S = GraphSmem;
  auto kern = use_wide ? gemm_graph_kernel<true> : gemm_graph_kernel<false>;
  if (smem_optin(reinterpret_cast<const void*>(kern), S::TOTAL) != IVC_OK) return IVC_ECUDA;
  TraceScope ts("connector.graph", L.stream);
  return launch_k(kern, dim3(2 * pairs), dim3(GEMM_THREADS), S::TOTAL, L.stream, 2, m, g,
                  L.status);
}

}  // namespace ivc
