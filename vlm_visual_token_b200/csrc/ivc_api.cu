// ivc_api.cu — the C ABI of libivc.so (declared in include/ivc.h).
//
// Each entry point validates its arguments on the host, carves its scratch
// buffers out of the caller's workspace and enqueues the kernels of the hot
// path on the caller's stream. Nothing here computes on the host and nothing
// allocates device memory.
#include <cuda_runtime.h>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "ivc_gemm.cuh"
#include "ivc_internal.h"

using namespace ivc;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeader = 256;  // status word lives at offset 0

inline size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// Sequential carve-out of workspace buffers (sizes only when base == nullptr).
struct Carver {
  char* base;
  size_t off = kHeader;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align_up(count * sizeof(T));
    return p;
  }
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool mlp_shape_ok(const ivc_mlp* m) {
  if (!m || (m->n_linear != 2 && m->n_linear != 3)) return false;
  for (int i = 0; i <= m->n_linear; ++i)
    if (m->dims[i] <= 0 || m->dims[i] % 64 != 0) return false;
  return true;
}

int mlp_ptrs_ok(const ivc_mlp* m) {
  if (!m->ln_gamma || !m->ln_beta) return IVC_EINVAL;
  for (int i = 0; i < m->n_linear; ++i) {
    if (!m->W[i]) return IVC_EINVAL;
    if (!aligned16(m->W[i])) return IVC_EALIGN;
  }
  if (m->fold_colsum && (!m->fold_W0 || !m->fold_bias)) return IVC_EINVAL;
  if (m->fold_W0 && !aligned16(m->fold_W0)) return IVC_EALIGN;
  return IVC_OK;
}

int router_shape_ok(const ivc_router* r, int C) {
  if (!r) return IVC_EINVAL;
  if (r->D != C || r->heads * 64 != r->D) return IVC_EUNSUPPORTED;
  const int okK[4] = {256, 512, 1024, 2048};
  bool d_ok = false, g_ok = false;
  for (int k : okK) {
    d_ok |= r->D == k;
    g_ok |= r->gate_hidden == k;
  }
  if (!d_ok || !g_ok) return IVC_EUNSUPPORTED;
  if (r->quantile_scope != 0 && r->quantile_scope != 1) return IVC_EINVAL;
  if (!(r->rel_q >= 0.0 && r->rel_q <= 1.0)) return IVC_EINVAL;  // also NaN
  if (r->pool_mode != IVC_POOL_FOLDED && r->pool_mode != IVC_POOL_LITERAL) return IVC_EINVAL;
  if (r->gate_residual != 0 && r->gate_residual != 1) return IVC_EINVAL;
  if (r->pool_mode == IVC_POOL_FOLDED && (r->heads > 16 || r->D % 128 != 0))
    return IVC_EUNSUPPORTED;
  if (!r->query || !r->gWout) return IVC_EINVAL;
  if (!aligned16(r->query)) return IVC_EALIGN;
  {
    // the folds of ivc_router_fold: all or none, folded pooling only
    const void* f[8] = {r->fold_u1,     r->fold_c1,     r->fold_wqo[0], r->fold_wqo[1],
                        r->fold_wqo[2], r->fold_bqo[0], r->fold_bqo[1], r->fold_bqo[2]};
    int set = 0;
    for (const void* p : f) {
      set += p != nullptr;
      if (!aligned16(p)) return IVC_EALIGN;
    }
    if (set != 0 && (set != 8 || r->pool_mode != IVC_POOL_FOLDED)) return IVC_EINVAL;
  }
  for (int l = 0; l < 4; ++l) {
    const void* ws[6] = {r->Wq[l], r->Wk[l], r->Wv[l], r->Wo[l], r->gW1[l], r->gW2[l]};
    for (const void* w : ws) {
      if (!w) return IVC_EINVAL;
      if (!aligned16(w)) return IVC_EALIGN;
    }
    if (!r->gln_g[l] || !r->gln_b[l]) return IVC_EINVAL;
  }
  return IVC_OK;
}

// Buffers one ps_project needs (given rows and the MLP).
struct PsBufs {
  float* mean = nullptr;
  float* rstd = nullptr;
  bf16* fold_W0 = nullptr;
  float* fold_cs = nullptr;
  float* fold_b = nullptr;
  bf16* h1 = nullptr;
  bf16* h2 = nullptr;
  float* split_part = nullptr;  // split-K scratch (flash flows only), shared
  int* split_s = nullptr;
  int* done = nullptr;          // row-block counters of the multi-Linear launch
};

void carve_ps(Carver& cv, const ivc_mlp* m, long long rows, bool need_stats, PsBufs& b) {
  if (need_stats) {
    b.mean = cv.take<float>(rows);
    b.rstd = cv.take<float>(rows);
  }
  if (!m->fold_colsum) {
    b.fold_W0 = cv.take<bf16>(static_cast<size_t>(m->dims[1]) * m->dims[0]);
    b.fold_cs = cv.take<float>(m->dims[1]);
    b.fold_b = cv.take<float>(m->dims[1]);
  }
  b.h1 = cv.take<bf16>(rows * m->dims[1]);
  if (m->n_linear == 3) b.h2 = cv.take<bf16>(rows * m->dims[2]);
  // one counter per 256-row block and Linear
  b.done = cv.take<int>(static_cast<size_t>((rows + 255) / 256) * m->n_linear);
}

struct RouteBufs {
  float* KV = nullptr;   // literal pooling: K/V of the 4 layers
  bf16* U2 = nullptr;    // folded pooling: split u of one layer [T][32][D]
  float* cb = nullptr;   //   c [T][16]
  float* S = nullptr;    //   single-pass attention: chunk max / sum [2][T*8*16];
                         //   tensor-core form: split scores [T*1024][32]
  bf16* P2 = nullptr;    //   tensor-core form: split softmax weights [T*128][1024]
  float* Z = nullptr;    //   single-pass attention: chunk sums [T][8][16][D];
                         //   tensor-core form: split weighted sums [T*128][D]
  float* z = nullptr;    //   merged weighted sums [T][16][D]
  float* h = nullptr;    //   gating state [T][D] (persistent router, fused Gating)
  unsigned* bar = nullptr;  // fused router: grid barrier words
  float* Q1;
  float* Q;
  float* O;
  float* q;
  float* u1;
  float* u2;
};

void carve_route(Carver& cv, const ivc_router* r, int T, RouteBufs& b) {
  const long long D = r->D;
  if (r->pool_mode == IVC_POOL_LITERAL) {
    b.KV = cv.take<float>(static_cast<size_t>(T) * 1024 * 8 * D);
  } else {
    b.U2 = cv.take<bf16>(static_cast<size_t>(T) * 32 * D);
    b.cb = cv.take<float>(static_cast<size_t>(T) * 16);
    b.S = cv.take<float>(static_cast<size_t>(T) * 1024 * 32);
    b.P2 = cv.take<bf16>(static_cast<size_t>(T) * 128 * 1024);
    b.Z = cv.take<float>(static_cast<size_t>(T) * 128 * D);
    b.z = cv.take<float>(static_cast<size_t>(T) * 16 * D);
  }
  b.h = cv.take<float>(static_cast<size_t>(T) * D);
  b.bar = cv.take<unsigned>(2);
  b.Q1 = cv.take<float>(D);
  b.Q = cv.take<float>(static_cast<size_t>(T) * D);
  b.O = cv.take<float>(static_cast<size_t>(T) * D);
  b.q = cv.take<float>(static_cast<size_t>(T) * D);
  b.u1 = cv.take<float>(static_cast<size_t>(T) * r->gate_hidden);
  b.u2 = cv.take<float>(static_cast<size_t>(T) * D);
}

#define IVC_TRY(expr)          \
  do {                         \
    const int _rc = (expr);    \
    if (_rc != IVC_OK) return _rc; \
  } while (0)

// Tiles routed to one path (router-first flow), all on the device: the
// listed tile ids, their count, and the first output row of each.
struct Routed {
  const int* list;
  const int* count;
  const int* base;
};

// pixel_shuffle + MLP with the statistics already in b.mean / b.rstd. With
// rt, only the listed tiles are computed (rows in list order) and the last
// Linear stores each tile's rows at its output offset in y.
int ps_mlp(const void* x, int T, int C, bool half, int flags, const ivc_mlp* m, bf16* y,
           const PsBufs& b, const Launch& L, const Routed* rt = nullptr, int reserve_sms = 0) {
  static const char* const kTags[2][3] = {{"mlp2.fc1", "mlp2.fc2", "mlp2.fc3"},
                                          {"mlp1.fc1", "mlp1.fc2", "mlp1.fc3"}};
  const long long rows = static_cast<long long>(T) * (half ? 256 : 64);
  const bf16* W0 = static_cast<const bf16*>(m->fold_W0);
  const float* cs = m->fold_colsum;
  const float* fb = m->fold_bias;
  if (!cs) {
    IVC_TRY(launch_fold(static_cast<const bf16*>(m->W[0]), static_cast<const bf16*>(m->b[0]),
                        static_cast<const bf16*>(m->ln_gamma),
                        static_cast<const bf16*>(m->ln_beta), m->dims[1], m->dims[0],
                        b.fold_W0, b.fold_cs, b.fold_b, L));
    W0 = b.fold_W0;
    cs = b.fold_cs;
    fb = b.fold_b;
  }
  const int remap = (flags & IVC_PS_V1) ? (half ? 1 : 2) : 0;
  GemmCall c{};
  c.tag = kTags[half][0];
  c.a_mode = half ? A_PS_HALF : ((flags & IVC_PS_QUARTER_TWICE) ? A_PS_QUARTER_TWICE : A_PS_QUARTER);
  c.a = x;
  c.T = T;
  c.C = C;
  c.M = static_cast<int>(rows);
  c.N = m->dims[1];
  c.K = m->dims[0];
  c.groups = 1;
  c.B[0] = W0;
  c.epi_mode = EPI_LNFOLD;
  c.gelu = 1;
  c.colsum = cs;
  c.fbias = fb;
  c.row_mean = b.mean;
  c.row_rstd = b.rstd;
  c.out = b.h1;
  c.ldo = m->dims[1];
  c.split_part = b.split_part;
  c.split_s = b.split_s;
  c.reserve_sms = reserve_sms;
  // with weights folded ahead of time the first Linear reads only x and
  // them; the statistics (ps_stats, which may still be running) are read in
  // its epilogue alone. (A fold launched just above writes its weights.)
  c.epi_dep_only = (rt == nullptr && m->fold_colsum != nullptr) ? 1 : 0;
  const int item_rows = half ? 256 : 64;
  if (rt) {
    c.list = rt->list;
    c.list_count = rt->count;
    c.item_rows = item_rows;
    c.stats_remap = 1;
  }
  IVC_TRY(launch_gemm(c, L));
  const bf16* a = b.h1;
  for (int i = 1; i < m->n_linear; ++i) {
    const bool last = i + 1 == m->n_linear;
    GemmCall d{};
    d.tag = kTags[half][i];
    d.a_mode = A_PLAIN;
    d.a = a;
    d.M = static_cast<int>(rows);
    d.N = m->dims[i + 1];
    d.K = m->dims[i];
    d.groups = 1;
    d.B[0] = m->W[i];
    d.bias[0] = static_cast<const bf16*>(m->b[i]);
    d.epi_mode = EPI_BIAS;
    d.gelu = last ? 0 : 1;
    d.remap = last ? remap : 0;
    d.out = last ? y : b.h2;
    d.ldo = m->dims[i + 1];
    d.split_part = b.split_part;
    d.split_s = b.split_s;
    d.reserve_sms = reserve_sms;
    if (rt) {
      d.list_count = rt->count;
      d.item_rows = item_rows;
      d.out_base = last ? rt->base : nullptr;
    }
    IVC_TRY(launch_gemm(d, L));
    a = b.h2;
  }
  return IVC_OK;
}

// The connector's Linears run as one persistent launch (ivc_gemm_graph.cuh)
// where the shapes allow it, unless IVC_GEMM_GRAPH=0 selects one launch per
// Linear.
bool gemm_graph_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_GEMM_GRAPH");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

// 256 x 512 tiles for an MLP's first Linear in the single launch: with
// K >= 8192 (mlp2's, K = 16C; the InternViT-6B connector's mlp1, K = 12800)
// when it has many rounds of tiles (1, the default), never
// (IVC_GRAPH_WIDE=0), or always, whatever K and size (2: the parity tests of
// the wide tiles on small shapes).
int graph_wide_mode() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_GRAPH_WIDE");
    v = (e && (e[0] == '0' || e[0] == '2')) ? e[0] - '0' : 1;
  }
  return v;
}

// The Linears of one pixel_shuffle + MLP as graph problems (appended to
// `probs`; the first reads x through the pixel_shuffle view with the
// LayerNorm fold, each later one the previous one's output). The weights
// must be folded already (W0, cs, fb).
void mlp_problems(const void* x, int T, int C, bool half, int flags, const ivc_mlp* m,
                  const bf16* W0, const float* cs, const float* fb, bf16* y, const PsBufs& b,
                  std::vector<GraphProblemCall>& probs) {
  const int rows = T * (half ? 256 : 64);
  const int remap = (flags & IVC_PS_V1) ? (half ? 1 : 2) : 0;
  GraphProblemCall c{};
  c.a_mode = half ? A_PS_HALF : ((flags & IVC_PS_QUARTER_TWICE) ? A_PS_QUARTER_TWICE : A_PS_QUARTER);
  c.a = x;
  c.T = T;
  c.C = C;
  c.M = rows;
  c.N = m->dims[1];
  c.K = m->dims[0];
  c.B = W0;
  c.epi_mode = EPI_LNFOLD;
  c.gelu = 1;
  c.colsum = cs;
  c.fbias = fb;
  c.row_mean = b.mean;
  c.row_rstd = b.rstd;
  c.out = b.h1;
  c.ldo = m->dims[1];
  c.dep = -1;
  const int wide_mode = graph_wide_mode();
  c.wide = wide_mode == 2 ? 2 : (wide_mode == 1 && c.K >= 8192 ? 1 : 0);
  probs.push_back(c);
  for (int i = 1; i < m->n_linear; ++i) {
    const bool last = i + 1 == m->n_linear;
    GraphProblemCall d{};
    d.a_mode = A_PLAIN;
    d.a = i == 1 ? b.h1 : b.h2;
    d.M = rows;
    d.N = m->dims[i + 1];
    d.K = m->dims[i];
    d.B = m->W[i];
    d.bias = static_cast<const bf16*>(m->b[i]);
    d.epi_mode = EPI_BIAS;
    d.gelu = last ? 0 : 1;
    d.remap = last ? remap : 0;
    d.out = last ? static_cast<void*>(y) : static_cast<void*>(b.h2);
    d.ldo = m->dims[i + 1];
    d.dep = i - 1;  // the previous Linear of this MLP, as an index into this MLP's list
    probs.push_back(d);
  }
}

// LayerNorm-folded weights of the first Linear: the caller's (ivc_mlp_fold)
// or folded now into the workspace.
int folded_weights(const ivc_mlp* m, const PsBufs& b, const Launch& L, const bf16** W0,
                   const float** cs, const float** fb) {
  *W0 = static_cast<const bf16*>(m->fold_W0);
  *cs = m->fold_colsum;
  *fb = m->fold_bias;
  if (*cs) return IVC_OK;
  IVC_TRY(launch_fold(static_cast<const bf16*>(m->W[0]), static_cast<const bf16*>(m->b[0]),
                      static_cast<const bf16*>(m->ln_gamma), static_cast<const bf16*>(m->ln_beta),
                      m->dims[1], m->dims[0], b.fold_W0, b.fold_cs, b.fold_b, L));
  *W0 = b.fold_W0;
  *cs = b.fold_cs;
  *fb = b.fold_b;
  return IVC_OK;
}

int gating_and_route(int T, const int32_t* image_offsets, int I, const ivc_router* r, float* gate,
                     uint8_t* mask, int32_t* offsets, int32_t* total, const RouteBufs& b,
                     const Launch& L);

// One folded pooling layer (see ivc_router.cu): u/c from the layer's query,
// then either the single-pass attention (scores, running softmax and
// weighted sums per 128-token chunk, chunks merged) or scores = X u^T on the
// tensor cores, masked softmax, z = p X on the tensor cores; o = Wv z + bv.
// Q is [T, D], or the shared query (ldq = 0, Tq = 1). With u1/c1 (layer 1's
// fold of the shared query, from ivc_router_fold) there is no fold to do.
int folded_layer(const void* x, const int32_t* valid_len, int T, const ivc_router* r, int l,
                 const float* Q, long long ldq, const RouteBufs& b, const Launch& L,
                 const bf16* u1 = nullptr, const float* c1 = nullptr) {
  const int D = r->D;
  const int Tq = (ldq == 0 || u1 != nullptr) ? 1 : T;
  const bf16* U2 = u1 != nullptr ? u1 : b.U2;
  const float* cb = u1 != nullptr ? c1 : b.cb;
  if (u1 == nullptr)
    IVC_TRY(launch_pool_fold_query(Q, ldq, Tq, static_cast<const bf16*>(r->Wk[l]),
                                   static_cast<const bf16*>(r->bk[l]), D, b.U2, b.cb, L));
  if (pool_attend_wanted()) {
    // chunk partials in Z, their statistics in S, merged sums in z
    IVC_TRY(launch_pool_attend(x, U2, Tq, cb, valid_len, T, D, r->heads, b.Z, b.S, b.z, L));
    return launch_pool_vproj_heads(b.z, T, D, static_cast<const bf16*>(r->Wv[l]),
                                   static_cast<const bf16*>(r->bv[l]), b.O, L);
  }
  GemmCall s{};
  s.tag = "pool.scores";
  s.a_mode = A_PLAIN;
  s.a = x;
  s.M = T * 1024;
  s.N = 32;
  s.K = D;
  s.groups = 1;
  s.B[0] = U2;
  s.b_mode = B_K3D;
  s.b_batches = Tq;
  s.b_batch_rows = Tq == 1 ? T * 1024 : 1024;
  s.b_ld = D;
  s.b_batch_stride = 32LL * D;
  s.epi_mode = EPI_BIAS;
  s.out = b.S;
  s.out_f32 = 1;
  s.ldo = 32;
  IVC_TRY(launch_gemm(s, L));
  IVC_TRY(launch_pool_softmax(b.S, cb, Tq == 1 ? 0 : 16, valid_len, T, r->heads, b.P2, L));
  GemmCall z{};
  z.tag = "pool.wsum";
  z.a_mode = A_PLAIN;
  z.a = b.P2;
  z.M = T * 128;
  z.N = D;
  z.K = 1024;
  z.groups = 1;
  z.B[0] = x;
  z.b_mode = B_MN3D;
  z.b_batches = T;
  z.b_batch_rows = 128;
  z.b_ld = D;
  z.b_batch_stride = 1024LL * D;
  z.epi_mode = EPI_BIAS;
  z.out = b.Z;
  z.out_f32 = 1;
  z.m_valid = 32;
  z.ldo = D;
  IVC_TRY(launch_gemm(z, L));
  return launch_pool_vproj(b.Z, T, D, static_cast<const bf16*>(r->Wv[l]),
                           static_cast<const bf16*>(r->bv[l]), b.O, L);
}

// The tail of each folded pooling layer as one cooperative launch
// (ivc_router_coop.cu) with IVC_POOL_TAIL=1. Off by default: on the 16 CTAs
// it can have beside the connector its merge of the chunk partials and its
// projections are bandwidth-starved (73 us per call; dual flow 0.557 against
// 0.399 ms with the separate kernels).
bool pool_tail_wanted() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_POOL_TAIL");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

// fused_default: use the persistent single-launch router when it applies and
// IVC_ROUTER_FUSED does not say otherwise. The separate kernels, overlapped
// through programmatic dependent launch, now measure faster even alone
// (0.191 against 0.224 ms per ivc_vir_route on the 13-tile image), so every
// caller passes false; IVC_ROUTER_FUSED=1 selects the persistent kernel.
int route_impl(const void* x, const int32_t* valid_len, int T, const int32_t* image_offsets,
               int I, const ivc_router* r, float* gate, uint8_t* mask, int32_t* offsets,
               int32_t* total, const RouteBufs& b, const Launch& L, bool fused_default) {
  const int D = r->D;
  if (router_fused_supported(r) && router_fused_wanted(fused_default)) {
    FusedRouterBufs f{b.Q, b.U2, b.cb, b.S, b.Z, b.z, b.O, b.q, b.h, b.u1, b.u2, b.bar};
    return launch_router_fused(r, x, valid_len, T, image_offsets, I, gate, mask, offsets, total,
                               f, L);
  }
  if (r->pool_mode == IVC_POOL_FOLDED && pool_tail_wanted() && pool_attend_wanted() &&
      pool_tail_supported(D, r->heads)) {
    // per layer: the single-pass attention, then its tail (merge, value,
    // output and next query projections, next key fold) in one cooperative
    // launch; layer 1's query is shared by every tile
    IVC_TRY(launch_gemv_bf16x(static_cast<const bf16*>(r->query), D,
                              static_cast<const bf16*>(r->Wq[0]),
                              static_cast<const bf16*>(r->bq[0]), D, b.Q1, L));
    IVC_TRY(launch_pool_fold_query(b.Q1, 0, 1, static_cast<const bf16*>(r->Wk[0]),
                                   static_cast<const bf16*>(r->bk[0]), D, b.U2, b.cb, L));
    float* mstat = b.S;
    float* lstat = b.S + static_cast<size_t>(T) * 8 * 16;
    for (int l = 0; l < 4; ++l) {
      IVC_TRY(launch_pool_attend(x, b.U2, l == 0 ? 1 : T, b.cb, valid_len, T, D, r->heads, b.Z,
                                 b.S, b.z, L, false));
      IVC_TRY(launch_pool_tail(r, l, b.Z, mstat, lstat, T, b.O, b.q, b.Q, b.U2, b.cb, b.bar, L));
    }
    return gating_and_route(T, image_offsets, I, r, gate, mask, offsets, total, b, L);
  }
  if (r->pool_mode == IVC_POOL_FOLDED) {
    // With the weight folds of ivc_router_fold: layer 1 starts from its
    // folded query, and each later layer's query comes from the previous
    // layer's merged head outputs through P_l = Wq_{l+1} Wo_l in one
    // projection.
    const bool pre = r->fold_u1 != nullptr;
    if (!pre)
      IVC_TRY(launch_gemv_bf16x(static_cast<const bf16*>(r->query), D,
                                static_cast<const bf16*>(r->Wq[0]),
                                static_cast<const bf16*>(r->bq[0]), D, b.Q1, L));
    for (int l = 0; l < 4; ++l) {
      if (l == 0) {
        IVC_TRY(folded_layer(x, valid_len, T, r, 0, b.Q1, 0, b, L,
                             static_cast<const bf16*>(r->fold_u1), r->fold_c1));
      } else {
        if (!pre)
          IVC_TRY(launch_gemv(b.q, D, T, D, static_cast<const bf16*>(r->Wq[l]),
                              static_cast<const bf16*>(r->bq[l]), D, b.Q, D, 0, L));
        IVC_TRY(folded_layer(x, valid_len, T, r, l, b.Q, D, b, L));
      }
      if (pre && l < 3)
        IVC_TRY(launch_gemv_split(b.O, D, T, D, static_cast<const bf16*>(r->fold_wqo[l]),
                                  r->fold_bqo[l], D, b.Q, D, L));
      else
        IVC_TRY(launch_gemv(b.O, D, T, D, static_cast<const bf16*>(r->Wo[l]),
                            static_cast<const bf16*>(r->bo[l]), D, b.q, D, 0, L));
    }
    return gating_and_route(T, image_offsets, I, r, gate, mask, offsets, total, b, L);
  }
  // K/V projections of the four layers: one grouped GEMM, X [T*1024, D].
  GemmCall c{};
  c.tag = "pool.kv";
  c.a_mode = A_PLAIN;
  c.a = x;
  c.M = T * 1024;
  c.N = D;
  c.K = D;
  c.groups = 8;
  for (int l = 0; l < 4; ++l) {
    c.B[2 * l] = r->Wk[l];
    c.B[2 * l + 1] = r->Wv[l];
    c.bias[2 * l] = static_cast<const bf16*>(r->bk[l]);
    c.bias[2 * l + 1] = static_cast<const bf16*>(r->bv[l]);
  }
  c.epi_mode = EPI_BIAS;
  c.out = b.KV;
  c.out_f32 = 1;  // K/V kept in fp32: bf16 K/V alone moves the gates by ~1e-3
  c.ldo = 8LL * D;
  IVC_TRY(launch_gemm(c, L));
  const long long ldkv = 8LL * D;
  // layer 1: the query is the same for every tile.
  IVC_TRY(launch_gemv_bf16x(static_cast<const bf16*>(r->query), D,
                            static_cast<const bf16*>(r->Wq[0]),
                            static_cast<const bf16*>(r->bq[0]), D, b.Q1, L));
  for (int l = 0; l < 4; ++l) {
    const float* Q = b.Q1;
    long long ldq = 0;
    if (l > 0) {
      IVC_TRY(launch_gemv(b.q, D, T, D, static_cast<const bf16*>(r->Wq[l]),
                          static_cast<const bf16*>(r->bq[l]), D, b.Q, D, 0, L));
      Q = b.Q;
      ldq = D;
    }
    IVC_TRY(launch_pool_attention(Q, ldq, b.KV, ldkv, 2 * l * D, (2 * l + 1) * D, valid_len, T, D,
                                  r->heads, b.O, L));
    IVC_TRY(launch_gemv(b.O, D, T, D, static_cast<const bf16*>(r->Wo[l]),
                        static_cast<const bf16*>(r->bo[l]), D, b.q, D, 0, L));
  }
  return gating_and_route(T, image_offsets, I, r, gate, mask, offsets, total, b, L);
}

// The Gating as one cooperative kernel (ivc_router_coop.cu) with
// IVC_GATING_FUSED=1. Off by default: beside the connector (16 CTAs on the
// SMs it leaves free) it measured 66 us per call against its 13 separate
// launches, which overlap through programmatic dependent launch (dual flow
// 0.399 vs 0.379 ms per call on the 13-tile image).
bool gating_fused_wanted() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_GATING_FUSED");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

// Gating on the pooled vectors (in b.q), the 2-way head, then routing.
int gating_and_route(int T, const int32_t* image_offsets, int I, const ivc_router* r, float* gate,
                     uint8_t* mask, int32_t* offsets, int32_t* total, const RouteBufs& b,
                     const Launch& L) {
  const int D = r->D;
  const int G = r->gate_hidden;
  if (gating_fused_wanted() && gating_fused_supported(D, G)) {
    // the whole Gating MLP and its softmax head in one cooperative launch
    IVC_TRY(launch_gating_fused(b.q, T, D, G, r, b.h, b.u1, b.u2, gate, b.bar, L));
    return launch_route(gate, T, image_offsets, I, r->rel_q, r->abs_t, r->quantile_scope, mask,
                        offsets, total, L);
  }
  for (int k = 0; k < 4; ++k) {
    IVC_TRY(launch_gemv(b.q, D, T, D, static_cast<const bf16*>(r->gW1[k]),
                        static_cast<const bf16*>(r->gb1[k]), G, b.u1, G, 1, L));
    IVC_TRY(launch_gemv(b.u1, G, T, G, static_cast<const bf16*>(r->gW2[k]),
                        static_cast<const bf16*>(r->gb2[k]), D, b.u2, D, 0, L));
    IVC_TRY(launch_residual_ln(b.q, b.u2, static_cast<const bf16*>(r->gln_g[k]),
                               static_cast<const bf16*>(r->gln_b[k]), T, D, r->gate_residual, L));
  }
  IVC_TRY(launch_gate_head(b.q, static_cast<const bf16*>(r->gWout),
                           static_cast<const bf16*>(r->gbout), T, D, gate, L));
  return launch_route(gate, T, image_offsets, I, r->rel_q, r->abs_t, r->quantile_scope, mask,
                      offsets, total, L);
}

// Connector GEMMs beside the router in ivc_flash_compress: SMs they leave to
// the router's small kernels (IVC_DUAL_RESERVE, default 36). With the
// connector's Linears in one persistent launch the router is the longer of
// the two: 0.382 / 0.377 / 0.367 / 0.352 / 0.353 ms per call on the 13-tile
// image for 12 / 20 / 28 / 36 / 44 SMs. IVC_DUAL_MLP2_FIRST=1 puts mlp2
// before mlp1 when the Linears run as separate launches.
int dual_reserve_sms() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_DUAL_RESERVE");
    v = e ? std::atoi(e) : 36;
    if (v < 0) v = 0;
  }
  return v;
}
bool dual_mlp2_first() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_DUAL_MLP2_FIRST");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

// Side stream (highest priority) and fork/join events used by
// ivc_flash_compress to run the router next to the connector, created once
// per device. The router's kernels are small and latency-bound; at high
// priority they take SMs as soon as connector GEMM CTAs retire.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

int side_stream(SideStream** out) {
  static std::mutex mu;
  static SideStream per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return IVC_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  SideStream& s = per_dev[dev];
  if (!s.stream) {
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return IVC_ECUDA;
    if (cudaStreamCreateWithPriority(&s.stream, cudaStreamNonBlocking, hi) != cudaSuccess)
      return IVC_ECUDA;
    if (cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess)
      return IVC_ECUDA;
  }
  *out = &s;
  return IVC_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return IVC_EINVAL;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return IVC_EALIGN;
  if (ws_bytes < need) return IVC_EWORKSPACE;
  return IVC_OK;
}

size_t ps_ws(int T, const ivc_mlp* m, bool half) {
  Carver cv(nullptr);
  PsBufs b;
  carve_ps(cv, m, static_cast<long long>(T) * (half ? 256 : 64), true, b);
  return cv.off;
}

size_t route_ws(int T, const ivc_router* r) {
  Carver cv(nullptr);
  RouteBufs b;
  carve_route(cv, r, T, b);
  return cv.off;
}

// Routed tile lists of the router-first flow: list_u, base_u, list_c,
// base_c [T] and the two counts.
struct ListBufs {
  int* list_u;
  int* base_u;
  int* list_c;
  int* base_c;
  int* counts;
};

void carve_lists(Carver& cv, int T, ListBufs& l) {
  l.list_u = cv.take<int>(T);
  l.base_u = cv.take<int>(T);
  l.list_c = cv.take<int>(T);
  l.base_c = cv.take<int>(T);
  l.counts = cv.take<int>(2);
}

// One layout for both flash flows (dual path and router-first), so that one
// workspace size serves either entry point.
struct FlashBufs {
  PsBufs b1, b2;
  bf16* Y256;
  bf16* Y64;
  RouteBufs br;
  ListBufs lists;
  int* done;
};

void carve_flash(Carver& cv, int T, const ivc_mlp* m1, const ivc_mlp* m2, const ivc_router* r,
                 FlashBufs& f) {
  carve_ps(cv, m1, static_cast<long long>(T) * 256, true, f.b1);
  carve_ps(cv, m2, static_cast<long long>(T) * 64, true, f.b2);
  f.Y256 = cv.take<bf16>(static_cast<size_t>(T) * 256 * m1->dims[m1->n_linear]);
  f.Y64 = cv.take<bf16>(static_cast<size_t>(T) * 64 * m2->dims[m2->n_linear]);
  carve_route(cv, r, T, f.br);
  carve_lists(cv, T, f.lists);
  // one split-K scratch for all connector GEMMs (they run one after another)
  f.b1.split_part = f.b2.split_part = cv.take<float>(splitk_part_floats());
  f.b1.split_s = f.b2.split_s = cv.take<int>(4);
  // row-block counters of both MLPs' Linears in one launch
  f.done = cv.take<int>(static_cast<size_t>(T) * m1->n_linear +
                        static_cast<size_t>((T * 64 + 255) / 256) * m2->n_linear);
}

size_t flash_ws(int T, const ivc_mlp* m1, const ivc_mlp* m2, const ivc_router* r) {
  Carver cv(nullptr);
  FlashBufs f;
  carve_flash(cv, T, m1, m2, r, f);
  return cv.off;
}

int ps_args_ok(const void* x, int T, int C, const ivc_mlp* m, bool half) {
  if (T < 0 || C <= 0) return IVC_EINVAL;
  if (!m) return IVC_EINVAL;
  if (C % 64 != 0 || !mlp_shape_ok(m)) return IVC_EUNSUPPORTED;
  if (m->dims[0] != (half ? 4 : 16) * C) return IVC_EUNSUPPORTED;
  if (static_cast<long long>(T) * 256 > 0x7fffffffLL) return IVC_EUNSUPPORTED;
  if (T > 0 && !x) return IVC_EINVAL;
  if (!aligned16(x)) return IVC_EALIGN;
  return mlp_ptrs_ok(m);
}

}  // namespace

extern "C" {

const char* ivc_strerror(int status) {
  switch (status) {
    case IVC_OK: return "ok";
    case IVC_EINVAL: return "invalid argument";
    case IVC_EUNSUPPORTED: return "unsupported shape";
    case IVC_EWORKSPACE: return "workspace too small";
    case IVC_ECUDA: return "CUDA call failed";
    case IVC_EDEVICE: return "device status word set";
    case IVC_EALIGN: return "pointer not 16-byte aligned";
    default: return "unknown status";
  }
}

int ivc_version(void) { return 100; }

size_t ivc_workspace_size(int op, int T, int C, const ivc_mlp* m, const ivc_mlp* m2,
                          const ivc_router* r) {
  if (T < 0 || C <= 0) return 0;
  switch (op) {
    case IVC_OP_PS_PROJECT_HALF:
      return mlp_shape_ok(m) ? ps_ws(T, m, true) : 0;
    case IVC_OP_PS_PROJECT_QUARTER:
      return mlp_shape_ok(m) ? ps_ws(T, m, false) : 0;
    case IVC_OP_VIR_ROUTE:
      return router_shape_ok(r, C) == IVC_OK ? route_ws(T, r) : 0;
    case IVC_OP_FLASH_COMPRESS:
      if (!mlp_shape_ok(m) || !mlp_shape_ok(m2) || router_shape_ok(r, C) != IVC_OK) return 0;
      return flash_ws(T, m, m2, r);
    default:
      return 0;
  }
}

size_t ivc_mlp_fold_size(const ivc_mlp* m) {
  if (!mlp_shape_ok(m)) return 0;
  return align_up(static_cast<size_t>(m->dims[1]) * m->dims[0] * sizeof(bf16)) +
         2 * align_up(static_cast<size_t>(m->dims[1]) * sizeof(float));
}

int ivc_mlp_fold(ivc_mlp* m, void* dst, size_t dst_bytes, ivc_stream_t stream) {
  if (!m || !dst) return IVC_EINVAL;
  if (!mlp_shape_ok(m)) return IVC_EUNSUPPORTED;
  if (!m->ln_gamma || !m->ln_beta || !m->W[0]) return IVC_EINVAL;
  if (reinterpret_cast<uintptr_t>(dst) % kAlign) return IVC_EALIGN;
  if (dst_bytes < ivc_mlp_fold_size(m)) return IVC_EWORKSPACE;
  char* p = static_cast<char*>(dst);
  bf16* W0 = reinterpret_cast<bf16*>(p);
  p += align_up(static_cast<size_t>(m->dims[1]) * m->dims[0] * sizeof(bf16));
  float* cs = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(m->dims[1]) * sizeof(float));
  float* fb = reinterpret_cast<float*>(p);
  Launch L{static_cast<cudaStream_t>(stream), nullptr};
  IVC_TRY(launch_fold(static_cast<const bf16*>(m->W[0]), static_cast<const bf16*>(m->b[0]),
                      static_cast<const bf16*>(m->ln_gamma), static_cast<const bf16*>(m->ln_beta),
                      m->dims[1], m->dims[0], W0, cs, fb, L));
  m->fold_W0 = W0;
  m->fold_colsum = cs;
  m->fold_bias = fb;
  return IVC_OK;
}

// ivc_router_fold: the weights checked as for a call, the fold fields aside.
static int router_fold_shape(const ivc_router* r) {
  if (!r) return IVC_EINVAL;
  ivc_router w = *r;
  w.fold_u1 = nullptr;
  w.fold_c1 = nullptr;
  for (int l = 0; l < 3; ++l) {
    w.fold_wqo[l] = nullptr;
    w.fold_bqo[l] = nullptr;
  }
  IVC_TRY(router_shape_ok(&w, w.D));
  if (w.pool_mode != IVC_POOL_FOLDED || w.D % 64 != 0) return IVC_EUNSUPPORTED;
  return IVC_OK;
}

size_t ivc_router_fold_size(const ivc_router* r) {
  if (router_fold_shape(r) != IVC_OK) return 0;
  const size_t D = static_cast<size_t>(r->D);
  return align_up(D * sizeof(float)) + align_up(32 * D * sizeof(bf16)) +
         align_up(16 * sizeof(float)) +
         3 * (align_up(2 * D * D * sizeof(bf16)) + align_up(D * sizeof(float)));
}

int ivc_router_fold(ivc_router* r, void* dst, size_t dst_bytes, ivc_stream_t stream) {
  if (!r || !dst) return IVC_EINVAL;
  IVC_TRY(router_fold_shape(r));
  if (reinterpret_cast<uintptr_t>(dst) % kAlign) return IVC_EALIGN;
  if (dst_bytes < ivc_router_fold_size(r)) return IVC_EWORKSPACE;
  const int D = r->D;
  const size_t Dz = static_cast<size_t>(D);
  char* p = static_cast<char*>(dst);
  float* q1 = reinterpret_cast<float*>(p);
  p += align_up(Dz * sizeof(float));
  bf16* u1 = reinterpret_cast<bf16*>(p);
  p += align_up(32 * Dz * sizeof(bf16));
  float* c1 = reinterpret_cast<float*>(p);
  p += align_up(16 * sizeof(float));
  bf16* wqo[3];
  float* bqo[3];
  for (int l = 0; l < 3; ++l) {
    wqo[l] = reinterpret_cast<bf16*>(p);
    p += align_up(2 * Dz * Dz * sizeof(bf16));
    bqo[l] = reinterpret_cast<float*>(p);
    p += align_up(Dz * sizeof(float));
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  Launch L{s, nullptr};
  IVC_TRY(launch_gemv_bf16x(static_cast<const bf16*>(r->query), D,
                            static_cast<const bf16*>(r->Wq[0]), static_cast<const bf16*>(r->bq[0]),
                            D, q1, L));
  IVC_TRY(launch_pool_fold_query(q1, 0, 1, static_cast<const bf16*>(r->Wk[0]),
                                 static_cast<const bf16*>(r->bk[0]), D, u1, c1, L));
  for (int l = 0; l < 3; ++l)
    IVC_TRY(launch_wq_wo_fold(static_cast<const bf16*>(r->Wq[l + 1]),
                              static_cast<const bf16*>(r->bq[l + 1]),
                              static_cast<const bf16*>(r->Wo[l]), static_cast<const bf16*>(r->bo[l]),
                              D, wqo[l], bqo[l], s));
  r->fold_u1 = u1;
  r->fold_c1 = c1;
  for (int l = 0; l < 3; ++l) {
    r->fold_wqo[l] = wqo[l];
    r->fold_bqo[l] = bqo[l];
  }
  return IVC_OK;
}

int ivc_ps_project(const void* x, int T, int C, float scale, int flags, const ivc_mlp* m,
                   void* y, void* workspace, size_t ws_bytes, ivc_stream_t stream) {
  const bool half = scale == 0.5f;
  if (!half && scale != 0.25f) return IVC_EINVAL;
  if (flags & ~(IVC_PS_V1 | IVC_PS_QUARTER_TWICE)) return IVC_EINVAL;
  IVC_TRY(ps_args_ok(x, T, C, m, half));
  if (T > 0 && !y) return IVC_EINVAL;
  if (!aligned16(y)) return IVC_EALIGN;
  IVC_TRY(check_ws(workspace, ws_bytes, ps_ws(T, m, half)));
  if (T == 0) return IVC_OK;
  Launch L{static_cast<cudaStream_t>(stream), static_cast<int*>(workspace)};
  Carver cv(workspace);
  PsBufs b;
  const long long rows = static_cast<long long>(T) * (half ? 256 : 64);
  carve_ps(cv, m, rows, true, b);
  std::vector<GraphProblemCall> probs;
  if (gemm_graph_enabled())
    mlp_problems(x, T, C, half, flags, m, nullptr, nullptr, nullptr, static_cast<bf16*>(y), b,
                 probs);
  if (!probs.empty() && graph_supported(probs.data(), static_cast<int>(probs.size()))) {
    // fold (if needed), counters, statistics, then every Linear in one
    // launch that overlaps the statistics kernel's tail
    const bf16* W0;
    const float *cs, *fb;
    IVC_TRY(folded_weights(m, b, L, &W0, &cs, &fb));
    probs[0].B = W0;
    probs[0].colsum = cs;
    probs[0].fbias = fb;
    const int n_ctr = graph_counters(probs.data(), static_cast<int>(probs.size()));
    IVC_TRY(cu_check(cudaMemsetAsync(b.done, 0, sizeof(int) * n_ctr, L.stream)));
    IVC_TRY(launch_ps_stats(static_cast<const bf16*>(x), T, C, half ? b.mean : nullptr,
                            half ? b.rstd : nullptr, half ? nullptr : b.mean,
                            half ? nullptr : b.rstd, L));
    return launch_gemm_graph(probs.data(), static_cast<int>(probs.size()), b.done, 0, L);
  }
  IVC_TRY(launch_ps_stats(static_cast<const bf16*>(x), T, C, half ? b.mean : nullptr,
                          half ? b.rstd : nullptr, half ? nullptr : b.mean,
                          half ? nullptr : b.rstd, L));
  return ps_mlp(x, T, C, half, flags, m, static_cast<bf16*>(y), b, L);
}

int ivc_vir_route(const void* x, const int32_t* valid_len, int T, int C,
                  const int32_t* image_offsets, int I, const ivc_router* r, float* gate,
                  uint8_t* mask, int32_t* offsets, void* workspace, size_t ws_bytes,
                  ivc_stream_t stream) {
  if (T < 0 || C <= 0 || I < 0) return IVC_EINVAL;
  IVC_TRY(router_shape_ok(r, C));
  if (!offsets || (T > 0 && (!x || !gate || !mask))) return IVC_EINVAL;
  if (T > 0 && r->quantile_scope == 0 && !image_offsets) return IVC_EINVAL;
  if (!aligned16(x)) return IVC_EALIGN;
  IVC_TRY(check_ws(workspace, ws_bytes, route_ws(T, r)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) return cu_check(cudaMemsetAsync(offsets, 0, sizeof(int32_t), s));
  Launch L{s, static_cast<int*>(workspace)};
  Carver cv(workspace);
  RouteBufs b;
  carve_route(cv, r, T, b);
  return route_impl(x, valid_len, T, image_offsets, I, r, gate, mask, offsets, nullptr, b, L,
                    false);
}

int ivc_route(const float* gate, int T, const int32_t* image_offsets, int I, double rel_q,
              double abs_t, int scope, uint8_t* mask, int32_t* offsets, int32_t* total,
              void* workspace, size_t ws_bytes, ivc_stream_t stream) {
  if (T < 0 || I < 0 || (scope != 0 && scope != 1)) return IVC_EINVAL;
  if (!(rel_q >= 0.0 && rel_q <= 1.0)) return IVC_EINVAL;
  if (!offsets || (T > 0 && (!gate || !mask))) return IVC_EINVAL;
  if (T > 0 && scope == 0 && !image_offsets) return IVC_EINVAL;
  IVC_TRY(check_ws(workspace, ws_bytes, IVC_ROUTE_WORKSPACE_BYTES));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    IVC_TRY(cu_check(cudaMemsetAsync(offsets, 0, sizeof(int32_t), s)));
    return total ? cu_check(cudaMemsetAsync(total, 0, sizeof(int32_t), s)) : IVC_OK;
  }
  Launch L{s, static_cast<int*>(workspace)};
  return launch_route(gate, T, image_offsets, I, rel_q, abs_t, scope, mask, offsets, total, L);
}

int ivc_flash_compress(const void* x, const int32_t* valid_len, int T, int C,
                       const int32_t* image_offsets, int I, const ivc_mlp* mlp1,
                       const ivc_mlp* mlp2, const ivc_router* r, void* out, float* gate,
                       uint8_t* mask, int32_t* offsets, int32_t* total, void* workspace,
                       size_t ws_bytes, ivc_stream_t stream) {
  if (T < 0 || C <= 0 || I < 0) return IVC_EINVAL;
  IVC_TRY(ps_args_ok(x, T, C, mlp1, true));
  IVC_TRY(ps_args_ok(x, T, C, mlp2, false));
  const int H = mlp1->dims[mlp1->n_linear];
  if (mlp2->dims[mlp2->n_linear] != H) return IVC_EUNSUPPORTED;
  IVC_TRY(router_shape_ok(r, C));
  if (!offsets || !total || (T > 0 && (!out || !gate || !mask))) return IVC_EINVAL;
  if (T > 0 && r->quantile_scope == 0 && !image_offsets) return IVC_EINVAL;
  if (!aligned16(out)) return IVC_EALIGN;
  IVC_TRY(check_ws(workspace, ws_bytes, flash_ws(T, mlp1, mlp2, r)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    IVC_TRY(cu_check(cudaMemsetAsync(offsets, 0, sizeof(int32_t), s)));
    return cu_check(cudaMemsetAsync(total, 0, sizeof(int32_t), s));
  }
  Launch L{s, static_cast<int*>(workspace)};
  Carver cv(workspace);
  FlashBufs f;
  carve_flash(cv, T, mlp1, mlp2, r, f);
  const PsBufs& b1 = f.b1;
  const PsBufs& b2 = f.b2;
  bf16* Y256 = f.Y256;
  bf16* Y64 = f.Y64;
  const RouteBufs& br = f.br;
  // The router (own buffers) runs on the side stream while the connector runs
  // on the caller's stream; they meet before compaction.
  SideStream* side = nullptr;
  IVC_TRY(side_stream(&side));
  Launch R{side->stream, L.status};
  IVC_TRY(cu_check(cudaEventRecord(side->fork, s)));
  IVC_TRY(cu_check(cudaStreamWaitEvent(side->stream, side->fork, 0)));
  int rc =
      route_impl(x, valid_len, T, image_offsets, I, r, gate, mask, offsets, total, br, R, false);
  // join even on failure so that the caller's stream never runs ahead of work
  // already enqueued on the side stream
  const int rc_rec = cu_check(cudaEventRecord(side->join, side->stream));
  if (rc == IVC_OK) rc = rc_rec;
  const int reserve = dual_reserve_sms();
  // both MLPs' Linears in one persistent launch, in the priority order
  // mlp2.fc1, mlp1.fc1, mlp2.fc2, mlp1.fc2, mlp2.fc3 (the long first Linear
  // of mlp2 first; each later Linear right after its input's)
  std::vector<GraphProblemCall> p1, p2, probs;
  std::vector<int> pos1, pos2;
  if (gemm_graph_enabled()) {
    mlp_problems(x, T, C, true, 0, mlp1, nullptr, nullptr, nullptr, Y256, b1, p1);
    mlp_problems(x, T, C, false, 0, mlp2, nullptr, nullptr, nullptr, Y64, b2, p2);
    pos1.resize(p1.size());
    pos2.resize(p2.size());
    for (size_t i = 0; i < p1.size() || i < p2.size(); ++i) {
      if (i < p2.size()) {
        pos2[i] = static_cast<int>(probs.size());
        probs.push_back(p2[i]);
        if (p2[i].dep >= 0) probs.back().dep = pos2[p2[i].dep];
      }
      if (i < p1.size()) {
        pos1[i] = static_cast<int>(probs.size());
        probs.push_back(p1[i]);
        if (p1[i].dep >= 0) probs.back().dep = pos1[p1[i].dep];
      }
    }
  }
  if (rc == IVC_OK && !probs.empty() &&
      graph_supported(probs.data(), static_cast<int>(probs.size()))) {
    const bf16 *W01, *W02;
    const float *cs1, *fb1, *cs2, *fb2;
    rc = folded_weights(mlp1, b1, L, &W01, &cs1, &fb1);
    if (rc == IVC_OK) rc = folded_weights(mlp2, b2, L, &W02, &cs2, &fb2);
    probs[pos1[0]].B = W01;
    probs[pos1[0]].colsum = cs1;
    probs[pos1[0]].fbias = fb1;
    probs[pos2[0]].B = W02;
    probs[pos2[0]].colsum = cs2;
    probs[pos2[0]].fbias = fb2;
    const int n_ctr = graph_counters(probs.data(), static_cast<int>(probs.size()));
    if (rc == IVC_OK) rc = cu_check(cudaMemsetAsync(f.done, 0, sizeof(int) * n_ctr, s));
    if (rc == IVC_OK)
      rc = launch_ps_stats(static_cast<const bf16*>(x), T, C, b1.mean, b1.rstd, b2.mean, b2.rstd,
                           L);
    if (rc == IVC_OK)
      rc = launch_gemm_graph(probs.data(), static_cast<int>(probs.size()), f.done, reserve, L);
  } else if (rc == IVC_OK) {
    // one launch per Linear (IVC_GEMM_GRAPH=0)
    rc = launch_ps_stats(static_cast<const bf16*>(x), T, C, b1.mean, b1.rstd, b2.mean, b2.rstd, L);
    const bool mlp2_first = dual_mlp2_first();
    for (int k = 0; k < 2 && rc == IVC_OK; ++k) {
      if ((k == 0) == mlp2_first)
        rc = ps_mlp(x, T, C, false, 0, mlp2, Y64, b2, L, nullptr, reserve);
      else
        rc = ps_mlp(x, T, C, true, 0, mlp1, Y256, b1, L, nullptr, reserve);
    }
  }
  const int rc_wait = rc_rec == IVC_OK ? cu_check(cudaStreamWaitEvent(s, side->join, 0)) : rc_rec;
  if (rc != IVC_OK) return rc;
  if (rc_wait != IVC_OK) return rc_wait;
  return launch_compact(Y256, Y64, mask, offsets, T, H, static_cast<bf16*>(out), L);
}

int ivc_flash_compress_routed(const void* x, const int32_t* valid_len, int T, int C,
                              const int32_t* image_offsets, int I, const ivc_mlp* mlp1,
                              const ivc_mlp* mlp2, const ivc_router* r, void* out, float* gate,
                              uint8_t* mask, int32_t* offsets, int32_t* total, void* workspace,
                              size_t ws_bytes, ivc_stream_t stream) {
  if (T < 0 || C <= 0 || I < 0) return IVC_EINVAL;
  IVC_TRY(ps_args_ok(x, T, C, mlp1, true));
  IVC_TRY(ps_args_ok(x, T, C, mlp2, false));
  const int H = mlp1->dims[mlp1->n_linear];
  if (mlp2->dims[mlp2->n_linear] != H) return IVC_EUNSUPPORTED;
  IVC_TRY(router_shape_ok(r, C));
  if (!offsets || !total || (T > 0 && (!out || !gate || !mask))) return IVC_EINVAL;
  if (T > 0 && r->quantile_scope == 0 && !image_offsets) return IVC_EINVAL;
  if (!aligned16(out)) return IVC_EALIGN;
  IVC_TRY(check_ws(workspace, ws_bytes, flash_ws(T, mlp1, mlp2, r)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    IVC_TRY(cu_check(cudaMemsetAsync(offsets, 0, sizeof(int32_t), s)));
    return cu_check(cudaMemsetAsync(total, 0, sizeof(int32_t), s));
  }
  Launch L{s, static_cast<int*>(workspace)};
  Carver cv(workspace);
  FlashBufs f;
  carve_flash(cv, T, mlp1, mlp2, r, f);
  // Router first: it needs only x. Then each tile runs through the path it
  // was routed to, and the last Linear of each MLP stores its rows at the
  // tile's output offset, so no compaction pass remains.
  IVC_TRY(launch_ps_stats(static_cast<const bf16*>(x), T, C, f.b1.mean, f.b1.rstd, f.b2.mean,
                          f.b2.rstd, L));
  IVC_TRY(route_impl(x, valid_len, T, image_offsets, I, r, gate, mask, offsets, total, f.br, L,
                     false));
  const ListBufs& lb = f.lists;
  IVC_TRY(launch_route_lists(mask, offsets, T, lb.list_u, lb.base_u, lb.list_c, lb.base_c,
                             lb.counts, L));
  const Routed ru{lb.list_u, lb.counts, lb.base_u};
  const Routed rc{lb.list_c, lb.counts + 1, lb.base_c};
  IVC_TRY(ps_mlp(x, T, C, true, 0, mlp1, static_cast<bf16*>(out), f.b1, L, &ru));
  return ps_mlp(x, T, C, false, 0, mlp2, static_cast<bf16*>(out), f.b2, L, &rc);
}

int ivc_set_router_wait_limit(long long cycles) {
  if (cycles < 0) return IVC_EINVAL;
  set_router_late_wait_cycles(cycles);
  return IVC_OK;
}

int ivc_device_status(void* workspace, int* bits, ivc_stream_t stream) {
  if (!workspace || !bits) return IVC_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return IVC_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return IVC_ECUDA;
  if (v != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(int), s) != cudaSuccess) return IVC_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return IVC_ECUDA;
  }
  *bits = v;
  return v ? IVC_EDEVICE : IVC_OK;
}

}  // extern "C"
