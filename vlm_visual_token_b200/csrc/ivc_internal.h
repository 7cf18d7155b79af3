// ivc_internal.h — host-side launchers shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "ivc.h"

namespace ivc {

typedef __nv_bfloat16 bf16;

// Status word bits (mirror enum ivc_device_bits).
constexpr int DEV_BAD_VALID_LEN = IVC_DEV_BAD_VALID_LEN;
constexpr int DEV_BAD_OFFSETS = IVC_DEV_BAD_OFFSETS;
constexpr int DEV_WAIT_TIMEOUT = IVC_DEV_WAIT_TIMEOUT;
constexpr int DEV_GROUP_TOO_LARGE = IVC_DEV_GROUP_TOO_LARGE;
constexpr int DEV_BAD_PROMPT = IVC_DEV_BAD_PROMPT;

struct Launch {
  cudaStream_t stream;
  int* status;     // device status word (workspace header)
  int sm_budget;   // > 0: SMs a persistent kernel may assume free (beside other work); 0: all
};

// Brackets one kernel launch with CUDA events when tracing is on (ivc_trace.cu).
class TraceScope {
 public:
  TraceScope(const char* name, cudaStream_t s);
  ~TraceScope();
  TraceScope(const TraceScope&) = delete;
  TraceScope& operator=(const TraceScope&) = delete;

 private:
  cudaStream_t stream_;
  bool active_;
  size_t idx_ = 0;
};

// Converts a CUDA error into IVC_ECUDA (and remembers nothing else).
inline int cu_check(cudaError_t e) { return e == cudaSuccess ? IVC_OK : IVC_ECUDA; }

// Launches `kern` with programmatic stream serialisation (see pdl_wait in
// ivc_ptx.cuh) and, when cluster_x > 1, thread-block clusters of cluster_x.
template <typename... KArgs, typename... Args>
inline int launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                    int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cu_check(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
}

// -------------------------------------------------------------- connector
// Per-row LayerNorm statistics of the pixel-shuffled rows, read straight
// from the [T,32,32,C] features: mean/rstd of every factor-0.5 row
// (T*256 rows of 4C values) and/or every factor-0.25 row (T*64 rows of 16C).
int launch_ps_stats(const bf16* x, int T, int C, float* mean_half, float* rstd_half,
                    float* mean_quarter, float* rstd_quarter, const Launch& L);

// LayerNorm affine fold into the first Linear (see ivc_mlp_fold).
int launch_fold(const bf16* W, const bf16* b, const bf16* gamma, const bf16* beta, int N, int K,
                bf16* W_out, float* colsum, float* fbias, const Launch& L);

// One GEMM of the connector or of the pooling projections.
struct GemmCall {
  const char* tag;     // role, for tracing ("mlp1.fc1", "pool.kv", ...)
  int a_mode;          // AMode
  const void* a;       // A base (features for the pixel_shuffle modes)
  int T, C;            // pixel_shuffle modes
  int M, N, K;
  int groups;          // >1: group g uses B[g], bias[g], output column offset g*N
  const void* B[8];
  int b_mode;          // BMode: K-major 2-D (default), K-major 3-D batched, MN-major 3-D
  int b_batch_rows;    // 3-D modes: rows of A (multiple of 128) per B batch
  int b_batches;       // 3-D modes: number of batches
  long long b_ld;      // 3-D modes: elements between consecutive rows (K-major: n; MN: k)
  long long b_batch_stride;  // 3-D modes: elements between batches
  const bf16* bias[8];
  int epi_mode;        // EpiMode
  int gelu;
  int remap;
  const float* colsum;
  const float* fbias;
  const float* row_mean;
  const float* row_rstd;
  void* out;
  int out_f32;         // store fp32 (pooling K/V) instead of bf16
  int m_valid;         // >0: store only rows with (row % 128) < m_valid
  long long ldo;
  // routed rows (router-first flow; GemmArgs in ivc_gemm.cuh): M is then the
  // upper bound T * item_rows, the device count decides
  const int* list;
  const int* list_count;
  const int* out_base;
  int item_rows;
  int stats_remap;
  // split-K scratch (optional): splitk_part_floats() fp32 values and one int
  float* split_part;
  int* split_s;
  // SMs to leave to concurrent work (the router beside the connector) when
  // that does not add a round of output tiles; 0 = use every SM
  int reserve_sms;
  // only the epilogue reads what the previous kernel wrote (GemmArgs)
  int epi_dep_only;
};
int launch_gemm(const GemmCall& c, const Launch& L);

// Several connector Linears in one persistent launch (ivc_gemm_graph.cuh).
// Problems are given in priority order; `dep` names an earlier problem whose
// output rows (256-row block m) tile row block m reads (its A operand), or -1.
// Every problem uses 256 x 256 tiles on CTA pairs, K-major weights and a bf16
// output; `done` holds graph_counters() ints that must be zero at launch.
struct GraphProblemCall {
  int a_mode;          // AMode
  const void* a;       // A base (features for the pixel_shuffle modes)
  int T, C;            // pixel_shuffle modes
  int M, N, K;
  const void* B;       // nn.Linear weight [N, K]
  const bf16* bias;    // EPI_BIAS (may be null)
  int epi_mode, gelu, remap;
  const float* colsum;
  const float* fbias;
  const float* row_mean;
  const float* row_rstd;
  void* out;
  long long ldo;
  int dep;
  int wide;            // 1: 256 x 512 tiles if the problem has many rounds of
                       // 256-wide tiles; 2: 256 x 512 tiles
};
int launch_gemm_graph(const GraphProblemCall* probs, int n, int* done, int reserve_sms,
                      const Launch& L);
// Row-block counters launch_gemm_graph needs for these problems.
int graph_counters(const GraphProblemCall* probs, int n);
// Whether launch_gemm_graph takes these problems: K a multiple of 128 (two
// k-blocks per stage), C a multiple of 128 for the pixel_shuffle views, N a
// multiple of 32, dependencies on earlier problems with the same rows.
bool graph_supported(const GraphProblemCall* probs, int n);
// Size of the split-K partial buffer: enough for any GEMM shape on this device.
size_t splitk_part_floats();

// -------------------------------------------------------------- router
// Y[m, n] = act(sum_k X[m, k] W[n, k] + b[n]); X fp32 [M, ldx], W bf16 [N, K].
int launch_gemv(const float* X, long long ldx, int M, int K, const bf16* W, const bf16* b, int N,
                float* Y, long long ldy, int gelu, const Launch& L);
// Same with a bf16 input vector broadcast (M = 1).
// Y = X P^T + c with P an fp32 matrix stored as bf16 hi | lo per row
// (W2 [N, 2K]) and an fp32 bias c.
int launch_gemv_split(const float* X, long long ldx, int M, int K, const bf16* W2,
                      const float* bf, int N, float* Y, long long ldy, const Launch& L);
// Once per weight set: P = Wq Wo as a bf16 hi | lo pair per row (P2 [D, 2D])
// and c = Wq bo + bq (fp32 [D]).
int launch_wq_wo_fold(const bf16* Wq, const bf16* bq, const bf16* Wo, const bf16* bo, int D,
                      bf16* P2, float* c, cudaStream_t stream);
int launch_gemv_bf16x(const bf16* x, int K, const bf16* W, const bf16* b, int N, float* Y,
                      const Launch& L);
// Masked single-query multi-head attention of one pooling layer.
int launch_pool_attention(const float* Q, long long ldq, const float* KV, long long ldkv,
                          int koff, int voff, const int32_t* valid_len, int T, int D, int heads,
                          float* O, const Launch& L);
// Folded pooling (up to 16 heads of 64): u/c of one layer from Q [Tq, D] (Tq = 1:
// the same query for every tile); in the tensor-core form the scores' softmax
// into the split P2 operand and o = Wv z + bv from the split weighted sums
// Z [T*128, D].
int launch_pool_fold_query(const float* Q, long long ldq, int Tq, const bf16* Wk, const bf16* bk,
                           int D, bf16* U2, float* cb, const Launch& L);
int launch_pool_softmax(const float* S, const float* cb, int cb_stride, const int32_t* valid_len,
                        int T, int heads, bf16* P2, const Launch& L);
int launch_pool_vproj(const float* Z, int T, int D, const bf16* Wv, const bf16* bv, float* O,
                      const Launch& L);
// The same scores, softmax and weighted sums in one pass over x (two
// launches): per 128-token chunk unnormalised sums Zp [T*8*16, D] and their
// running max / sum (stats: 2 * T*8*16 floats), merged into z [T*16, D];
// then o = Wv z + bv reads z row (tile*16 + head).
// The same chunk partials from the tensor-core (tcgen05) form of the
// attention (ivc_attend_tc.cu), selected inside launch_pool_attend with
// IVC_ATTEND_TC=1.
bool attend_tc_wanted();
int launch_pool_attend_tc(const void* x, const bf16* U2, int Tq, const float* cb,
                          const int32_t* valid_len, int T, int D, int heads, float* Zp,
                          float* stats, const Launch& L);
// combine = false: the chunk partials are left for launch_pool_tail to merge.
// allow_tc = false: the mma.sync form even where the tcgen05 one is selected.
int launch_pool_attend(const void* x, const bf16* U2, int Tq, const float* cb,
                       const int32_t* valid_len, int T, int D, int heads, float* Zp, float* stats,
                       float* z, const Launch& L, bool combine = true, bool allow_tc = true);
// The tcgen05 attention's partials per tile and the shapes it takes.
int pool_attend_tc_chunks();
bool pool_attend_tc_supported(int D, int heads);
// The tail of folded pooling layer l as one cooperative launch of D/64 CTAs
// (ivc_router_coop.cu): merge of the chunk partials (Zp, stats as left by
// launch_pool_attend with combine = false), O = Wv z + bv, q = Wo O + bo, and
// unless l is the last layer Q = Wq' q + bq' and the next layer's folded key
// projection U2, cb. bar: one zeroed counter word.
bool pool_tail_supported(int D, int heads);
int launch_pool_tail(const ivc_router* r, int l, const float* Zp, const float* mstat,
                     const float* lstat, int T, float* O, float* q, float* Q, bf16* U2, float* cb,
                     unsigned* bar, const Launch& L);
int launch_pool_vproj_heads(const float* z, int T, int D, const bf16* Wv, const bf16* bv, float* O,
                            const Launch& L);
// Folded pooling through launch_pool_attend (default) or through the
// tensor-core scores / softmax / weighted-sum kernels (IVC_POOL_ATTEND=0).
bool pool_attend_wanted();
// The whole folded router (pooling, gating, routing) as one cooperative
// persistent kernel (ivc_router_fused.cu).
struct FusedRouterBufs {
  float* Q;
  bf16* U2;
  float* cb;
  float* stats;  // 2 * T*8*16 floats
  float* Zp;     // [T*8*16, D]
  float* z;
  float* O;
  float* q;
  float* h;
  float* u1;
  float* u2;
  unsigned* bar;
};
// Tensor map of a row-major [rows, cols] bf16 matrix, box 64 columns x
// box_rows rows, 128-byte swizzle (ivc_connector.cu).
int map_rows_2d(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows);

// Tensor map of a bf16 tensor of `rank` dims (innermost first; strides in
// bytes of dims 1..rank-1, in any order), box `box`, 128-byte swizzle.
int map_bf16(CUtensorMap* m, int rank, const void* base, const unsigned long long* dims,
             const unsigned long long* strides_bytes, const unsigned* box);
// Folded pooling can run as one persistent cooperative kernel (grid barriers
// between its phases) or as separate kernels. IVC_ROUTER_FUSED=1 / 0 forces
// the choice; otherwise the caller's default_on decides.
bool router_fused_wanted(bool default_on);
// The test limit of the persistent router's grid barriers after the gating
// (ivc_set_router_wait_limit): 0 = the default bound.
long long router_late_wait_cycles();
void set_router_late_wait_cycles(long long cycles);
bool router_fused_supported(const ivc_router* r);
int launch_router_fused(const ivc_router* r, const void* x, const int32_t* valid_len, int T,
                        const int32_t* image_offsets, int I, float* gate, uint8_t* mask,
                        int32_t* offsets, int32_t* total, const FusedRouterBufs& b,
                        const Launch& L);
// h[t] += LN(u[t]) * gamma + beta over D (inside = 1: h[t] = LN(h[t] + u[t]) ...).
int launch_residual_ln(float* h, const float* u, const bf16* gamma, const bf16* beta, int T,
                       int D, int inside, const Launch& L);
// The whole Gating (4 residual blocks and the softmax head) as one
// cooperative launch of up to 16 CTAs (ivc_gating.cu): pooled [T, D] in,
// gate [T, 2] out; h [T, D], u1 [T, G], u2 [T, D] scratch, bar one zeroed
// counter word.
bool gating_fused_supported(int D, int G);
int launch_gating_fused(const float* pooled, int T, int D, int G, const ivc_router* r, float* h,
                        float* u1, float* u2, float* gate, unsigned* bar, const Launch& L);
// gate[t] = softmax(Wout h[t] + bout), Wout [2, D].
int launch_gate_head(const float* h, const bf16* Wout, const bf16* bout, int T, int D,
                     float* gate, const Launch& L);
// From the routing mask and row offsets: the uncompressed tiles (list_u,
// their first output rows base_u) and the compressed ones (list_c, base_c),
// each in tile order; counts[0] = #uncompressed, counts[1] = #compressed.
int launch_route_lists(const uint8_t* mask, const int32_t* offsets, int T, int* list_u,
                       int* base_u, int* list_c, int* base_c, int* counts, const Launch& L);
// Quantile + double threshold + row-count scan.
int launch_route(const float* gate, int T, const int32_t* image_offsets, int I, double rel_q,
                 double abs_t, int scope, uint8_t* mask, int32_t* offsets, int32_t* total,
                 const Launch& L);
// out[offsets[t] + j] = mask[t] ? Y64[t*64 + j] : Y256[t*256 + j].
int launch_compact(const bf16* Y256, const bf16* Y64, const uint8_t* mask,
                   const int32_t* offsets, int T, int H, bf16* out, const Launch& L);

// SMs of the current device (queried once per device).
int num_sms();

// Raises `kern`'s dynamic shared-memory limit to at least `bytes` on the
// current device, once per (kernel, device) for the largest size asked so far
// (ivc_device_once.h). IVC_OK, or IVC_ECUDA when the attribute call fails.
int smem_optin(const void* kern, size_t bytes);

}  // namespace ivc
