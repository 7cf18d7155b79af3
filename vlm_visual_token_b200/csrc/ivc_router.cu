// ivc_router.cu — the Flash Visual Resolution Router (ViR) kernels for sm_100a.
//
// InternVL3_5-4B-Flash "Gating and CrossAttentionPooling" article:
//   section 2  CrossAttentionPooling — a learnable query refined by 4
//              multi-head cross-attention layers over a tile's tokens, pad
//              tokens masked out;
//   section 3  Gating — 4 residual blocks Linear -> GELU -> Dropout -> Linear
//              -> Dropout -> LayerNorm, then Linear(hidden, 2) and softmax;
//   section 4  gate > quantile(gate, 0.1) and gate >= 0.5 per image;
// InternVL3_5-2B-Flash dual-path article, "路由决策" (operators of the double
// threshold) and section 5 of the 4B-Flash article (tiles spliced back in
// order, 64 or 256 rows each).
//
// Two forms of the pooling, chosen by ivc_router.pool_mode:
//  * folded (default): the single query lets each layer's K and V
//    projections be reassociated onto the query (see "folded pooling"
//    below); per layer two thin tensor-core contractions with the raw
//    features, a masked softmax and skinny projections remain;
//  * literal: the K and V projections of all four layers are one grouped
//    tensor-core GEMM (ivc_gemm.cuh) with fp32 output, then a masked
//    softmax-weighted sum per (head, tile) over fp32 K/V (rounding K/V to
//    bf16 alone moves the gate probabilities by about 1e-3 on the 13-tile
//    workload).
// All router vectors between steps are fp32.
#include <cuda_runtime.h>

#include <cstdlib>
#include <type_traits>

#include "ivc_internal.h"
#include "ivc_ptx.cuh"

namespace ivc {

__device__ __forceinline__ float gelu_f(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

// ---------------------------------------------------------------- skinny GEMV
// Y[m, n] = act(sum_k X[m, k] W[n, k] + b[n]) for few rows m (router vectors),
// on the tensor cores (m16n8k16). A CTA of 8 warps owns 16 consecutive columns
// (two n8 tiles, so that each staged input row serves 16 columns). One thread
// brings their 16 weight rows (contiguous in W) into shared memory with one
// bulk copy issued before waiting for the previous kernel, and up to 16 input
// rows per round (one bulk copy per row) on the same mbarrier. Warp w
// multiplies the k-range [w K/8, (w+1) K/8): fp32 inputs are split into a bf16
// pair hi + lo (two MMAs per k-step, fp32 accumulate, about 16 significant
// bits of the input kept), bf16 inputs enter as they are. The 8 warps' partial
// tiles are summed through shared memory.
constexpr int GEMV_THREADS = 256;
constexpr int GEMV_WARPS = GEMV_THREADS / 32;
constexpr int GEMV_COLS = 16;  // output columns per CTA (two n8 tiles)
constexpr int GEMV_NT = GEMV_COLS / 8;
constexpr int GEMV_ROWS = 16;  // input rows per round

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4],
                                          const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// v = hi + lo, hi = bf16(v), lo = bf16(v - hi), two lanes per 32-bit word.
__device__ __forceinline__ void split2(float2 v, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 l = __floats2bfloat162_rn(v.x - __low2float(h), v.y - __high2float(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Where the input row of output row m comes from: row m of X (GV_PLAIN);
// Z[m*128 + h] + Z[m*128 + 16 + h] (GV_PAIRED: the split weighted sums of the
// tensor-core pooling form); z[m*16 + h] (GV_HEADROW: the combined weighted
// sums of the single-pass form); h = (first column of the CTA) / 64.
enum GemvRows { GV_PLAIN = 0, GV_PAIRED = 1, GV_HEADROW = 2 };

template <typename XT, int ROWS, bool WS = false>
struct GemvLayout {
  // staged input rows (padded by 8 elements), the weight rows (unpadded, one
  // copy; with split weights each row holds the hi and then the lo part), the
  // warps' partial tiles; after a 16-byte mbarrier slot
  __host__ __device__ static size_t x_bytes(int K) {
    return (ROWS == GV_PAIRED ? 2 : 1) * static_cast<size_t>(GEMV_ROWS) * (K + 8) * sizeof(XT);
  }
  __host__ __device__ static size_t w_bytes(int K) {
    return static_cast<size_t>(GEMV_COLS) * K * 2 * (WS ? 2 : 1);
  }
  __host__ __device__ static size_t total(int K) {
    return 16 + x_bytes(K) + w_bytes(K) + static_cast<size_t>(GEMV_WARPS) * GEMV_ROWS * GEMV_COLS * 4;
  }
};

// ROWS: see GemvRows (ldx is the row length of Z / z in the pooling modes).
// WS: the weights are an fp32 matrix split into bf16 hi and lo parts, row n of
// W = [hi(W[n, 0..K)) | lo(W[n, 0..K))] (fp32 inputs only); the product takes
// hi.hi + lo.hi + hi.lo of input and weight parts. `bf` (fp32, optional) is a
// bias used instead of `b`.
template <typename XT, int ROWS, bool WS = false>
__global__ void __launch_bounds__(GEMV_THREADS)
    gemv_kernel(const XT* __restrict__ X, long long ldx, int M, int K,
                const bf16* __restrict__ W, const bf16* __restrict__ b,
                const float* __restrict__ bf, int N, float* __restrict__ Y, long long ldy,
                int gelu, int* __restrict__ status) {
  static_assert(!WS || sizeof(XT) == 4, "split weights take fp32 inputs");
  using Lay = GemvLayout<XT, ROWS, WS>;
  constexpr int WF = WS ? 2 : 1;  // weight row length in units of K
  constexpr bool PAIRED = ROWS == GV_PAIRED;
  extern __shared__ __align__(16) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  XT* sx = reinterpret_cast<XT*>(smem + 16);
  const bf16* sw = reinterpret_cast<const bf16*>(smem + 16 + Lay::x_bytes(K));
  float* red = reinterpret_cast<float*>(smem + 16 + Lay::x_bytes(K) + Lay::w_bytes(K));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  const int c0 = blockIdx.x * GEMV_COLS;
  const int w_rows = min(GEMV_COLS, N - c0);
  const int xp = K + 8;
  const int h = ROWS != GV_PLAIN ? c0 / 64 : 0;
  const uint32_t xrow = K * sizeof(XT);
  const int rows0 = min(GEMV_ROWS, M);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    // the weights do not depend on the previous kernel: request them now,
    // with the byte count of the first round of input rows as well
    mbar_arrive_expect_tx(bar, w_rows * K * 2 * WF + rows0 * xrow * (PAIRED ? 2 : 1));
    bulk_load(const_cast<bf16*>(sw), W + static_cast<size_t>(c0) * K * WF, w_rows * K * 2 * WF,
              bar);
  }
  __syncthreads();  // barrier initialised before anyone waits on it
  pdl_wait();
  pdl_trigger();
  bool ok = true;
  const int kw = K / GEMV_WARPS;
  for (int m0 = 0, round = 0; m0 < M; m0 += GEMV_ROWS, ++round) {
    const int rows = min(GEMV_ROWS, M - m0);
    if (threadIdx.x == 0) {
      if (round > 0) mbar_arrive_expect_tx(bar, rows * xrow * (PAIRED ? 2 : 1));
      for (int r = 0; r < rows; ++r) {
        if constexpr (PAIRED) {
          const XT* zr = X + (static_cast<long long>(m0 + r) * 128 + h) * ldx;
          bulk_load(sx + r * xp, zr, xrow, bar);
          bulk_load(sx + (GEMV_ROWS + r) * xp, zr + 16 * ldx, xrow, bar);
        } else if constexpr (ROWS == GV_HEADROW) {
          bulk_load(sx + r * xp, X + (static_cast<long long>(m0 + r) * 16 + h) * ldx, xrow, bar);
        } else {
          bulk_load(sx + r * xp, X + static_cast<long long>(m0 + r) * ldx, xrow, bar);
        }
      }
    }
    ok = __syncthreads_and(ok && mbar_wait(bar, round & 1)) != 0;  // uniform decision
    if (!ok) {
      if (threadIdx.x == 0 && status != nullptr) atomicOr(status, DEV_WAIT_TIMEOUT);
      break;
    }
    // rows >= `rows` of the A tile hold stale values; they only reach output
    // rows that are never stored
    float acc[GEMV_NT][4] = {};
    int wr[GEMV_NT];  // weight row of this lane per n8 tile (rows past N read row 0)
#pragma unroll
    for (int j = 0; j < GEMV_NT; ++j) wr[j] = 8 * j + g < w_rows ? 8 * j + g : 0;
    for (int ks = warp * kw; ks < (warp + 1) * kw; ks += 16) {
      const int k = ks + t2;
      uint32_t bw[GEMV_NT][2];
#pragma unroll
      for (int j = 0; j < GEMV_NT; ++j) {
        const bf16* wrow = sw + static_cast<size_t>(wr[j]) * K * WF;
        bw[j][0] = *reinterpret_cast<const uint32_t*>(wrow + k);
        bw[j][1] = *reinterpret_cast<const uint32_t*>(wrow + k + 8);
      }
      if constexpr (sizeof(XT) == 2) {
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t*>(sx + g * xp + k);
        a[1] = *reinterpret_cast<const uint32_t*>(sx + (g + 8) * xp + k);
        a[2] = *reinterpret_cast<const uint32_t*>(sx + g * xp + k + 8);
        a[3] = *reinterpret_cast<const uint32_t*>(sx + (g + 8) * xp + k + 8);
#pragma unroll
        for (int j = 0; j < GEMV_NT; ++j) mma_16816(acc[j], a, bw[j]);
      } else {
        const float* fx = reinterpret_cast<const float*>(sx);
        float2 v[4] = {*reinterpret_cast<const float2*>(fx + g * xp + k),
                       *reinterpret_cast<const float2*>(fx + (g + 8) * xp + k),
                       *reinterpret_cast<const float2*>(fx + g * xp + k + 8),
                       *reinterpret_cast<const float2*>(fx + (g + 8) * xp + k + 8)};
        if constexpr (PAIRED) {
          const float* fz = fx + GEMV_ROWS * xp;
          const float2 z[4] = {*reinterpret_cast<const float2*>(fz + g * xp + k),
                               *reinterpret_cast<const float2*>(fz + (g + 8) * xp + k),
                               *reinterpret_cast<const float2*>(fz + g * xp + k + 8),
                               *reinterpret_cast<const float2*>(fz + (g + 8) * xp + k + 8)};
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = make_float2(v[i].x + z[i].x, v[i].y + z[i].y);
        }
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) split2(v[i], ah[i], al[i]);
#pragma unroll
        for (int j = 0; j < GEMV_NT; ++j) {
          mma_16816(acc[j], ah, bw[j]);
          mma_16816(acc[j], al, bw[j]);
          if constexpr (WS) {
            const bf16* wrow = sw + static_cast<size_t>(wr[j]) * K * WF + K;
            const uint32_t bl[2] = {*reinterpret_cast<const uint32_t*>(wrow + k),
                                    *reinterpret_cast<const uint32_t*>(wrow + k + 8)};
            mma_16816(acc[j], ah, bl);
          }
        }
      }
    }
    float* rw = red + warp * (GEMV_ROWS * GEMV_COLS);
#pragma unroll
    for (int j = 0; j < GEMV_NT; ++j) {
      rw[g * GEMV_COLS + 8 * j + t2] = acc[j][0];
      rw[g * GEMV_COLS + 8 * j + t2 + 1] = acc[j][1];
      rw[(g + 8) * GEMV_COLS + 8 * j + t2] = acc[j][2];
      rw[(g + 8) * GEMV_COLS + 8 * j + t2 + 1] = acc[j][3];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < GEMV_ROWS * GEMV_COLS; o += GEMV_THREADS) {
      const int r = o / GEMV_COLS, c = o % GEMV_COLS;
      if (r < rows && c < w_rows) {
        float y = 0.f;
#pragma unroll
        for (int w = 0; w < GEMV_WARPS; ++w) y += red[w * GEMV_ROWS * GEMV_COLS + o];
        if (bf != nullptr)
          y += bf[c0 + c];
        else if (b != nullptr)
          y += __bfloat162float(b[c0 + c]);
        if (gelu) y = gelu_f(y);
        Y[static_cast<long long>(m0 + r) * ldy + c0 + c] = y;
      }
    }
    __syncthreads();  // staged rows and partials consumed before the next round
  }
}

template <typename XT, int ROWS = GV_PLAIN, bool WS = false>
static int dispatch_gemv(const XT* X, long long ldx, int M, int K, const bf16* W, const bf16* b,
                         const float* bf, int N, float* Y, long long ldy, int gelu,
                         const Launch& L) {
  if (M == 0 || N == 0) return IVC_OK;
  if (K % (16 * GEMV_WARPS) != 0 || K > 2048 || N % 8 != 0) return IVC_EUNSUPPORTED;
  constexpr bool PAIRED = ROWS == GV_PAIRED;
  constexpr int KMAX = (PAIRED || WS) ? 1024 : 2048;
  if (K > KMAX) return IVC_EUNSUPPORTED;
  using Lay = GemvLayout<XT, ROWS, WS>;
  const int smem = static_cast<int>(Lay::total(K));
  // once per device, for the widest K this instantiation accepts
  if (smem_optin(reinterpret_cast<const void*>(gemv_kernel<XT, ROWS, WS>), Lay::total(KMAX)) !=
      IVC_OK)
    return IVC_ECUDA;
  TraceScope ts(ROWS != GV_PLAIN ? "pool.vproj"
                                 : (WS ? "pool.wqo" : (gelu ? "router.gemv_gelu" : "router.gemv")),
                L.stream);
  return launch_k(gemv_kernel<XT, ROWS, WS>, dim3((N + GEMV_COLS - 1) / GEMV_COLS),
                  dim3(GEMV_THREADS), smem, L.stream, 1, X, ldx, M, K, W, b, bf, N, Y, ldy, gelu,
                  L.status);
}

int launch_gemv(const float* X, long long ldx, int M, int K, const bf16* W, const bf16* b, int N,
                float* Y, long long ldy, int gelu, const Launch& L) {
  return dispatch_gemv<float>(X, ldx, M, K, W, b, nullptr, N, Y, ldy, gelu, L);
}

int launch_gemv_split(const float* X, long long ldx, int M, int K, const bf16* W2,
                      const float* bf, int N, float* Y, long long ldy, const Launch& L) {
  return dispatch_gemv<float, GV_PLAIN, true>(X, ldx, M, K, W2, nullptr, bf, N, Y, ldy, 0, L);
}

int launch_gemv_bf16x(const bf16* x, int K, const bf16* W, const bf16* b, int N, float* Y,
                      const Launch& L) {
  return dispatch_gemv<bf16>(x, 0, 1, K, W, b, nullptr, N, Y, 0, 0, L);
}

int launch_pool_vproj(const float* Z, int T, int D, const bf16* Wv, const bf16* bv, float* O,
                      const Launch& L) {
  return dispatch_gemv<float, GV_PAIRED>(Z, D, T, D, Wv, bv, nullptr, D, O, D, 0, L);
}

int launch_pool_vproj_heads(const float* z, int T, int D, const bf16* Wv, const bf16* bv, float* O,
                            const Launch& L) {
  return dispatch_gemv<float, GV_HEADROW>(z, D, T, D, Wv, bv, nullptr, D, O, D, 0, L);
}

// ---------------------------------------------------------------- pooling attention
// One CTA per (head, tile). Scores s_t = (Q_h . K_h[t]) / sqrt(64) for the
// valid prefix t < len; softmax in fp32; o_h = sum_t p_t V_h[t] / sum_t p_t.
constexpr int ATT_THREADS = 256;
constexpr int TILE_TOKENS = 1024;
constexpr int HEAD_DIM = 64;

__global__ void __launch_bounds__(ATT_THREADS)
    pool_attention_kernel(const float* __restrict__ Q, long long ldq,
                          const float* __restrict__ KV, long long ldkv, int koff, int voff,
                          const int32_t* __restrict__ valid_len, float* __restrict__ O, int D,
                          int* __restrict__ status) {
  __shared__ float s_q[HEAD_DIM];
  __shared__ float s_p[TILE_TOKENS];
  __shared__ float s_red[ATT_THREADS / 32][HEAD_DIM];
  __shared__ float s_scalar[ATT_THREADS / 32];
  const int h = blockIdx.x, tile = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  int n = TILE_TOKENS;
  if (valid_len != nullptr) {
    n = valid_len[tile];
    if (n < 1 || n > TILE_TOKENS) {
      if (threadIdx.x == 0) atomicOr(status, DEV_BAD_VALID_LEN);
      n = n < 1 ? 1 : TILE_TOKENS;
    }
  }
  if (threadIdx.x < HEAD_DIM)
    s_q[threadIdx.x] = Q[tile * ldq + h * HEAD_DIM + threadIdx.x] * 0.125f;  // 1/sqrt(64)
  __syncthreads();
  const float* kbase = KV + static_cast<long long>(tile) * TILE_TOKENS * ldkv + koff + h * HEAD_DIM;
  float mx = -INFINITY;
  for (int t = threadIdx.x; t < n; t += ATT_THREADS) {
    const float4* kr = reinterpret_cast<const float4*>(kbase + t * ldkv);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < HEAD_DIM / 4; ++c) {
      const float4 k4 = kr[c];
      s = fmaf(k4.x, s_q[4 * c], s);
      s = fmaf(k4.y, s_q[4 * c + 1], s);
      s = fmaf(k4.z, s_q[4 * c + 2], s);
      s = fmaf(k4.w, s_q[4 * c + 3], s);
    }
    s_p[t] = s;
    mx = fmaxf(mx, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_scalar[warp] = mx;
  __syncthreads();
  mx = s_scalar[0];
#pragma unroll
  for (int i = 1; i < ATT_THREADS / 32; ++i) mx = fmaxf(mx, s_scalar[i]);
  __syncthreads();
  float sum = 0.f;
  for (int t = threadIdx.x; t < n; t += ATT_THREADS) {
    const float e = expf(s_p[t] - mx);
    s_p[t] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_scalar[warp] = sum;
  __syncthreads();
  sum = 0.f;
#pragma unroll
  for (int i = 0; i < ATT_THREADS / 32; ++i) sum += s_scalar[i];
  // weighted V: warp w takes tokens w, w+8, ...; lane l owns dims 2l, 2l+1
  const float* vbase = KV + static_cast<long long>(tile) * TILE_TOKENS * ldkv + voff + h * HEAD_DIM;
  float a0 = 0.f, a1 = 0.f;
  for (int t = warp; t < n; t += ATT_THREADS / 32) {
    const float2 v2 = *reinterpret_cast<const float2*>(vbase + t * ldkv + 2 * lane);
    const float p = s_p[t];
    a0 = fmaf(p, v2.x, a0);
    a1 = fmaf(p, v2.y, a1);
  }
  s_red[warp][2 * lane] = a0;
  s_red[warp][2 * lane + 1] = a1;
  __syncthreads();
  if (threadIdx.x < HEAD_DIM) {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < ATT_THREADS / 32; ++i) acc += s_red[i][threadIdx.x];
    O[static_cast<long long>(tile) * D + h * HEAD_DIM + threadIdx.x] = acc / sum;
  }
}

int launch_pool_attention(const float* Q, long long ldq, const float* KV, long long ldkv,
                          int koff, int voff, const int32_t* valid_len, int T, int D, int heads,
                          float* O, const Launch& L) {
  if (T == 0) return IVC_OK;
  if (heads * HEAD_DIM != D) return IVC_EUNSUPPORTED;
  TraceScope ts("pool.attention", L.stream);
  return launch_k(pool_attention_kernel, dim3(heads, T), dim3(ATT_THREADS), 0, L.stream, 1, Q,
                  ldq, KV, ldkv, koff, voff, valid_len, O, D, L.status);
}

// ---------------------------------------------------------------- folded pooling
// The single query of each pooling layer lets the K and V projections be
// reassociated (exactly, in real arithmetic):
//   score_t = Q_h . (Wk_h x_t + bk_h) / 8 = x_t . u_h + c_h,
//       u_h = Wk_h^T Q_h / 8,  c_h = bk_h . Q_h / 8;
//   o_h = sum_t p_t (Wv_h x_t + bv_h) = Wv_h z_h + bv_h,  z_h = sum_t p_t x_t,
// since the softmax weights of the valid tokens sum to 1. The two
// contractions with the raw features x (scores: x u^T, sums: p x) run on the
// tensor cores; their fp32 right-hand sides u and p are fed as bf16 pairs
// hi + lo (hi = bf16(v), lo = bf16(v - hi)), keeping ~16 significant bits.

// u/c of one layer. Grid (D/128, heads <= 16); thread = feature column c.
// U2[t][j][c]: j < 16 hi part of u_j, j >= 16 lo part of u_{j-16}; rows of
// heads that do not exist are left as they are (their score columns and
// weighted-sum rows are never read).
__global__ void __launch_bounds__(128) pool_fold_query_kernel(
    const float* __restrict__ Q, long long ldq, int Tq, const bf16* __restrict__ Wk,
    const bf16* __restrict__ bk, int D, bf16* __restrict__ U2, float* __restrict__ cb) {
  __shared__ float s_q[64][HEAD_DIM];  // 64 tiles x head slice of Q
  const int h = blockIdx.y;
  const int c = blockIdx.x * 128 + threadIdx.x;
  float w[HEAD_DIM];
#pragma unroll
  for (int d = 0; d < HEAD_DIM; ++d)
    w[d] = __bfloat162float(Wk[static_cast<long long>(h * HEAD_DIM + d) * D + c]);
  pdl_wait();
  pdl_trigger();
  for (int t0 = 0; t0 < Tq; t0 += 64) {
    const int nt = min(64, Tq - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < nt * HEAD_DIM; i += 128)
      s_q[i / HEAD_DIM][i % HEAD_DIM] =
          Q[(t0 + i / HEAD_DIM) * ldq + h * HEAD_DIM + i % HEAD_DIM] * 0.125f;
    __syncthreads();
    for (int t = 0; t < nt; ++t) {
      // four independent partial sums (ILP), then combined
      float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int d = 0; d < HEAD_DIM; ++d) p[d & 3] = fmaf(w[d], s_q[t][d], p[d & 3]);
      const float u = (p[0] + p[1]) + (p[2] + p[3]);
      const bf16 hi = __float2bfloat16_rn(u);
      const bf16 lo = __float2bfloat16_rn(u - __bfloat162float(hi));
      bf16* base = U2 + static_cast<long long>(t0 + t) * 32 * D;
      base[static_cast<long long>(h) * D + c] = hi;
      base[static_cast<long long>(16 + h) * D + c] = lo;
    }
    if (blockIdx.x == 0 && threadIdx.x < nt) {
      float acc = 0.f;
      for (int d = 0; d < HEAD_DIM; ++d)
        acc = fmaf(bk ? __bfloat162float(bk[h * HEAD_DIM + d]) : 0.f, s_q[threadIdx.x][d], acc);
      cb[(t0 + threadIdx.x) * 16 + h] = acc;
    }
  }
}

// ---------------------------------------------------------------- weight folds
// Once per set of router weights: the output projection of pooling layer l
// and the query projection of layer l+1 follow each other with nothing in
// between (InternVL3_5-4B-Flash article, section 2: the layers are chained
// with no residual or norm), so Wq_{l+1} (Wo_l o + bo_l) + bq_{l+1} =
// P o + (Wq_{l+1} bo_l + bq_{l+1}) with P = Wq_{l+1} Wo_l. P is formed in
// fp32 (exact bf16 products, fp32 sums) and stored as a bf16 pair, row n =
// [hi(P[n, :]) | lo(P[n, :])], hi = bf16(P), lo = bf16(P - hi): about 16
// significant bits, read by the split-weight GEMV.
constexpr int WF_TILE = 64;  // output tile of the product kernel
constexpr int WF_KC = 16;    // inner-dimension chunk staged per step

__global__ void __launch_bounds__(256) wq_wo_fold_kernel(const bf16* __restrict__ A,
                                                         const bf16* __restrict__ B, int D,
                                                         bf16* __restrict__ P2) {
  // P[n][k] = sum_j A[n][j] B[j][k], A = Wq (rows n), B = Wo (rows j)
  __shared__ float sa[WF_KC][WF_TILE + 1];  // sa[j][n]
  __shared__ float sb[WF_KC][WF_TILE];      // sb[j][k]
  const int n0 = blockIdx.y * WF_TILE, k0 = blockIdx.x * WF_TILE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 4 x 4 outputs each
  float acc[4][4] = {};
  for (int j0 = 0; j0 < D; j0 += WF_KC) {
    for (int i = threadIdx.x; i < WF_KC * WF_TILE; i += 256) {
      const int r = i / WF_KC, c = i % WF_KC;  // A tile: row n0 + r, column j0 + c
      sa[c][r] = __bfloat162float(A[static_cast<size_t>(n0 + r) * D + j0 + c]);
      const int rb = i / WF_TILE, cb = i % WF_TILE;  // B tile: row j0 + rb, column k0 + cb
      sb[rb][cb] = __bfloat162float(B[static_cast<size_t>(j0 + rb) * D + k0 + cb]);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < WF_KC; ++j) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sa[j][ty * 4 + i];
        b[i] = sb[j][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(a[i], b[q], acc[i][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = n0 + ty * 4 + i;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = k0 + tx * 4 + q;
      const bf16 hi = __float2bfloat16_rn(acc[i][q]);
      const bf16 lo = __float2bfloat16_rn(acc[i][q] - __bfloat162float(hi));
      P2[static_cast<size_t>(n) * 2 * D + k] = hi;
      P2[static_cast<size_t>(n) * 2 * D + D + k] = lo;
    }
  }
}

// c[n] = sum_j A[n][j] bo[j] + bq[n] (fp32); one warp per row, either bias
// may be absent (zero).
__global__ void __launch_bounds__(256) wq_bo_fold_kernel(const bf16* __restrict__ A,
                                                         const bf16* __restrict__ bo,
                                                         const bf16* __restrict__ bq, int D,
                                                         float* __restrict__ c) {
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (n >= D) return;
  float acc = 0.f;
  if (bo != nullptr)
    for (int j = lane; j < D; j += 32)
      acc = fmaf(__bfloat162float(A[static_cast<size_t>(n) * D + j]), __bfloat162float(bo[j]), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) c[n] = acc + (bq != nullptr ? __bfloat162float(bq[n]) : 0.f);
}

int launch_wq_wo_fold(const bf16* Wq, const bf16* bq, const bf16* Wo, const bf16* bo, int D,
                      bf16* P2, float* c, cudaStream_t stream) {
  if (D % WF_TILE != 0) return IVC_EUNSUPPORTED;
  wq_wo_fold_kernel<<<dim3(D / WF_TILE, D / WF_TILE), 256, 0, stream>>>(Wq, Wo, D, P2);
  const int rc = cu_check(cudaGetLastError());
  if (rc != IVC_OK) return rc;
  wq_bo_fold_kernel<<<dim3((D + 7) / 8), 256, 0, stream>>>(Wq, bo, bq, D, c);
  return cu_check(cudaGetLastError());
}

int launch_pool_fold_query(const float* Q, long long ldq, int Tq, const bf16* Wk, const bf16* bk,
                           int D, bf16* U2, float* cb, const Launch& L) {
  if (Tq == 0) return IVC_OK;
  const int heads = D / HEAD_DIM;
  if (D % 128 != 0 || heads > 16) return IVC_EUNSUPPORTED;
  TraceScope ts("pool.fold_query", L.stream);
  return launch_k(pool_fold_query_kernel, dim3(D / 128, heads), dim3(128), 0, L.stream, 1, Q, ldq,
                  Tq, Wk, bk, D, U2, cb);
}

// Masked softmax of one (head, tile) from the split scores; writes the
// weights as a bf16 hi/lo pair into rows h and 16+h of the tile's 128-row
// block of P2 (rows 32..127 zero), the A operand of the weighted-sum GEMM.
__global__ void __launch_bounds__(ATT_THREADS)
    pool_softmax_kernel(const float* __restrict__ S, const float* __restrict__ cb, int cb_stride,
                        const int32_t* __restrict__ valid_len, bf16* __restrict__ P2,
                        int* __restrict__ status) {
  __shared__ float s_p[TILE_TOKENS];
  __shared__ float s_scalar[ATT_THREADS / 32];
  const int h = blockIdx.x, tile = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  int n = TILE_TOKENS;
  if (valid_len != nullptr) {
    n = valid_len[tile];
    if (n < 1 || n > TILE_TOKENS) {
      if (threadIdx.x == 0) atomicOr(status, DEV_BAD_VALID_LEN);
      n = n < 1 ? 1 : TILE_TOKENS;
    }
  }
  const float c = cb[tile * cb_stride + h];
  const float* srow = S + static_cast<long long>(tile) * TILE_TOKENS * 32;
  float mx = -INFINITY;
  for (int t = threadIdx.x; t < n; t += ATT_THREADS) {
    const float v = srow[t * 32 + h] + srow[t * 32 + 16 + h] + c;
    s_p[t] = v;
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_scalar[warp] = mx;
  __syncthreads();
  mx = s_scalar[0];
#pragma unroll
  for (int i = 1; i < ATT_THREADS / 32; ++i) mx = fmaxf(mx, s_scalar[i]);
  __syncthreads();
  float sum = 0.f;
  for (int t = threadIdx.x; t < n; t += ATT_THREADS) {
    const float e = expf(s_p[t] - mx);
    s_p[t] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_scalar[warp] = sum;
  __syncthreads();
  sum = 0.f;
#pragma unroll
  for (int i = 0; i < ATT_THREADS / 32; ++i) sum += s_scalar[i];
  const float inv = 1.0f / sum;
  bf16* blk = P2 + static_cast<long long>(tile) * 128 * TILE_TOKENS;
  for (int t = threadIdx.x; t < TILE_TOKENS; t += ATT_THREADS) {
    const float p = t < n ? s_p[t] * inv : 0.f;
    const bf16 hi = __float2bfloat16_rn(p);
    blk[h * TILE_TOKENS + t] = hi;
    blk[(16 + h) * TILE_TOKENS + t] = __float2bfloat16_rn(p - __bfloat162float(hi));
  }
  // rows 32..127 of the block stay zero, shared out over the heads' CTAs
  const bf16 z = __float2bfloat16_rn(0.f);
  const int per = (96 + gridDim.x - 1) / gridDim.x;
  for (int r = 32 + per * h; r < min(128, 32 + per * (h + 1)); ++r)
    for (int t = threadIdx.x; t < TILE_TOKENS; t += ATT_THREADS) blk[r * TILE_TOKENS + t] = z;
}

int launch_pool_softmax(const float* S, const float* cb, int cb_stride, const int32_t* valid_len,
                        int T, int heads, bf16* P2, const Launch& L) {
  if (T == 0) return IVC_OK;
  if (heads < 1 || heads > 16) return IVC_EUNSUPPORTED;
  TraceScope ts("pool.softmax", L.stream);
  return launch_k(pool_softmax_kernel, dim3(heads, T), dim3(ATT_THREADS), 0, L.stream, 1, S, cb,
                  cb_stride, valid_len, P2, L.status);
}

// ---------------------------------------------------------------- single-pass pooling attention
// The same layer as scores + softmax + weighted sum above, with one read of
// the features (the split-softmax, or flash-decoding, form of attention with
// one query per head): CTA (tile, chunk of ATTN_CHUNK tokens) streams its
// tokens ATTN_STEP at a time (one TMA box of {64 channels, 32 tokens, D/64
// chunks}, 128-byte swizzle, double-buffered; a slot is refilled after the
// next step's scores are summed, two CTA barriers per step) and per step
//   1. s[t][j] = x_t . U2[j] for the 32 split rows j (warp w multiplies its
//      D/8 channels with m16n8k16 MMAs, the U2 fragments held in registers
//      for the whole CTA; the 8 partial 32x32 tiles, stored column by
//      column, are summed in shared memory), s_h = s[t][h] + s[t][16 + h] +
//      c_h, invalid tokens -inf;
//   2. running max m_h and sum l_h (rescaled by exp(m_old - m_new)), the
//      weights e = exp(s - m_h) split into a bf16 hi/lo pair;
//   3. Zc[h][c] = Zc[h][c] * exp(m_old - m_new) + sum_t e_t x_t[c] with the
//      hi and lo weights into the same fp32 accumulators (warp w owns
//      channels [w D/8, (w+1) D/8), accumulators in registers).
// The chunk's unnormalised Zc, m and l go to global memory; pool_combine_
// kernel merges a tile's ATTN_NCH chunks:
//   z_h = sum_c exp(m_c - M) Zc_h / sum_c exp(m_c - M) l_c,  M = max_c m_c.
constexpr int ATTN_STEP = 32;                        // tokens per staged box
constexpr int ATTN_CHUNK = 128;                      // tokens per CTA
constexpr int ATTN_NCH = TILE_TOKENS / ATTN_CHUNK;   // chunks (partials) per tile
constexpr int ATTN_RED_PITCH = 36;                   // floats per column of a partial score tile
constexpr int ATTN_P_PITCH = 40;                     // bf16 per row of the weight tile (80 B)

__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__host__ __device__ constexpr size_t attend_smem_bytes(int D) {
  // alignment slack, two staging slots, 8 partial score tiles, hi/lo weights
  return 1024 + 2 * static_cast<size_t>(D) * 64 + 8 * 32 * ATTN_RED_PITCH * 4 +
         2 * 16 * ATTN_P_PITCH * 2;
}

// KS = D / 128: k16 steps of a warp's channel slice (D = 128 .. 1024).
template <int KS>
__global__ void __launch_bounds__(256, 1)
    pool_attend_kernel(const __grid_constant__ CUtensorMap xmap, const bf16* __restrict__ U2,
                       int u2_per_tile, const float* __restrict__ cb, int cb_stride,
                       const int32_t* __restrict__ valid_len, int heads, float* __restrict__ Zp,
                       float* __restrict__ mstat, float* __restrict__ lstat,
                       int* __restrict__ status) {
  constexpr int D = 128 * KS;
  constexpr int SLOT = D * 64;  // D/64 chunks x 32 tokens x 128 B
  constexpr int CHUNK_BYTES = ATTN_STEP * 128;
  constexpr int NT = 2 * KS;    // n8 tiles of a warp's weighted-sum channels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* red = reinterpret_cast<float*>(sm + 2 * SLOT);
  bf16* sp = reinterpret_cast<bf16*>(red + 8 * 32 * ATTN_RED_PITCH);  // [hi, lo][16][pitch]
  __shared__ float s_m[16], s_l[16], s_scale[16];
  __shared__ __align__(8) uint64_t s_mb[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  const int tile = blockIdx.x / ATTN_NCH, chunk = blockIdx.x % ATTN_NCH;
  const int tok0 = chunk * ATTN_CHUNK;
  // x and valid_len are inputs of the call and the previous kernel waited
  // for its own predecessor before letting this one start: both are read
  // before pdl_wait.
  int n = TILE_TOKENS;
  if (valid_len != nullptr) {
    n = valid_len[tile];
    if (n < 1 || n > TILE_TOKENS) {
      if (threadIdx.x == 0 && chunk == 0) atomicOr(status, DEV_BAD_VALID_LEN);
      n = n < 1 ? 1 : TILE_TOKENS;
    }
  }
  const int nsteps = max(0, min(ATTN_CHUNK / ATTN_STEP, (n - tok0 + ATTN_STEP - 1) / ATTN_STEP));
  if (threadIdx.x == 0) {
    mbar_init(&s_mb[0], 1);
    mbar_init(&s_mb[1], 1);
    fence_mbar_init();
    for (int st = 0; st < min(2, nsteps); ++st) {
      mbar_arrive_expect_tx(&s_mb[st], SLOT);
      tma_load_3d(sm + st * SLOT, &xmap, &s_mb[st], 0, tile * TILE_TOKENS + tok0 + st * ATTN_STEP,
                  0);
    }
  }
  if (threadIdx.x < 16) {
    s_m[threadIdx.x] = -INFINITY;
    s_l[threadIdx.x] = 0.f;
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const size_t row0 = (static_cast<size_t>(tile) * ATTN_NCH + chunk) * 16;
  if (nsteps == 0) {  // every token of the chunk is padding
    if (threadIdx.x < 16) {
      mstat[row0 + threadIdx.x] = -INFINITY;
      lstat[row0 + threadIdx.x] = 0.f;
    }
    return;
  }
  // B fragments of the scores (B[k = channel][n = split row] = U2[n][k]) for
  // this warp's channels; rows of heads that do not exist are zero
  const bf16* u = U2 + (u2_per_tile ? static_cast<size_t>(tile) * 32 * D : 0);
  uint32_t ub[KS][4][2];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int k = (warp * KS + ks) * 16 + t2;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int r = nt * 8 + g;
      const bool live = (r & 15) < heads;
      const bf16* ur = u + static_cast<size_t>(r) * D + k;
      ub[ks][nt][0] = live ? __ldg(reinterpret_cast<const unsigned*>(ur)) : 0u;
      ub[ks][nt][1] = live ? __ldg(reinterpret_cast<const unsigned*>(ur + 8)) : 0u;
    }
  }
  const int sh = threadIdx.x >> 4, stl = threadIdx.x & 15;  // softmax: head, token pair
  const float c_h = sh < heads ? cb[static_cast<size_t>(tile) * cb_stride + sh] : 0.f;
  float accz[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) accz[nt][i] = 0.f;
  bool ok = true;
  for (int st = 0; st < nsteps; ++st) {
    const int slot = st & 1;
    const uint8_t* sx = sm + slot * SLOT;
    ok = mbar_wait(&s_mb[slot], (st >> 1) & 1) && ok;
    // 1. partial scores of this warp's channels
    float accs[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) accs[mt][nt][i] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int kg = warp * KS + ks;
      const int c = kg >> 2, ja = ((kg & 3) << 1) + (lane >> 4);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int ra = mt * 16 + (lane & 15);
        uint32_t af[4];
        ldsm4(af, sx + c * CHUNK_BYTES + ra * 128 + ((ja ^ (ra & 7)) << 4));
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_16816(accs[mt][nt], af, ub[ks][nt]);
      }
    }
    float* rw = red + warp * 32 * ATTN_RED_PITCH;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int r = mt * 16 + g, j = nt * 8 + t2;
        rw[j * ATTN_RED_PITCH + r] = accs[mt][nt][0];
        rw[(j + 1) * ATTN_RED_PITCH + r] = accs[mt][nt][1];
        rw[j * ATTN_RED_PITCH + r + 8] = accs[mt][nt][2];
        rw[(j + 1) * ATTN_RED_PITCH + r + 8] = accs[mt][nt][3];
      }
    ok = __syncthreads_and(ok) != 0;
    if (!ok) break;
    // every warp has finished the previous step's weighted sums: its slot takes
    // the step after this one
    if (threadIdx.x == 0 && st >= 1 && st + 1 < nsteps) {
      mbar_arrive_expect_tx(&s_mb[slot ^ 1], SLOT);
      tma_load_3d(sm + (slot ^ 1) * SLOT, &xmap, &s_mb[slot ^ 1], 0,
                  tile * TILE_TOKENS + tok0 + (st + 1) * ATTN_STEP, 0);
    }
    // 2. running softmax of head sh over tokens 2 stl and 2 stl + 1
    {
      const int tb = tok0 + st * ATTN_STEP;
      // column sh of the hi part and 16 + sh of the lo part, token-contiguous
      float sv[2] = {c_h, c_h};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float* rc = red + w * 32 * ATTN_RED_PITCH;
        const float2 hi = *reinterpret_cast<const float2*>(rc + sh * ATTN_RED_PITCH + 2 * stl);
        const float2 lo =
            *reinterpret_cast<const float2*>(rc + (16 + sh) * ATTN_RED_PITCH + 2 * stl);
        sv[0] += hi.x + lo.x;
        sv[1] += hi.y + lo.y;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (!(sh < heads && tb + 2 * stl + i < n)) sv[i] = -INFINITY;
      float mx = fmaxf(sv[0], sv[1]);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = s_m[sh];
      const float m_new = fmaxf(m_old, mx);
      float e[2] = {0.f, 0.f}, scale = 1.f;
      if (m_new != -INFINITY) {
        scale = expf(m_old - m_new);
        e[0] = expf(sv[0] - m_new);
        e[1] = expf(sv[1] - m_new);
      }
      float sum = e[0] + e[1];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const bf16 hi = __float2bfloat16_rn(e[i]);
        sp[sh * ATTN_P_PITCH + 2 * stl + i] = hi;
        sp[(16 + sh) * ATTN_P_PITCH + 2 * stl + i] =
            __float2bfloat16_rn(e[i] - __bfloat162float(hi));
      }
      __syncwarp();  // every lane has read s_m[sh]
      if (stl == 0) {
        s_l[sh] = s_l[sh] * scale + sum;
        s_m[sh] = m_new;
        s_scale[sh] = scale;
      }
    }
    __syncthreads();
    // 3. rescale and accumulate this warp's channels of Zc
    {
      const float sc0 = s_scale[g], sc1 = s_scale[g + 8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        accz[nt][0] *= sc0;
        accz[nt][1] *= sc0;
        accz[nt][2] *= sc1;
        accz[nt][3] *= sc1;
      }
#pragma unroll
      for (int kk = 0; kk < ATTN_STEP / 16; ++kk) {
        uint32_t ah[4], al[4];
        const int pr = lane & 15, pk = kk * 16 + 8 * (lane >> 4);
        ldsm4(ah, sp + pr * ATTN_P_PITCH + pk);
        ldsm4(al, sp + (16 + pr) * ATTN_P_PITCH + pk);
        const int r = kk * 16 + (lane & 15);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
          const int cw = warp * (D / 8) + 8 * (nt + (lane >> 4));
          const int c = cw >> 6, j = (cw & 63) >> 3;
          uint32_t bf[4];
          ldsm4_trans(bf, sx + c * CHUNK_BYTES + r * 128 + ((j ^ (r & 7)) << 4));
          const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
          mma_16816(accz[nt], ah, b0);
          mma_16816(accz[nt], al, b0);
          mma_16816(accz[nt + 1], ah, b1);
          mma_16816(accz[nt + 1], al, b1);
        }
      }
    }
    // no barrier here: the weights and s_scale are rewritten only after the
    // next step's first barrier, and the score partials were read before the last
  }
  if (!ok) {
    if (threadIdx.x == 0) atomicOr(status, DEV_WAIT_TIMEOUT);
    return;
  }
  float* zp = Zp + row0 * D;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int c = warp * (D / 8) + nt * 8 + t2;
    *reinterpret_cast<float2*>(zp + static_cast<size_t>(g) * D + c) =
        make_float2(accz[nt][0], accz[nt][1]);
    *reinterpret_cast<float2*>(zp + static_cast<size_t>(g + 8) * D + c) =
        make_float2(accz[nt][2], accz[nt][3]);
  }
  if (threadIdx.x < 16) {
    mstat[row0 + threadIdx.x] = s_m[threadIdx.x];
    lstat[row0 + threadIdx.x] = s_l[threadIdx.x];
  }
}

// Grid (heads, T): z[tile][h] from the tile's ATTN_NCH chunk partials
// (chunks without a valid token, l = 0, are skipped).
template <int NCH>
__global__ void __launch_bounds__(256)
    pool_combine_kernel(const float* __restrict__ Zp, const float* __restrict__ mstat,
                        const float* __restrict__ lstat, int D, float* __restrict__ z) {
  const int h = blockIdx.x, tile = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const size_t r0 = static_cast<size_t>(tile) * NCH * 16 + h;
  float w[NCH];
  float M = -INFINITY;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    w[c] = lstat[r0 + 16 * c] > 0.f ? mstat[r0 + 16 * c] : -INFINITY;
    M = fmaxf(M, w[c]);
  }
  float L = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    w[c] = w[c] == -INFINITY ? 0.f : expf(w[c] - M);
    L += w[c] * lstat[r0 + 16 * c];
  }
  const float inv = 1.0f / L;
  for (int c4 = threadIdx.x * 4; c4 < D; c4 += 1024) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      if (w[c] == 0.f) continue;
      const float4 v = __ldg(reinterpret_cast<const float4*>(Zp + (r0 + 16 * c) * D + c4));
      acc.x = fmaf(w[c], v.x, acc.x);
      acc.y = fmaf(w[c], v.y, acc.y);
      acc.z = fmaf(w[c], v.z, acc.z);
      acc.w = fmaf(w[c], v.w, acc.w);
    }
    *reinterpret_cast<float4*>(z + (static_cast<size_t>(tile) * 16 + h) * D + c4) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

bool pool_attend_wanted() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_POOL_ATTEND");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

template <int KS>
static int launch_attend_ks(const CUtensorMap& xmap, const bf16* U2, int u2_per_tile,
                            const float* cb, int cb_stride, const int32_t* valid_len, int T,
                            int heads, float* Zp, float* mstat, float* lstat, const Launch& L) {
  const size_t smem = attend_smem_bytes(128 * KS);
  if (smem_optin(reinterpret_cast<const void*>(pool_attend_kernel<KS>), smem) != IVC_OK)
    return IVC_ECUDA;
  return launch_k(pool_attend_kernel<KS>, dim3(T * ATTN_NCH), dim3(256), smem, L.stream, 1, xmap,
                  U2, u2_per_tile, cb, cb_stride, valid_len, heads, Zp, mstat, lstat, L.status);
}

int launch_pool_attend(const void* x, const bf16* U2, int Tq, const float* cb,
                       const int32_t* valid_len, int T, int D, int heads, float* Zp, float* stats,
                       float* z, const Launch& L, bool combine, bool allow_tc) {
  if (T == 0) return IVC_OK;
  if (D % 128 != 0 || D > 1024 || heads < 1 || heads > 16 || heads * 64 != D)
    return IVC_EUNSUPPORTED;
  CUtensorMap xmap;
  {
    // x as {64 channels, T*1024 tokens, D/64 chunks}: rows of 2D bytes, chunks 128 B apart
    const unsigned long long dims[3] = {64, static_cast<unsigned long long>(T) * TILE_TOKENS,
                                        static_cast<unsigned long long>(D) / 64};
    const unsigned long long strides[2] = {static_cast<unsigned long long>(D) * 2, 128};
    const unsigned box[3] = {64, ATTN_STEP, static_cast<unsigned>(D / 64)};
    if (map_bf16(&xmap, 3, x, dims, strides, box) != IVC_OK) return IVC_ECUDA;
  }
  float* mstat = stats;
  float* lstat = stats + static_cast<size_t>(T) * ATTN_NCH * 16;
  const int u2_per_tile = Tq == 1 ? 0 : 1;
  const int cb_stride = Tq == 1 ? 0 : 16;
  const bool tc = allow_tc && attend_tc_wanted() && pool_attend_tc_supported(D, heads);
  int rc;
  if (tc) {
    // 128-token items: the same partials per tile as the mma.sync form
    if (pool_attend_tc_chunks() != ATTN_NCH) return IVC_EUNSUPPORTED;
    rc = launch_pool_attend_tc(x, U2, Tq, cb, valid_len, T, D, heads, Zp, stats, L);
  } else {
    TraceScope ts("pool.attend", L.stream);
    // one instantiation per width (the warps' register tiles are sized by it)
    auto run = [&](auto ks) {
      return launch_attend_ks<decltype(ks)::value>(xmap, U2, u2_per_tile, cb, cb_stride,
                                                   valid_len, T, heads, Zp, mstat, lstat, L);
    };
    switch (D / 128) {
      case 1: rc = run(std::integral_constant<int, 1>{}); break;
      case 2: rc = run(std::integral_constant<int, 2>{}); break;
      case 3: rc = run(std::integral_constant<int, 3>{}); break;
      case 4: rc = run(std::integral_constant<int, 4>{}); break;
      case 5: rc = run(std::integral_constant<int, 5>{}); break;
      case 6: rc = run(std::integral_constant<int, 6>{}); break;
      case 7: rc = run(std::integral_constant<int, 7>{}); break;
      default: rc = run(std::integral_constant<int, 8>{}); break;
    }
  }
  if (rc != IVC_OK || !combine) return rc;
  TraceScope ts("pool.combine", L.stream);
  return launch_k(pool_combine_kernel<ATTN_NCH>, dim3(heads, T), dim3(256), 0, L.stream, 1, Zp,
                  mstat, lstat, D, z);
}

// ---------------------------------------------------------------- residual + LayerNorm
// inside = 0: h[t] += (u[t] - mean) * rstd * gamma + beta;
// inside = 1: v = h[t] + u[t], h[t] = (v - mean) * rstd * gamma + beta
// (biased variance, eps 1e-5; D <= 2048).
__global__ void __launch_bounds__(256) residual_ln_kernel(float* __restrict__ h,
                                                          const float* __restrict__ u,
                                                          const bf16* __restrict__ gamma,
                                                          const bf16* __restrict__ beta, int D,
                                                          int inside) {
  __shared__ float s_red[8];
  __shared__ float s_v[2048];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  const float* u0 = u + static_cast<long long>(t) * D;
  const float* hr0 = h + static_cast<long long>(t) * D;
  for (int i = threadIdx.x; i < D; i += 256) s_v[i] = inside ? hr0[i] + u0[i] : u0[i];
  __syncthreads();
  const float* ur = s_v;
  float s = 0.f;
  for (int i = threadIdx.x; i < D; i += 256) s += ur[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) s_red[warp] = s;
  __syncthreads();
  float mean = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) mean += s_red[i];
  mean /= D;
  __syncthreads();
  float v = 0.f;
  for (int i = threadIdx.x; i < D; i += 256) {
    const float d = ur[i] - mean;
    v = fmaf(d, d, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float var = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) var += s_red[i];
  var /= D;
  const float rstd = 1.0f / sqrtf(var + 1e-5f);
  float* hr = h + static_cast<long long>(t) * D;
  // every load before the first store (a store to h could alias gamma or
  // beta for the compiler, which would serialise the loads behind it)
  float out[8];  // D <= 2048 over 256 threads
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = threadIdx.x + 256 * j;
    if (i < D) {
      const float n = (ur[i] - mean) * rstd * __bfloat162float(gamma[i]) +
                      __bfloat162float(beta[i]);
      out[j] = inside ? n : hr[i] + n;
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = threadIdx.x + 256 * j;
    if (i < D) hr[i] = out[j];
  }
}

int launch_residual_ln(float* h, const float* u, const bf16* gamma, const bf16* beta, int T,
                       int D, int inside, const Launch& L) {
  if (T == 0) return IVC_OK;
  if (D > 2048) return IVC_EUNSUPPORTED;
  TraceScope ts("gate.residual_ln", L.stream);
  return launch_k(residual_ln_kernel, dim3(T), dim3(256), 0, L.stream, 1, h, u, gamma, beta, D,
                  inside);
}

// ---------------------------------------------------------------- gate head
// One warp per tile: two dot products of length D, then a 2-way softmax.
__global__ void __launch_bounds__(256) gate_head_kernel(const float* __restrict__ h,
                                                        const bf16* __restrict__ Wout,
                                                        const bf16* __restrict__ bout, int T,
                                                        int D, float* __restrict__ gate) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  const float* hr = h + static_cast<long long>(t) * D;
  float l0 = 0.f, l1 = 0.f;
  for (int i = lane; i < D; i += 32) {
    const float v = hr[i];
    l0 = fmaf(__bfloat162float(Wout[i]), v, l0);
    l1 = fmaf(__bfloat162float(Wout[D + i]), v, l1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (lane == 0) {
    if (bout) {
      l0 += __bfloat162float(bout[0]);
      l1 += __bfloat162float(bout[1]);
    }
    const float m = fmaxf(l0, l1);
    const float e0 = expf(l0 - m), e1 = expf(l1 - m);
    const float s = e0 + e1;
    gate[2 * t] = e0 / s;
    gate[2 * t + 1] = e1 / s;
  }
}

int launch_gate_head(const float* h, const bf16* Wout, const bf16* bout, int T, int D,
                     float* gate, const Launch& L) {
  if (T == 0) return IVC_OK;
  TraceScope ts("gate.head", L.stream);
  return launch_k(gate_head_kernel, dim3((T + 7) / 8), dim3(256), 0, L.stream, 1, h, Wout, bout,
                  T, D, gate);
}

// ---------------------------------------------------------------- routing
// Single CTA. For each group (image, or the whole batch): the group's gate
// column 0 values are placed in ascending order by rank (ties broken by tile
// index), the linear-interpolation quantile is taken in fp64 with each
// operation rounded on its own (no fused multiply-add), and tile t is marked
// compressed iff gate > quantile and gate >= abs_t. Then the 64/256 row
// counts are prefix-summed into offsets[0..T] and total.
constexpr int ROUTE_THREADS = 1024;

__global__ void __launch_bounds__(ROUTE_THREADS)
    route_kernel(const float* __restrict__ gate, int T, const int32_t* __restrict__ offs, int I,
                 double rel_q, double abs_t, int scope, uint8_t* __restrict__ mask,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ total,
                 int* __restrict__ status) {
  extern __shared__ double s_dyn[];  // values then sorted values, IVC_MAX_QUANTILE_GROUP each
  double* s_vals = s_dyn;
  double* s_sorted = s_dyn + IVC_MAX_QUANTILE_GROUP;
  __shared__ double s_qv;
  __shared__ int s_bad;
  __shared__ int s_warp[ROUTE_THREADS / 32];
  __shared__ int s_carry;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    int bad = 0;
    if (scope == 0) {
      if (offs[0] != 0 || offs[I] != T) bad = 1;
      for (int i = 0; i < I && !bad; ++i)
        if (offs[i + 1] < offs[i]) bad = 1;
      if (bad) atomicOr(status, DEV_BAD_OFFSETS);
    }
    s_bad = bad;
  }
  __syncthreads();
  const int groups = scope == 0 ? I : 1;
  for (int gi = 0; gi < groups; ++gi) {
    int s = 0, e = T;
    if (scope == 0) {
      if (s_bad) break;
      s = offs[gi];
      e = offs[gi + 1];
    }
    const int n = e - s;
    if (n <= 0) continue;
    if (n > IVC_MAX_QUANTILE_GROUP) {
      if (threadIdx.x == 0) atomicOr(status, DEV_GROUP_TOO_LARGE);
      for (int i = threadIdx.x; i < n; i += ROUTE_THREADS) mask[s + i] = 0;
      __syncthreads();
      continue;
    }
    int my_nan = 0;
    for (int i = threadIdx.x; i < n; i += ROUTE_THREADS) {
      const double v = static_cast<double>(gate[2 * (s + i)]);
      s_vals[i] = v;
      my_nan |= isnan(v) ? 1 : 0;
    }
    // a NaN gate makes the group's quantile NaN (as torch.quantile does), so
    // no tile of the group passes the strict > test; the rank sort, whose
    // ranks assume a total order, is skipped
    const int any_nan = __syncthreads_or(my_nan);
    if (!any_nan) {
      for (int i = threadIdx.x; i < n; i += ROUTE_THREADS) {
        const double v = s_vals[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
          const double u = s_vals[j];
          rank += (u < v) || (u == v && j < i);
        }
        s_sorted[rank] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && any_nan) s_qv = __longlong_as_double(0x7ff8000000000000LL);
    if (threadIdx.x == 0 && !any_nan) {
      const double pos = __dmul_rn(rel_q, static_cast<double>(n - 1));
      const double flo = floor(pos);
      const int lo = static_cast<int>(flo);
      const int hi = static_cast<int>(ceil(pos));
      const double w = __dsub_rn(pos, flo);
      const double diff = __dsub_rn(s_sorted[hi], s_sorted[lo]);
      s_qv = __dadd_rn(s_sorted[lo], __dmul_rn(w, diff));
    }
    __syncthreads();
    const double qv = s_qv;
    for (int i = threadIdx.x; i < n; i += ROUTE_THREADS) {
      const double v = s_vals[i];
      mask[s + i] = (v > qv && v >= abs_t) ? 1 : 0;
    }
    __syncthreads();
  }
  if (scope == 0 && s_bad) {
    for (int i = threadIdx.x; i < T; i += ROUTE_THREADS) mask[i] = 0;
  }
  __syncthreads();
  // exclusive scan of the row counts
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int base = 0; base < T; base += ROUTE_THREADS) {
    const int i = base + threadIdx.x;
    const int cnt = i < T ? (mask[i] ? 64 : 256) : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += v;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + s_carry;
    if (i < T) offsets[i] = before + incl - cnt;
    __syncthreads();
    if (threadIdx.x == ROUTE_THREADS - 1) s_carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    offsets[T] = s_carry;
    if (total) *total = s_carry;
  }
}

int launch_route(const float* gate, int T, const int32_t* image_offsets, int I, double rel_q,
                 double abs_t, int scope, uint8_t* mask, int32_t* offsets, int32_t* total,
                 const Launch& L) {
  const size_t smem = 2 * IVC_MAX_QUANTILE_GROUP * sizeof(double);
  if (smem_optin(reinterpret_cast<const void*>(route_kernel), smem) != IVC_OK) return IVC_ECUDA;
  TraceScope ts("route", L.stream);
  return launch_k(route_kernel, dim3(1), dim3(ROUTE_THREADS), smem, L.stream, 1, gate, T,
                  image_offsets, I, rel_q, abs_t, scope, mask, offsets, total, L.status);
}

// ---------------------------------------------------------------- routed lists
// Single CTA (router-first flow). The compressed tiles, in tile order, are
// list_c[0..n_c) with their first output rows base_c (= offsets[t]); the
// others are list_u / base_u. n_u and n_c go to counts[0], counts[1].
__global__ void __launch_bounds__(ROUTE_THREADS)
    route_lists_kernel(const uint8_t* __restrict__ mask, const int32_t* __restrict__ offsets,
                       int T, int* __restrict__ list_u, int* __restrict__ base_u,
                       int* __restrict__ list_c, int* __restrict__ base_c,
                       int* __restrict__ counts) {
  __shared__ int s_warp[ROUTE_THREADS / 32];
  __shared__ int s_carry;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int base = 0; base < T; base += ROUTE_THREADS) {
    const int i = base + threadIdx.x;
    const int c = (i < T && mask[i]) ? 1 : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += v;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const int jc = (warp > 0 ? s_warp[warp - 1] : 0) + s_carry + incl - c;  // compressed before i
    if (i < T) {
      if (c) {
        list_c[jc] = i;
        base_c[jc] = offsets[i];
      } else {
        list_u[i - jc] = i;
        base_u[i - jc] = offsets[i];
      }
    }
    __syncthreads();
    if (threadIdx.x == ROUTE_THREADS - 1) s_carry = jc + c;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    counts[0] = T - s_carry;
    counts[1] = s_carry;
  }
}

int launch_route_lists(const uint8_t* mask, const int32_t* offsets, int T, int* list_u,
                       int* base_u, int* list_c, int* base_c, int* counts, const Launch& L) {
  TraceScope ts("route.lists", L.stream);
  return launch_k(route_lists_kernel, dim3(1), dim3(ROUTE_THREADS), 0, L.stream, 1, mask, offsets,
                  T, list_u, base_u, list_c, base_c, counts);
}

// ---------------------------------------------------------------- compaction
// Grid (T, 32): CTA (t, y) copies rows 8y..8y+7 of tile t when they exist
// (64 rows for a compressed tile, 256 otherwise): 8 rows x H bf16, each
// thread first loading all of its 16-byte pieces (H / 128 of them per
// thread-row pair, 8 for H = 2048), then storing them.
constexpr int COMPACT_ROWS = 8;

__global__ void __launch_bounds__(256) compact_kernel(const bf16* __restrict__ Y256,
                                                      const bf16* __restrict__ Y64,
                                                      const uint8_t* __restrict__ mask,
                                                      const int32_t* __restrict__ offsets, int H,
                                                      bf16* __restrict__ out) {
  const int t = blockIdx.x;
  const int r0 = blockIdx.y * COMPACT_ROWS;
  pdl_wait();
  pdl_trigger();
  const bool comp = mask[t] != 0;
  const int rows = comp ? 64 : 256;
  if (r0 >= rows) return;
  const bf16* src = comp ? Y64 + (static_cast<long long>(t) * 64 + r0) * H
                         : Y256 + (static_cast<long long>(t) * 256 + r0) * H;
  bf16* dst = out + (static_cast<long long>(offsets[t]) + r0) * H;
  const int n = COMPACT_ROWS * H / 8;  // 16-byte pieces of the 8 rows (contiguous)
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int i0 = 0; i0 < n; i0 += 8 * 256) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + k * 256 + threadIdx.x;
      if (i < n) u[k] = __ldcs(s4 + i);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + k * 256 + threadIdx.x;
      if (i < n) __stcs(d4 + i, u[k]);
    }
  }
}

int launch_compact(const bf16* Y256, const bf16* Y64, const uint8_t* mask,
                   const int32_t* offsets, int T, int H, bf16* out, const Launch& L) {
  if (T == 0) return IVC_OK;
  TraceScope ts("compact", L.stream);
  return launch_k(compact_kernel, dim3(T, 256 / COMPACT_ROWS), dim3(256), 0, L.stream, 1, Y256,
                  Y64, mask, offsets, H, out);
}

}  // namespace ivc
