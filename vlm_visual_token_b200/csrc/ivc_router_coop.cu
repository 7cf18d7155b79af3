// ivc_router_coop.cu — cooperative multi-phase kernels of the ViR router
// for the flow in which the router runs beside the connector on a few SMs:
// the Gating MLP with its softmax head, and the tail of each pooling layer.
//
// InternVL3_5-4B-Flash "Gating and CrossAttentionPooling" article:
//  * section 3 (Gating): 4 residual blocks (Linear -> GELU -> Dropout ->
//    Linear -> Dropout -> LayerNorm around a residual; dropout is the
//    identity at inference), then Linear(hidden, 2) and a softmax whose
//    column 0 is the probability of compressing the tile;
//  * section 2 (CrossAttentionPooling): per layer the query's attention over
//    the tile's tokens, the value and output projections, and the next
//    layer's query projection. In the folded form (ivc_router.cu) the key
//    projection is folded into the query, u_h = Wk_h^T Q_h / 8, and the
//    attention kernel leaves per-chunk partial weighted sums of x; the tail
//    merges them (z_h), projects o_h = Wv_h z_h + bv_h, q = Wo o + bo,
//    Q' = Wq' q + bq', and folds the next layer's keys into Q'.
//
// As separate kernels these are chains of tiny dependent launches (two
// vector-matrix products and a row LayerNorm per gating block; merge, three
// projections and a fold per pooling layer), each at a device-time floor of
// several microseconds. Here each chain is one cooperative launch of a few
// CTAs (16 for the InternVL widths, so that it fits in the SMs the connector
// leaves free beside it), with a bounded software grid barrier between
// dependent phases:
//   Gating, per block b:  u1 = GELU(W1_b h + b1_b);  u2 = W2_b u1 + b2_b;
//                         h = h + LN(u2) (or LN(h + u2)); the last block's
//                         rows go straight on to the head softmax(Wout h + bout)
//                         (h_0 = the pooled vectors; eleven grid barriers);
//   pooling tail:         merge + o = Wv z + bv;  q = Wo o + bo;
//                         [Q' = Wq' q + bq';  u', c' = fold of Wk' with Q']
//                         (three grid barriers, one after the last layer).
//
// A projection item is COLS consecutive output columns: the item's COLS
// weight rows arrive as one TMA box of a {64, rows, K/64} view (128-byte
// swizzle: the chunk of 64 k's of row r sits at chunk*COLS*128 + r*128, its
// 16-byte units XOR-ed with r % 8, so the B-fragment loads of 8 rows hit 8
// different bank groups). The requests for the next phase's first item are
// issued before the grid barrier that ends the current phase (weights do not
// depend on it). Input rows (fp32, up to 16 per round) come by one bulk copy
// per row into rows padded by 8 floats, or, for the value projection, are
// merged from the attention's chunk partials while the weights arrive. Warp
// w multiplies its K/8 slice with mma.sync m16n8k16, the fp32 inputs split
// into bf16 hi + lo (two MMAs per k-step, fp32 accumulation); the 8 partial
// tiles are summed in shared memory (over the input rows, which are consumed
// by then). Every wait is bounded; a wait that runs out sets
// IVC_DEV_WAIT_TIMEOUT and the CTA skips the rest, letting the copies it
// issued land before it exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ivc_internal.h"
#include "ivc_ptx.cuh"

namespace ivc {
namespace {

constexpr int GT_THREADS = 256;
constexpr int GT_WARPS = GT_THREADS / 32;
constexpr int GT_ROWS = 16;
constexpr int GT_MAX_CTAS = 16;

struct GatingArgs {
  CUtensorMap w1[4];  // W1_b [G, D] as {64, G, D/64}, box {64, COLS, D/64}
  CUtensorMap w2[4];  // W2_b [D, G] as {64, D, G/64}, box {64, COLS, G/64}
  const float* pooled;  // [T, D]
  const bf16 *b1[4], *b2[4], *ln_g[4], *ln_b[4], *Wout, *bout;
  int T, D, G, inside;
  float* h;   // [T, D]
  float* u1;  // [T, G]
  float* u2;  // [T, D]
  float* gate;  // [T, 2]
  unsigned* bar;  // arrival counter, zero at launch
  int* status;
};

__device__ __forceinline__ float gelu_g(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// v = hi + lo, hi = bf16(v), lo = bf16(v - hi), two lanes per 32-bit word.
__device__ __forceinline__ void split_hl(float2 v, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 l = __floats2bfloat162_rn(v.x - __low2float(h), v.y - __high2float(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ bool cta_wait_all(uint64_t* bar, uint32_t parity) {
  return __syncthreads_and(mbar_wait(bar, parity) ? 1 : 0) != 0;
}

// Monotonic arrival counter: barrier g completes at (g + 1) * gridDim.x.
__device__ bool gt_grid_sync(unsigned* bar, unsigned& gen) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned target = (gen + 1u) * gridDim.x;
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(bar), "r"(1u) : "memory");
    const long long t0 = clock64();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (static_cast<int>(v - target) >= 0) break;
      if (clock64() - t0 > IVC_WAIT_CYCLES) {
        ok = 0;
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  ++gen;
  return s_ok != 0;
}

template <int COLS>
struct GtSmem {
  // the weight box (COLS rows x K), then a region that holds the input rows
  // [16][K + 8] fp32 and, once they are consumed, the 8 warps' partial tiles
  // [8][16][COLS] fp32 (or the LayerNorm row buffer): as large as the larger
  __host__ __device__ static constexpr size_t w_bytes(int K) {
    return static_cast<size_t>(COLS) * K * 2;
  }
  __host__ __device__ static constexpr size_t x_bytes(int K) {
    const size_t rows = static_cast<size_t>(GT_ROWS) * (K + 8) * 4;
    const size_t partials = static_cast<size_t>(GT_WARPS) * GT_ROWS * COLS * 4;
    return rows > partials ? rows : partials;
  }
  __host__ __device__ static constexpr size_t total(int K) { return 1024 + w_bytes(K) + x_bytes(K); }
};

// Input rows of a projection: rows [m0, m0 + rows) of a row-major fp32
// [T, K] matrix, one bulk copy per row (mbarrier 1).
struct BulkRows {
  const float* X;
  int K;
  __device__ void issue(int m0, int rows, float* sx, int xp, int /*c0*/, uint64_t* mb,
                        int& pend) const {
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&mb[1], rows * K * 4);
      asm volatile("fence.proxy.async.global;" ::: "memory");
      for (int r = 0; r < rows; ++r)
        bulk_load(sx + r * xp, X + static_cast<size_t>(m0 + r) * K, K * 4, &mb[1]);
    }
    pend |= 2;
  }
  __device__ bool wait(uint64_t* mb, uint32_t* ph, int& pend) const {
    if (!cta_wait_all(&mb[1], ph[1])) return false;
    ph[1] ^= 1;
    pend &= ~2;
    return true;
  }
};

// Input rows of the value projection: row t = z_h of tile t, head h = the
// item's head (its columns are that head's), merged from the attention's
// NCH chunk partials: z_h = sum_c exp(m_c - M) Zc_h / sum_c exp(m_c - M) l_c,
// M = max over the chunks with a valid token (l_c > 0).
template <int NCH>
struct MergedRows {
  const float* Zp;     // [T][NCH][16][D]
  const float* mstat;  // [T*NCH*16]
  const float* lstat;
  int D;
  __device__ void issue(int m0, int rows, float* sx, int xp, int c0, uint64_t*, int&) const {
    const int h = c0 / 64;
    for (int r = 0; r < rows; ++r) {
      const size_t r0 = static_cast<size_t>(m0 + r) * NCH * 16 + h;
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
      for (int k4 = threadIdx.x * 4; k4 < D; k4 += GT_THREADS * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          if (w[c] == 0.f) continue;
          const float4 v = __ldg(reinterpret_cast<const float4*>(Zp + (r0 + 16 * c) * D + k4));
          acc.x = fmaf(w[c], v.x, acc.x);
          acc.y = fmaf(w[c], v.y, acc.y);
          acc.z = fmaf(w[c], v.z, acc.z);
          acc.w = fmaf(w[c], v.w, acc.w);
        }
        *reinterpret_cast<float4*>(sx + r * xp + k4) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      }
    }
  }
  __device__ bool wait(uint64_t*, uint32_t*, int&) const {
    __syncthreads();  // the merged rows are written
    return true;
  }
};

// Y[m, c0 + j] = act(sum_k X[m, k] W[c0 + j, k] + b[c0 + j]) for the items of
// this CTA (item i = columns [i COLS, (i+1) COLS)), input rows from `stage`.
// On entry the first item's weight box may already be requested (bit 0 of
// pend). Returns false on a wait that ran out; pend then tells which
// barriers still have copies in flight (bit 0: weights, bit 1: input rows).
template <int COLS, typename Stage>
__device__ bool gt_project(const CUtensorMap* wmap, int K, int N, const Stage& stage, int T,
                           const bf16* __restrict__ bias, bool act, float* __restrict__ Y,
                           uint8_t* sm, uint64_t* mb, uint32_t* ph, int& pend) {
  using S = GtSmem<COLS>;
  constexpr int NT = COLS / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  const bf16* sw = reinterpret_cast<const bf16*>(sm);
  float* sx = reinterpret_cast<float*>(sm + S::w_bytes(K));
  const int xp = K + 8;
  const int kw = K / GT_WARPS;
  const int items = N / COLS;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int c0 = item * COLS;
    if (!(pend & 1)) {
      __syncthreads();  // the previous item's reads of the weight box are done
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&mb[0], COLS * K * 2);
        tma_load_3d(const_cast<bf16*>(sw), wmap, &mb[0], 0, c0, 0);
      }
      pend |= 1;
    }
    bool w_ready = false;
    for (int m0 = 0; m0 < T; m0 += GT_ROWS) {
      const int rows = min(GT_ROWS, T - m0);
      __syncthreads();  // the previous round's inputs and partials are consumed
      stage.issue(m0, rows, sx, xp, c0, mb, pend);
      if (!w_ready) {
        if (!cta_wait_all(&mb[0], ph[0])) return false;
        ph[0] ^= 1;
        pend &= ~1;
        w_ready = true;
      }
      if (!stage.wait(mb, ph, pend)) return false;
      // rows >= `rows` of the A tile hold stale values; they only reach
      // output rows that are never stored
      float acc[NT][4] = {};
      for (int ks = warp * kw; ks < (warp + 1) * kw; ks += 16) {
        const int k = ks + t2;
        const float2 v[4] = {*reinterpret_cast<const float2*>(sx + g * xp + k),
                             *reinterpret_cast<const float2*>(sx + (g + 8) * xp + k),
                             *reinterpret_cast<const float2*>(sx + g * xp + k + 8),
                             *reinterpret_cast<const float2*>(sx + (g + 8) * xp + k + 8)};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_hl(v[i], ah[i], al[i]);
        const int chunk = k >> 6, kc = k & 63;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const int r = 8 * j + g;
          const uint8_t* rowp =
              reinterpret_cast<const uint8_t*>(sw) + (static_cast<size_t>(chunk) * COLS + r) * 128;
          uint32_t bw[2];
          bw[0] = *reinterpret_cast<const uint32_t*>(rowp + (((kc >> 3) ^ (r & 7)) << 4) +
                                                      (kc & 7) * 2);
          bw[1] = *reinterpret_cast<const uint32_t*>(rowp + ((((kc + 8) >> 3) ^ (r & 7)) << 4) +
                                                      ((kc + 8) & 7) * 2);
          mma16816(acc[j], ah, bw);
          mma16816(acc[j], al, bw);
        }
      }
      __syncthreads();  // every warp is done with the staged inputs
      float* red = sx;  // [8 warps][16 rows][COLS]
      float* rw = red + warp * (GT_ROWS * COLS);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        rw[g * COLS + 8 * j + t2] = acc[j][0];
        rw[g * COLS + 8 * j + t2 + 1] = acc[j][1];
        rw[(g + 8) * COLS + 8 * j + t2] = acc[j][2];
        rw[(g + 8) * COLS + 8 * j + t2 + 1] = acc[j][3];
      }
      __syncthreads();
      for (int o = threadIdx.x; o < GT_ROWS * COLS; o += GT_THREADS) {
        const int r = o / COLS, c = o % COLS;
        if (r < rows) {
          float y = 0.f;
#pragma unroll
          for (int w = 0; w < GT_WARPS; ++w) y += red[w * GT_ROWS * COLS + o];
          if (bias != nullptr) y += __bfloat162float(bias[c0 + c]);
          Y[static_cast<size_t>(m0 + r) * N + c0 + c] = act ? gelu_g(y) : y;
        }
      }
    }
  }
  return true;
}

// The first item's weight box of the next projection phase (issued before the
// grid barrier that ends the current phase).
template <int COLS>
__device__ void gt_prefetch_w(const CUtensorMap* wmap, int K, int N, uint8_t* sm, uint64_t* mb,
                              int& pend) {
  __syncthreads();  // the current phase's reads of the weight box are done
  if (static_cast<int>(blockIdx.x) < N / COLS) {
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&mb[0], COLS * K * 2);
      tma_load_3d(sm, wmap, &mb[0], 0, static_cast<int>(blockIdx.x) * COLS, 0);
    }
    pend |= 1;
  }
}

// dst = h + LN(u) (inside 0) or LN(h + u) (inside 1) of one row of D values,
// through the shared row buffer s (D floats); returns nothing, writes dst.
__device__ void gt_residual_ln(const float* __restrict__ hrow, const float* __restrict__ urow,
                               const bf16* __restrict__ g, const bf16* __restrict__ be, float* s,
                               int D, int inside) {
  __shared__ float s_red[GT_WARPS];
  __shared__ float s_stat[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < D; i += GT_THREADS) s[i] = inside ? hrow[i] + urow[i] : urow[i];
  __syncthreads();
  float a = 0.f;
  for (int i = threadIdx.x; i < D; i += GT_THREADS) a += s[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  if (lane == 0) s_red[warp] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < GT_WARPS; ++i) t += s_red[i];
    s_stat[0] = t / D;
  }
  __syncthreads();
  const float mean = s_stat[0];
  float v = 0.f;
  for (int i = threadIdx.x; i < D; i += GT_THREADS) {
    const float d = s[i] - mean;
    v = fmaf(d, d, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < GT_WARPS; ++i) t += s_red[i];
    s_stat[1] = 1.0f / sqrtf(t / D + 1e-5f);
  }
  __syncthreads();
  const float rstd = s_stat[1];
  for (int i = threadIdx.x; i < D; i += GT_THREADS) {
    const float n = (s[i] - mean) * rstd * __bfloat162float(g[i]) + __bfloat162float(be[i]);
    s[i] = inside ? n : hrow[i] + n;
  }
  __syncthreads();
}

template <int COLS>
__global__ void __launch_bounds__(GT_THREADS, 1) gating_kernel(const __grid_constant__ GatingArgs a) {
  using S = GtSmem<COLS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t mb[2];  // 0: weight box, 1: input rows
  const int D = a.D, G = a.G, T = a.T;
  if (threadIdx.x == 0) {
    mbar_init(&mb[0], 1);
    mbar_init(&mb[1], 1);
    fence_mbar_init();
    for (int b = 0; b < 4; ++b) {
      tma_prefetch_desc(&a.w1[b]);
      tma_prefetch_desc(&a.w2[b]);
    }
  }
  __syncthreads();
  uint32_t ph[2] = {0u, 0u};
  int pend = 0;
  unsigned gen = 0;
  bool ok = true;
  // the first block's weights are inputs of the call: request them at once
  gt_prefetch_w<COLS>(&a.w1[0], D, G, sm, mb, pend);
  pdl_wait();
  pdl_trigger();
  float* srow = reinterpret_cast<float*>(sm + S::w_bytes(D > G ? D : G));  // LN row buffer
  for (int b = 0; b < 4 && ok; ++b) {
    const float* hin = b == 0 ? a.pooled : a.h;
    ok = gt_project<COLS>(&a.w1[b], D, G, BulkRows{hin, D}, T, a.b1[b], true, a.u1, sm, mb, ph,
                          pend);
    if (!ok) break;
    gt_prefetch_w<COLS>(&a.w2[b], G, D, sm, mb, pend);
    if (!(ok = gt_grid_sync(a.bar, gen))) break;
    ok = gt_project<COLS>(&a.w2[b], G, D, BulkRows{a.u1, G}, T, a.b2[b], false, a.u2, sm, mb, ph,
                          pend);
    if (!ok) break;
    if (b < 3) gt_prefetch_w<COLS>(&a.w1[b + 1], D, G, sm, mb, pend);
    if (!(ok = gt_grid_sync(a.bar, gen))) break;
    // residual LayerNorm, one row per CTA in turn; the last block's rows go
    // on to the head (one warp per logit)
    for (int m = blockIdx.x; m < T; m += gridDim.x) {
      const float* hr = hin + static_cast<size_t>(m) * D;
      gt_residual_ln(hr, a.u2 + static_cast<size_t>(m) * D, a.ln_g[b], a.ln_b[b], srow, D,
                     a.inside);
      if (b < 3) {
        for (int i = threadIdx.x; i < D; i += GT_THREADS) a.h[static_cast<size_t>(m) * D + i] = srow[i];
      } else {
        __shared__ float s_logit[2];
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (warp < 2) {
          float l = 0.f;
          for (int i = lane; i < D; i += 32)
            l = fmaf(__bfloat162float(a.Wout[warp * D + i]), srow[i], l);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
          if (lane == 0) s_logit[warp] = l + (a.bout ? __bfloat162float(a.bout[warp]) : 0.f);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
          const float mx = fmaxf(s_logit[0], s_logit[1]);
          const float e0 = expf(s_logit[0] - mx), e1 = expf(s_logit[1] - mx);
          a.gate[2 * m] = e0 / (e0 + e1);
          a.gate[2 * m + 1] = e1 / (e0 + e1);
        }
      }
      __syncthreads();  // the row buffer is free for the next row
    }
    if (b < 3 && !(ok = gt_grid_sync(a.bar, gen))) break;
  }
  // copies whose wait never succeeded: let them land before exit
  if (pend & 1) (void)mbar_wait(&mb[0], ph[0]);
  if (pend & 2) (void)mbar_wait(&mb[1], ph[1]);
  if (!ok && threadIdx.x == 0) atomicOr(a.status, DEV_WAIT_TIMEOUT);
}

template <int COLS>
int launch_gating_cols(const GatingArgs& a, int ctas, const Launch& L) {
  using S = GtSmem<COLS>;
  const int K = a.D > a.G ? a.D : a.G;
  // the LN row buffer (D floats) sits after the weight box, inside the input rows
  const size_t smem = S::total(K);
  if (smem > 227 * 1024) return IVC_EUNSUPPORTED;
  if (smem_optin(reinterpret_cast<const void*>(gating_kernel<COLS>), smem) != IVC_OK)
    return IVC_ECUDA;
  if (cudaMemsetAsync(a.bar, 0, sizeof(unsigned), L.stream) != cudaSuccess) return IVC_ECUDA;
  TraceScope ts("gate.fused", L.stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(GT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cu_check(cudaLaunchKernelEx(&cfg, gating_kernel<COLS>, a));
}

// ------------------------------------------------------------------ pooling tail
constexpr int PT_NCH = 8;  // attention chunks (partials) per tile

struct PoolTailArgs {
  CUtensorMap wv, wo, wq, wk;  // [D, D] as {64, D, D/64}, box {64, 64, D/64}
  const float* Zp;             // [T][8][16][D] chunk partials of this layer
  const float* mstat;          // [T*8*16] running max of each partial
  const float* lstat;          // [T*8*16] running sum of each partial
  const bf16 *bv, *bo, *bq, *bk;
  int T, D, last;              // last: no next layer (stop after q = Wo o + bo)
  float* O;                    // [T, D]
  float* q;                    // [T, D]: the layer's output (pooled after the last layer)
  float* Q;                    // [T, D]: the next layer's query
  bf16* U2;                    // [T][32][D]: its folded key projection, hi rows 0..15, lo 16..31
  float* cb;                   // [T][16]
  unsigned* bar;
  int* status;
};

// u_h = Wk_h^T Q_h / 8 (hi/lo bf16 pair) and c_h = bk_h . Q_h / 8 of the next
// layer, one head per item: the head's 64 key rows arrive as one box, the
// tiles' query slices are read from global memory into shared memory.
__device__ bool pt_fold(const PoolTailArgs& a, uint8_t* sm, uint64_t* mb, uint32_t* ph,
                        int& pend) {
  const int D = a.D, heads = D / 64;
  const bf16* sw = reinterpret_cast<const bf16*>(sm);
  float* sq = reinterpret_cast<float*>(sm + GtSmem<64>::w_bytes(D));  // [64 tiles][64]
  for (int h = blockIdx.x; h < heads; h += gridDim.x) {
    if (!(pend & 1)) {
      __syncthreads();
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&mb[0], 64 * D * 2);
        tma_load_3d(const_cast<bf16*>(sw), &a.wk, &mb[0], 0, h * 64, 0);
      }
      pend |= 1;
    }
    if (!cta_wait_all(&mb[0], ph[0])) return false;
    ph[0] ^= 1;
    pend &= ~1;
    for (int t0 = 0; t0 < a.T; t0 += 64) {
      const int nt = min(64, a.T - t0);
      __syncthreads();
      for (int i = threadIdx.x; i < nt * 64; i += GT_THREADS)
        sq[i] = a.Q[static_cast<size_t>(t0 + i / 64) * D + h * 64 + i % 64] * 0.125f;
      __syncthreads();
      for (int c = threadIdx.x; c < D; c += GT_THREADS) {
        const int chunk = c >> 6, kc = c & 63;
        for (int t = 0; t < nt; ++t) {
          float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
          for (int d = 0; d < 64; ++d) {
            const bf16 w = *reinterpret_cast<const bf16*>(
                reinterpret_cast<const uint8_t*>(sw) + (static_cast<size_t>(chunk) * 64 + d) * 128 +
                (((kc >> 3) ^ (d & 7)) << 4) + (kc & 7) * 2);
            p[d & 3] = fmaf(__bfloat162float(w), sq[t * 64 + d], p[d & 3]);
          }
          const float u = (p[0] + p[1]) + (p[2] + p[3]);
          const bf16 hi = __float2bfloat16_rn(u);
          const bf16 lo = __float2bfloat16_rn(u - __bfloat162float(hi));
          bf16* base = a.U2 + static_cast<size_t>(t0 + t) * 32 * D;
          base[static_cast<size_t>(h) * D + c] = hi;
          base[static_cast<size_t>(16 + h) * D + c] = lo;
        }
      }
      if (threadIdx.x < nt) {
        float acc = 0.f;
        for (int d = 0; d < 64; ++d)
          acc = fmaf(a.bk ? __bfloat162float(a.bk[h * 64 + d]) : 0.f, sq[threadIdx.x * 64 + d], acc);
        a.cb[(t0 + threadIdx.x) * 16 + h] = acc;
      }
    }
  }
  return true;
}

__global__ void __launch_bounds__(GT_THREADS, 1) pool_tail_kernel(const __grid_constant__ PoolTailArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t mb[2];  // 0: weight box, 1: input rows
  const int D = a.D, T = a.T;
  if (threadIdx.x == 0) {
    mbar_init(&mb[0], 1);
    mbar_init(&mb[1], 1);
    fence_mbar_init();
    tma_prefetch_desc(&a.wv);
    tma_prefetch_desc(&a.wo);
    if (!a.last) {
      tma_prefetch_desc(&a.wq);
      tma_prefetch_desc(&a.wk);
    }
  }
  __syncthreads();
  uint32_t ph[2] = {0u, 0u};
  int pend = 0;
  unsigned gen = 0;
  bool ok = true;
  gt_prefetch_w<64>(&a.wv, D, D, sm, mb, pend);  // weights are inputs of the call
  pdl_wait();
  pdl_trigger();
  do {
    ok = gt_project<64>(&a.wv, D, D, MergedRows<PT_NCH>{a.Zp, a.mstat, a.lstat, D}, T, a.bv, false,
                        a.O, sm, mb, ph, pend);
    if (!ok) break;
    gt_prefetch_w<64>(&a.wo, D, D, sm, mb, pend);
    if (!(ok = gt_grid_sync(a.bar, gen))) break;
    ok = gt_project<64>(&a.wo, D, D, BulkRows{a.O, D}, T, a.bo, false, a.q, sm, mb, ph, pend);
    if (!ok || a.last) break;
    gt_prefetch_w<64>(&a.wq, D, D, sm, mb, pend);
    if (!(ok = gt_grid_sync(a.bar, gen))) break;
    ok = gt_project<64>(&a.wq, D, D, BulkRows{a.q, D}, T, a.bq, false, a.Q, sm, mb, ph, pend);
    if (!ok) break;
    // the fold's first head: its key rows have the weight box's shape
    __syncthreads();
    if (static_cast<int>(blockIdx.x) < D / 64) {
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&mb[0], 64 * D * 2);
        tma_load_3d(sm, &a.wk, &mb[0], 0, static_cast<int>(blockIdx.x) * 64, 0);
      }
      pend |= 1;
    }
    if (!(ok = gt_grid_sync(a.bar, gen))) break;
    ok = pt_fold(a, sm, mb, ph, pend);
  } while (false);
  if (pend & 1) (void)mbar_wait(&mb[0], ph[0]);
  if (pend & 2) (void)mbar_wait(&mb[1], ph[1]);
  if (!ok && threadIdx.x == 0) atomicOr(a.status, DEV_WAIT_TIMEOUT);
}

}  // namespace

bool pool_tail_supported(int D, int heads) {
  // one head of 64 per projection item, at most 16 heads, the staged rows
  // of the widest projection within shared memory
  return heads * 64 == D && heads <= 16 && D % 128 == 0 && D >= 256 && D <= 1024;
}

int launch_pool_tail(const ivc_router* r, int l, const float* Zp, const float* mstat,
                     const float* lstat, int T, float* O, float* q, float* Q, bf16* U2, float* cb,
                     unsigned* bar, const Launch& L) {
  if (T == 0) return IVC_OK;
  const int D = r->D;
  if (!pool_tail_supported(D, r->heads)) return IVC_EUNSUPPORTED;
  PoolTailArgs a{};
  const unsigned long long d[3] = {64, static_cast<unsigned long long>(D),
                                   static_cast<unsigned long long>(D / 64)};
  const unsigned long long st[2] = {static_cast<unsigned long long>(D) * 2, 128};
  const unsigned box[3] = {64, 64, static_cast<unsigned>(D / 64)};
  a.last = l == 3 ? 1 : 0;
  if (map_bf16(&a.wv, 3, r->Wv[l], d, st, box) != IVC_OK) return IVC_ECUDA;
  if (map_bf16(&a.wo, 3, r->Wo[l], d, st, box) != IVC_OK) return IVC_ECUDA;
  if (!a.last) {
    if (map_bf16(&a.wq, 3, r->Wq[l + 1], d, st, box) != IVC_OK) return IVC_ECUDA;
    if (map_bf16(&a.wk, 3, r->Wk[l + 1], d, st, box) != IVC_OK) return IVC_ECUDA;
    a.bq = static_cast<const bf16*>(r->bq[l + 1]);
    a.bk = static_cast<const bf16*>(r->bk[l + 1]);
  }
  a.Zp = Zp;
  a.mstat = mstat;
  a.lstat = lstat;
  a.bv = static_cast<const bf16*>(r->bv[l]);
  a.bo = static_cast<const bf16*>(r->bo[l]);
  a.T = T;
  a.D = D;
  a.O = O;
  a.q = q;
  a.Q = Q;
  a.U2 = U2;
  a.cb = cb;
  a.bar = bar;
  a.status = L.status;
  const size_t smem = GtSmem<64>::total(D);
  if (smem_optin(reinterpret_cast<const void*>(pool_tail_kernel), smem) != IVC_OK)
    return IVC_ECUDA;
  if (cudaMemsetAsync(bar, 0, sizeof(unsigned), L.stream) != cudaSuccess) return IVC_ECUDA;
  TraceScope ts("pool.tail", L.stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(D / 64);
  cfg.blockDim = dim3(GT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cu_check(cudaLaunchKernelEx(&cfg, pool_tail_kernel, a));
}

bool gating_fused_supported(int D, int G) {
  // widths of 256..2048 (multiples of 128 for the warps' k-slices); the
  // LN row buffer must fit in the input-row region
  return D % 128 == 0 && G % 128 == 0 && D >= 256 && G >= 256 && D <= 2048 && G <= 2048;
}

int launch_gating_fused(const float* pooled, int T, int D, int G, const ivc_router* r, float* h,
                        float* u1, float* u2, float* gate, unsigned* bar, const Launch& L) {
  if (T == 0) return IVC_OK;
  if (!gating_fused_supported(D, G)) return IVC_EUNSUPPORTED;
  GatingArgs a{};
  const int cols = (D > G ? D : G) <= 1024 ? 64 : 16;
  for (int b = 0; b < 4; ++b) {
    const unsigned long long d1[3] = {64, static_cast<unsigned long long>(G),
                                      static_cast<unsigned long long>(D / 64)};
    const unsigned long long s1[2] = {static_cast<unsigned long long>(D) * 2, 128};
    const unsigned b1[3] = {64, static_cast<unsigned>(cols), static_cast<unsigned>(D / 64)};
    if (map_bf16(&a.w1[b], 3, r->gW1[b], d1, s1, b1) != IVC_OK) return IVC_ECUDA;
    const unsigned long long d2[3] = {64, static_cast<unsigned long long>(D),
                                      static_cast<unsigned long long>(G / 64)};
    const unsigned long long s2[2] = {static_cast<unsigned long long>(G) * 2, 128};
    const unsigned b2[3] = {64, static_cast<unsigned>(cols), static_cast<unsigned>(G / 64)};
    if (map_bf16(&a.w2[b], 3, r->gW2[b], d2, s2, b2) != IVC_OK) return IVC_ECUDA;
    a.b1[b] = static_cast<const bf16*>(r->gb1[b]);
    a.b2[b] = static_cast<const bf16*>(r->gb2[b]);
    a.ln_g[b] = static_cast<const bf16*>(r->gln_g[b]);
    a.ln_b[b] = static_cast<const bf16*>(r->gln_b[b]);
  }
  a.pooled = pooled;
  a.Wout = static_cast<const bf16*>(r->gWout);
  a.bout = static_cast<const bf16*>(r->gbout);
  a.T = T;
  a.D = D;
  a.G = G;
  a.inside = r->gate_residual;
  a.h = h;
  a.u1 = u1;
  a.u2 = u2;
  a.gate = gate;
  a.bar = bar;
  a.status = L.status;
  // one item of `cols` columns per CTA for the wider of the two projections
  int ctas = (D > G ? D : G) / cols;
  if (ctas > GT_MAX_CTAS) ctas = GT_MAX_CTAS;
  return cols == 64 ? launch_gating_cols<64>(a, ctas, L) : launch_gating_cols<16>(a, ctas, L);
}

}  // namespace ivc
