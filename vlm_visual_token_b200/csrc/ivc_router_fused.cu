// ivc_router_fused.cu — the whole ViR router (folded CrossAttentionPooling,
// Gating, routing) as one persistent cooperative kernel.
//
// InternVL3_5-4B-Flash "Gating and CrossAttentionPooling" article, sections
// 2-4: a learnable query refined by 4 masked multi-head cross-attention
// layers over a tile's tokens; Gating = 4 residual blocks (Linear -> GELU ->
// Linear -> LayerNorm) and Linear(D, 2) + softmax; gate > quantile(gate, 0.1)
// and gate >= 0.5 per image.
//
// The router is a chain of ~34 small dependent steps (vector-matrix
// products with 2 MB weights, two thin contractions with each tile's raw
// features per pooling layer, row LayerNorms). As separate kernels each
// step costs a launch and several memory round trips (~8 us per step on
// B200). Here all steps run in one launch: CTAs (one per SM) work through a
// phase's items, then meet at a software grid barrier (co-residency is
// guaranteed by the cooperative launch; every wait is bounded). Per pooling
// layer (the folded form of the single-query attention, see ivc_router.cu):
//   fold     u_h = Wk_h^T Q_h / 8, c_h = bk_h . Q_h / 8   (hi/lo bf16 split of u)
//   scores   s[t, h] = x_t . u_h  for every token        (mma.sync, fp32 accumulate)
//   softmax  p = softmax over the valid tokens, split hi/lo bf16
//   wsum     z_h = sum_t p_t x_t                          (mma.sync, fp32 accumulate)
//   vproj    o_h = Wv_h z_h + bv_h
//   oproj    q = Wo o + bo;  then Q of the next layer = Wq q + bq.
// Gating: u1 = GELU(W1 h + b1), u2 = W2 u1 + b2, then the residual LayerNorm,
// each a phase of its own. Selected with IVC_ROUTER_FUSED=1; the separate
// kernels stay the default while they measure faster.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdlib>

#include "ivc_internal.h"
#include "ivc_ptx.cuh"

namespace ivc {
namespace {

constexpr int RF_THREADS = 256;
constexpr int RF_WARPS = RF_THREADS / 32;
constexpr int RF_TOK = 1024;      // tokens per tile
constexpr int RF_HD = 64;         // head width
constexpr int RF_GEMV_COLS = 16;  // output columns per GEMV item (2 per warp)
constexpr int RF_ROWS = 16;       // input rows staged per GEMV round
constexpr int RF_MAXK = 2048;     // widest GEMV input

struct RouterFusedArgs {
  const bf16* x;  // [T, 1024, D]
  const int32_t* valid_len;
  int T, D, G, heads;
  const bf16 *query, *Wq[4], *bq[4], *Wk[4], *bk[4], *Wv[4], *bv[4], *Wo[4], *bo[4];
  const bf16 *gW1[4], *gb1[4], *gW2[4], *gb2[4], *gln_g[4], *gln_b[4], *gWout, *gbout;
  const int32_t* image_offsets;
  int I, scope, gate_inside;
  double rel_q, abs_t;
  // scratch
  float* Q;     // [T, D]
  bf16* U2;     // [T, 32, D]
  float* cb;    // [T, 16]
  float* S;     // [T, 32, 1024] split scores, token-contiguous
  bf16* P2;     // [T, 32, 1024] split softmax weights
  float* z;     // [T, 16, D]
  float* O;     // [T, D]
  float* q;     // [T, D]
  float* h;     // [T, D]
  float* u1;    // [T, G]
  float* u2;    // [T, D]
  unsigned* bar;  // [2]: arrival counter, generation (zeroed before launch)
  // outputs
  float* gate;
  uint8_t* mask;
  int32_t* offsets;
  int32_t* total;
  int* status;
};

__device__ __forceinline__ float gelu(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

// Grid-wide barrier over co-resident CTAs: one arrival counter that only
// grows (barrier g completes when it reaches (g + 1) * gridDim.x), so no CTA
// has to reset it; false after ~1 s without progress.
__device__ bool grid_sync(unsigned* bar, unsigned& gen) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned target = (gen + 1u) * gridDim.x;
    __threadfence();
    atomicAdd(bar, 1u);
    const long long t0 = clock64();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (static_cast<int>(v - target) >= 0) break;
      if (clock64() - t0 > IVC_WAIT_CYCLES) {
        ok = 0;
        break;
      }
      __nanosleep(20);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  ++gen;
  return s_ok != 0;
}

// ------------------------------------------------------------------ mma.sync
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copies `rows` rows of `bytes` (multiple of 16) from src (row pitch
// src_pitch bytes) into shared memory (row pitch dst_pitch bytes) with
// 16-byte cp.async pieces, all in flight at once; caller commits/waits.
__device__ __forceinline__ void async_rows(void* dst, int dst_pitch, const void* src,
                                           long long src_pitch, int rows, int bytes) {
  const int per_row = bytes >> 4;
  const int n = rows * per_row;
  for (int i = threadIdx.x; i < n; i += RF_THREADS) {
    const int r = i / per_row, p = i - r * per_row;
    cp_async16(static_cast<uint8_t*>(dst) + r * dst_pitch + p * 16,
               static_cast<const uint8_t*>(src) + r * src_pitch + p * 16);
  }
}

// ------------------------------------------------------------------ GEMV phase
// Y[m, n] = act(sum_k X(m)[k] W[n, k] + b[n]) for m < M. Items are blocks of
// RF_GEMV_COLS columns (warp w owns columns 2w, 2w+1 of the item). The item's
// weight rows (bf16) and up to RF_ROWS input rows (fp32, `row(m, c0)` = the
// input row of output row m for the item's columns c0..) are staged with
// cp.async in one go, then the dot products run from shared memory.
// Shared memory: RF_ROWS*K*4 (x) + RF_GEMV_COLS*K*2 (w).
template <typename RowFn>
__device__ void gemv_phase(int M, int K, int N, const bf16* __restrict__ W,
                           const bf16* __restrict__ b, float* __restrict__ Y, int ldy, bool act,
                           float* sx, RowFn row) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = (N + RF_GEMV_COLS - 1) / RF_GEMV_COLS;
  bf16* sw = reinterpret_cast<bf16*>(sx + RF_ROWS * K);
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int c0 = item * RF_GEMV_COLS;
    const int wrows = min(RF_GEMV_COLS, N - c0);
    for (int m0 = 0; m0 < M; m0 += RF_ROWS) {
      const int rows = min(RF_ROWS, M - m0);
      __syncthreads();
      if (m0 == 0) async_rows(sw, K * 2, W + static_cast<long long>(c0) * K, K * 2LL, wrows, K * 2);
      for (int r = 0; r < rows; ++r) async_rows(sx + r * K, K * 4, row(m0 + r, c0), 0, 1, K * 4);
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      const int n = c0 + 2 * warp;
      float acc[RF_ROWS][2];
#pragma unroll
      for (int r = 0; r < RF_ROWS; ++r) acc[r][0] = acc[r][1] = 0.f;
      const bf16* w0 = sw + min(2 * warp, wrows - 1) * K;
      const bf16* w1 = sw + min(2 * warp + 1, wrows - 1) * K;
      for (int k = lane * 4; k < K; k += 128) {
        const uint2 a = *reinterpret_cast<const uint2*>(w0 + k);
        const uint2 c = *reinterpret_cast<const uint2*>(w1 + k);
        const float wa[4] = {__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xffff0000u),
                             __uint_as_float(a.y << 16), __uint_as_float(a.y & 0xffff0000u)};
        const float wc[4] = {__uint_as_float(c.x << 16), __uint_as_float(c.x & 0xffff0000u),
                             __uint_as_float(c.y << 16), __uint_as_float(c.y & 0xffff0000u)};
#pragma unroll
        for (int r = 0; r < RF_ROWS; ++r) {
          if (r < rows) {
            const float4 xv = *reinterpret_cast<const float4*>(sx + r * K + k);
            acc[r][0] = fmaf(wa[0], xv.x, fmaf(wa[1], xv.y, fmaf(wa[2], xv.z, fmaf(wa[3], xv.w, acc[r][0]))));
            acc[r][1] = fmaf(wc[0], xv.x, fmaf(wc[1], xv.y, fmaf(wc[2], xv.z, fmaf(wc[3], xv.w, acc[r][1]))));
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RF_ROWS; ++r) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          acc[r][0] += __shfl_xor_sync(0xffffffffu, acc[r][0], o);
          acc[r][1] += __shfl_xor_sync(0xffffffffu, acc[r][1], o);
        }
      }
      if (lane < 2 && n + lane < N) {
        const float bias = b ? __bfloat162float(b[n + lane]) : 0.f;
#pragma unroll
        for (int r = 0; r < RF_ROWS; ++r) {
          if (r < rows) {
            float y = (lane == 0 ? acc[r][0] : acc[r][1]) + bias;
            if (act) y = gelu(y);
            Y[static_cast<long long>(m0 + r) * ldy + n + lane] = y;
          }
        }
      }
    }
  }
}

// dst = h + LN(u) * gamma + beta (inside = 0) or LN(h + u) * gamma + beta
// (inside = 1) for one row of D values (block-wide reductions). dst is a
// shared-memory row; it first holds the LayerNorm input.
__device__ void residual_ln_row(const float* __restrict__ hrow, const float* __restrict__ urow0,
                                const bf16* __restrict__ g, const bf16* __restrict__ bta,
                                float* dst, int D, int inside) {
  for (int i = threadIdx.x; i < D; i += RF_THREADS) dst[i] = inside ? hrow[i] + urow0[i] : urow0[i];
  __syncthreads();
  const float* urow = dst;
  __shared__ float s_red[RF_WARPS];
  __shared__ float s_stat[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float s = 0.f;
  for (int i = threadIdx.x; i < D; i += RF_THREADS) s += urow[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) s_red[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < RF_WARPS; ++i) t += s_red[i];
    s_stat[0] = t / D;
  }
  __syncthreads();
  const float mean = s_stat[0];
  float v = 0.f;
  for (int i = threadIdx.x; i < D; i += RF_THREADS) {
    const float d = urow[i] - mean;
    v = fmaf(d, d, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < RF_WARPS; ++i) t += s_red[i];
    s_stat[1] = 1.0f / sqrtf(t / D + 1e-5f);
  }
  __syncthreads();
  const float rstd = s_stat[1];
  for (int i = threadIdx.x; i < D; i += RF_THREADS) {
    const float n = (urow[i] - mean) * rstd * __bfloat162float(g[i]) + __bfloat162float(bta[i]);
    dst[i] = inside ? n : hrow[i] + n;
  }
}

// ------------------------------------------------------------------ fold phase
// Items (c-block of 128, head): U2[t][h][c] hi, U2[t][16+h][c] lo of
// u = Wk[h*64.., c] . Q[t, h*64..] / 8; cb[t][h] = bk . Q / 8 (c-block 0).
__device__ void fold_phase(const RouterFusedArgs& a, int l, int Tq, const float* __restrict__ Q,
                           long long ldq, float* s_q) {
  const int D = a.D;
  const int cblocks = D / 128;
  const int n_items = cblocks * a.heads;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int h = item / cblocks, cbk = item % cblocks;
    const int tid = threadIdx.x & 127;   // column within the block
    const int half = threadIdx.x >> 7;   // two halves share the tiles
    const int c = cbk * 128 + tid;
    float w[RF_HD];
#pragma unroll
    for (int d = 0; d < RF_HD; ++d)
      w[d] = __bfloat162float(a.Wk[l][static_cast<long long>(h * RF_HD + d) * D + c]);
    for (int t0 = 0; t0 < Tq; t0 += 64) {
      const int nt = min(64, Tq - t0);
      __syncthreads();
      for (int i = threadIdx.x; i < nt * RF_HD; i += RF_THREADS)
        s_q[i] = Q[(t0 + i / RF_HD) * ldq + h * RF_HD + i % RF_HD] * 0.125f;
      __syncthreads();
      for (int t = half; t < nt; t += 2) {
        float u = 0.f;
#pragma unroll
        for (int d = 0; d < RF_HD; ++d) u = fmaf(w[d], s_q[t * RF_HD + d], u);
        const bf16 hi = __float2bfloat16_rn(u);
        const bf16 lo = __float2bfloat16_rn(u - __bfloat162float(hi));
        bf16* base = a.U2 + static_cast<long long>(t0 + t) * 32 * D;
        base[static_cast<long long>(h) * D + c] = hi;
        base[static_cast<long long>(16 + h) * D + c] = lo;
      }
      if (cbk == 0 && threadIdx.x < nt) {
        float acc = 0.f;
        for (int d = 0; d < RF_HD; ++d)
          acc = fmaf(a.bk[l] ? __bfloat162float(a.bk[l][h * RF_HD + d]) : 0.f,
                     s_q[threadIdx.x * RF_HD + d], acc);
        a.cb[(t0 + threadIdx.x) * 16 + h] = acc;
      }
    }
  }
}

// ------------------------------------------------------------------ scores phase
// Items (tile, 64-token block). St[tile][j][t] = sum_c x[tile][t][c] U2[tu][j][c],
// j < 32 (hi rows 0..15, lo rows 16..31); tu = tile, or 0 when the query is
// shared. The item's 64 token rows and the tile's 32 U2 rows are staged in
// one cp.async batch; warp w computes m16 tile (w & 3) x n8 tiles
// 2(w >> 2), 2(w >> 2) + 1 with m16n8k16 bf16 MMAs over all channels.

__device__ void scores_phase(const RouterFusedArgs& a, bool shared_query, bf16* sm) {
  const int D = a.D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pitch = D + 8;
  const int n_items = a.T * (RF_TOK / 64);
  bf16* sx = sm;               // [64][pitch]
  bf16* su = sm + 64 * pitch;  // [32][pitch]
  const int mt = warp & 3, nb0 = 2 * (warp >> 2);
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int tile = item / (RF_TOK / 64), tb = item % (RF_TOK / 64);
    __syncthreads();
    async_rows(sx, pitch * 2, a.x + (static_cast<long long>(tile) * RF_TOK + tb * 64) * D, D * 2LL,
               64, D * 2);
    async_rows(su, pitch * 2, a.U2 + static_cast<long long>(shared_query ? 0 : tile) * 32 * D,
               D * 2LL, 32, D * 2);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    float acc[2][4] = {};
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t af[4];
      ldsm_x4(af, sx + (mt * 16 + (lane & 15)) * pitch + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t bfr[2];
        ldsm_x2(bfr, su + ((nb0 + q) * 8 + (lane & 7)) * pitch + ks * 16 + ((lane >> 3) & 1) * 8);
        mma_bf16_16816(acc[q], af, bfr);
      }
    }
    float* st = a.S + static_cast<long long>(tile) * 32 * RF_TOK + tb * 64 + mt * 16;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int j = (nb0 + q) * 8 + t2;
      st[static_cast<long long>(j) * RF_TOK + g] = acc[q][0];
      st[static_cast<long long>(j + 1) * RF_TOK + g] = acc[q][1];
      st[static_cast<long long>(j) * RF_TOK + g + 8] = acc[q][2];
      st[static_cast<long long>(j + 1) * RF_TOK + g + 8] = acc[q][3];
    }
  }
}

// ------------------------------------------------------------------ softmax phase
// Items (tile, head): p = softmax over the valid tokens of hi + lo + c, written
// as a bf16 hi/lo pair into rows h and 16 + h of P2[tile] (zero rows for heads
// that do not exist).
__device__ void softmax_phase(const RouterFusedArgs& a, bool shared_cb, float* sf) {
  __shared__ float s_red[RF_WARPS];
  __shared__ float s_val;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.T * 16;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int tile = item / 16, h = item % 16;
    bf16* prow = a.P2 + (static_cast<long long>(tile) * 32 + h) * RF_TOK;
    bf16* lrow = prow + 16 * RF_TOK;
    if (h >= a.heads) {
      for (int t = threadIdx.x; t < RF_TOK; t += RF_THREADS)
        prow[t] = lrow[t] = __float2bfloat16_rn(0.f);
      continue;
    }
    int n = RF_TOK;
    if (a.valid_len) {
      n = a.valid_len[tile];
      if (n < 1 || n > RF_TOK) {
        if (threadIdx.x == 0 && h == 0) atomicOr(a.status, DEV_BAD_VALID_LEN);
        n = n < 1 ? 1 : RF_TOK;
      }
    }
    const float c = a.cb[(shared_cb ? 0 : tile) * 16 + h];
    const float* shi = a.S + (static_cast<long long>(tile) * 32 + h) * RF_TOK;
    const float* slo = shi + 16 * RF_TOK;
    float v[RF_TOK / RF_THREADS];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < RF_TOK / RF_THREADS; ++u) {
      const int t = threadIdx.x + u * RF_THREADS;
      v[u] = shi[t] + slo[t] + c;
      if (t < n) mx = fmaxf(mx, v[u]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __syncthreads();
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = s_red[0];
      for (int i = 1; i < RF_WARPS; ++i) m = fmaxf(m, s_red[i]);
      s_val = m;
    }
    __syncthreads();
    mx = s_val;
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < RF_TOK / RF_THREADS; ++u) {
      const int t = threadIdx.x + u * RF_THREADS;
      v[u] = t < n ? expf(v[u] - mx) : 0.f;
      sum += v[u];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    __syncthreads();
    if (lane == 0) s_red[warp] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int i = 0; i < RF_WARPS; ++i) t += s_red[i];
      s_val = 1.0f / t;
    }
    __syncthreads();
    const float inv = s_val;
#pragma unroll
    for (int u = 0; u < RF_TOK / RF_THREADS; ++u) {
      const int t = threadIdx.x + u * RF_THREADS;
      const float p = v[u] * inv;
      const bf16 hi = __float2bfloat16_rn(p);
      prow[t] = hi;
      lrow[t] = __float2bfloat16_rn(p - __bfloat162float(hi));
    }
  }
  (void)sf;
}

// ------------------------------------------------------------------ wsum phase
// Items (tile, 64-channel block): z[tile][h][c] = sum_t (P_hi + P_lo)[h][t] x[tile][t][c].
// P2[tile] (32 x 1024) and the tile's x columns (1024 tokens x 64 channels)
// are staged in one cp.async batch; warp w computes channels 8w..8w+7 (one n8
// tile) for both m16 tiles (hi rows, lo rows) over all 1024 tokens.
constexpr int WS_PPITCH = RF_TOK + 8;  // bf16 per staged P2 row
constexpr int WS_XPITCH = 64 + 8;      // bf16 per staged x row (64 channels)

__device__ void wsum_phase(const RouterFusedArgs& a, bf16* sm) {
  const int D = a.D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cblocks = D / 64;
  const int n_items = a.T * cblocks;
  bf16* sp = sm;                     // [32][WS_PPITCH]
  bf16* sx = sm + 32 * WS_PPITCH;    // [1024][WS_XPITCH]
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  int staged_tile = -1;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int tile = item / cblocks, cbk = item % cblocks;
    __syncthreads();
    if (tile != staged_tile)
      async_rows(sp, WS_PPITCH * 2, a.P2 + static_cast<long long>(tile) * 32 * RF_TOK,
                 RF_TOK * 2LL, 32, RF_TOK * 2);
    staged_tile = tile;
    async_rows(sx, WS_XPITCH * 2, a.x + static_cast<long long>(tile) * RF_TOK * D + cbk * 64,
               D * 2LL, RF_TOK, 128);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    float acc[2][4] = {};
    for (int ks = 0; ks < RF_TOK / 16; ++ks) {
      uint32_t bfr[2];
      // B[k = token][n = channel] stored n-contiguous: transposed 8x8 loads
      ldsm_x2_trans(bfr, sx + (ks * 16 + (lane & 15)) * WS_XPITCH + warp * 8);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        uint32_t af[4];
        ldsm_x4(af, sp + (mt * 16 + (lane & 15)) * WS_PPITCH + ks * 16 + (lane >> 4) * 8);
        mma_bf16_16816(acc[mt], af, bfr);
      }
    }
    // row g of m-tile 0 is the hi part of head g, row g of m-tile 1 its lo part
    float* zt = a.z + static_cast<long long>(tile) * 16 * D + cbk * 64 + warp * 8 + t2;
    *reinterpret_cast<float2*>(zt + static_cast<long long>(g) * D) =
        make_float2(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1]);
    *reinterpret_cast<float2*>(zt + static_cast<long long>(g + 8) * D) =
        make_float2(acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
  }
}

// ------------------------------------------------------------------ routing
__device__ void route_phase(const RouterFusedArgs& a, double* s_vals, double* s_sorted) {
  if (blockIdx.x != 0) return;
  __shared__ double s_qv;
  __shared__ int s_bad;
  __shared__ int s_warp[RF_WARPS];
  __shared__ int s_carry;
  const int T = a.T;
  if (threadIdx.x == 0) {
    int bad = 0;
    if (a.scope == 0) {
      if (a.image_offsets[0] != 0 || a.image_offsets[a.I] != T) bad = 1;
      for (int i = 0; i < a.I && !bad; ++i)
        if (a.image_offsets[i + 1] < a.image_offsets[i]) bad = 1;
      if (bad) atomicOr(a.status, DEV_BAD_OFFSETS);
    }
    s_bad = bad;
  }
  __syncthreads();
  const int groups = a.scope == 0 ? a.I : 1;
  for (int gi = 0; gi < groups; ++gi) {
    int s = 0, e = T;
    if (a.scope == 0) {
      if (s_bad) break;
      s = a.image_offsets[gi];
      e = a.image_offsets[gi + 1];
    }
    const int n = e - s;
    if (n <= 0) continue;
    if (n > IVC_MAX_QUANTILE_GROUP) {
      if (threadIdx.x == 0) atomicOr(a.status, DEV_GROUP_TOO_LARGE);
      for (int i = threadIdx.x; i < n; i += RF_THREADS) a.mask[s + i] = 0;
      __syncthreads();
      continue;
    }
    for (int i = threadIdx.x; i < n; i += RF_THREADS) s_vals[i] = static_cast<double>(a.gate[2 * (s + i)]);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += RF_THREADS) {
      const double v = s_vals[i];
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const double u = s_vals[j];
        rank += (u < v) || (u == v && j < i);
      }
      s_sorted[rank] = v;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const double pos = __dmul_rn(a.rel_q, static_cast<double>(n - 1));
      const double flo = floor(pos);
      const int lo = static_cast<int>(flo);
      const int hi = static_cast<int>(ceil(pos));
      const double w = __dsub_rn(pos, flo);
      const double diff = __dsub_rn(s_sorted[hi], s_sorted[lo]);
      s_qv = __dadd_rn(s_sorted[lo], __dmul_rn(w, diff));
    }
    __syncthreads();
    const double qv = s_qv;
    for (int i = threadIdx.x; i < n; i += RF_THREADS) {
      const double v = s_vals[i];
      a.mask[s + i] = (v > qv && v >= a.abs_t) ? 1 : 0;
    }
    __syncthreads();
  }
  if (a.scope == 0 && s_bad)
    for (int i = threadIdx.x; i < T; i += RF_THREADS) a.mask[i] = 0;
  __syncthreads();
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int base = 0; base < T; base += RF_THREADS) {
    const int i = base + threadIdx.x;
    const int cnt = i < T ? (a.mask[i] ? 64 : 256) : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = lane < RF_WARPS ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += v;
      }
      if (lane < RF_WARPS) s_warp[lane] = w;
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + s_carry;
    if (i < T) a.offsets[i] = before + incl - cnt;
    __syncthreads();
    if (threadIdx.x == RF_THREADS - 1) s_carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    a.offsets[T] = s_carry;
    if (a.total) *a.total = s_carry;
  }
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(RF_THREADS, 1)
    router_fused_kernel(const __grid_constant__ RouterFusedArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* sf = reinterpret_cast<float*>(smem);
  bf16* sb = reinterpret_cast<bf16*>(smem);
  unsigned gen = 0;
  bool ok = true;
  const int T = a.T, D = a.D, G = a.G;
  auto sync = [&]() {
    if (ok) ok = grid_sync(a.bar, gen);
    return ok;
  };
  // layer 1's query is shared by all tiles: Q1 = Wq_1 query + bq_1 in row 0 of Q
  // (the bf16 query is widened into h first)
  if (blockIdx.x == 0)
    for (int k = threadIdx.x; k < D; k += RF_THREADS) a.h[k] = __bfloat162float(a.query[k]);
  if (sync())
    gemv_phase(1, D, D, a.Wq[0], a.bq[0], a.Q, D, false, sf, [&](int, int) { return a.h; });
  for (int l = 0; l < 4; ++l) {
    if (!sync()) break;
    const bool shared_q = l == 0;
    fold_phase(a, l, shared_q ? 1 : T, a.Q, shared_q ? 0 : D, sf);
    if (!sync()) break;
    scores_phase(a, shared_q, sb);
    if (!sync()) break;
    softmax_phase(a, shared_q, sf);
    if (!sync()) break;
    wsum_phase(a, sb);
    if (!sync()) break;
    // o = Wv_h z_h + bv: the input row of output row m for columns of head h is z[m][h]
    gemv_phase(T, D, D, a.Wv[l], a.bv[l], a.O, D, false, sf, [&](int m, int c0) {
      return a.z + (static_cast<long long>(m) * 16 + c0 / RF_HD) * D;
    });
    if (!sync()) break;
    gemv_phase(T, D, D, a.Wo[l], a.bo[l], a.q, D, false, sf,
               [&](int m, int) { return a.O + static_cast<long long>(m) * D; });
    if (l < 3) {
      if (!sync()) break;
      gemv_phase(T, D, D, a.Wq[l + 1], a.bq[l + 1], a.Q, D, false, sf,
                 [&](int m, int) { return a.q + static_cast<long long>(m) * D; });
    }
  }
  // Gating: h_0 = pooled = q; block b: u1 = GELU(W1 h_b + b1), u2 = W2 u1 + b2,
  // h_{b+1} = h_b + LN_b(u2) (rows spread over the CTAs, kept in h).
  for (int b = 0; b < 4; ++b) {
    if (!sync()) break;
    const float* hb = b == 0 ? a.q : a.h;
    gemv_phase(T, D, G, a.gW1[b], a.gb1[b], a.u1, G, true, sf,
               [&](int m, int) { return hb + static_cast<long long>(m) * D; });
    if (!sync()) break;
    gemv_phase(T, G, D, a.gW2[b], a.gb2[b], a.u2, D, false, sf,
               [&](int m, int) { return a.u1 + static_cast<long long>(m) * G; });
    if (!sync()) break;
    for (int m = blockIdx.x; m < T; m += gridDim.x) {
      residual_ln_row(hb + static_cast<long long>(m) * D, a.u2 + static_cast<long long>(m) * D,
                      a.gln_g[b], a.gln_b[b], sf, D, a.gate_inside);
      __syncthreads();
      for (int i = threadIdx.x; i < D; i += RF_THREADS) a.h[static_cast<long long>(m) * D + i] = sf[i];
      __syncthreads();
    }
  }
  // head: gate = softmax(Wout h_4 + bout), one warp per tile
  if (ok && sync()) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = blockIdx.x * RF_WARPS + warp; t < T; t += gridDim.x * RF_WARPS) {
      const float* hr = a.h + static_cast<long long>(t) * D;
      float l0 = 0.f, l1 = 0.f;
      for (int i = lane; i < D; i += 32) {
        const float v = hr[i];
        l0 = fmaf(__bfloat162float(a.gWout[i]), v, l0);
        l1 = fmaf(__bfloat162float(a.gWout[D + i]), v, l1);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      if (lane == 0) {
        if (a.gbout) {
          l0 += __bfloat162float(a.gbout[0]);
          l1 += __bfloat162float(a.gbout[1]);
        }
        const float mx = fmaxf(l0, l1);
        const float e0 = expf(l0 - mx), e1 = expf(l1 - mx);
        a.gate[2 * t] = e0 / (e0 + e1);
        a.gate[2 * t + 1] = e1 / (e0 + e1);
      }
    }
  }
  if (ok && sync())
    route_phase(a, reinterpret_cast<double*>(smem),
                reinterpret_cast<double*>(smem) + IVC_MAX_QUANTILE_GROUP);
  if (!ok && threadIdx.x == 0) atomicOr(a.status, DEV_WAIT_TIMEOUT);
}

size_t router_fused_smem(int D, int G) {
  const size_t K = static_cast<size_t>(D > G ? D : G);
  const size_t gemv = K * (RF_ROWS * sizeof(float) + RF_GEMV_COLS * sizeof(bf16));
  const size_t route = 2 * static_cast<size_t>(IVC_MAX_QUANTILE_GROUP) * sizeof(double);
  const size_t scores = static_cast<size_t>(96) * (D + 8) * sizeof(bf16);
  const size_t wsum = (static_cast<size_t>(32) * WS_PPITCH + static_cast<size_t>(RF_TOK) * WS_XPITCH) *
                      sizeof(bf16);
  size_t m = gemv;
  if (route > m) m = route;
  if (scores > m) m = scores;
  if (wsum > m) m = wsum;
  return m;
}

}  // namespace

bool router_fused_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("IVC_ROUTER_FUSED");
    on = (e && e[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

int launch_router_fused(const ivc_router* r, const void* x, const int32_t* valid_len, int T,
                        const int32_t* image_offsets, int I, float* gate, uint8_t* mask,
                        int32_t* offsets, int32_t* total, const FusedRouterBufs& b,
                        const Launch& L) {
  if (T == 0) return IVC_OK;
  if (r->D % 128 != 0 || r->heads > 16 || r->D > RF_MAXK || r->gate_hidden > RF_MAXK)
    return IVC_EUNSUPPORTED;
  RouterFusedArgs a{};
  a.x = static_cast<const bf16*>(x);
  a.valid_len = valid_len;
  a.T = T;
  a.D = r->D;
  a.G = r->gate_hidden;
  a.heads = r->heads;
  a.query = static_cast<const bf16*>(r->query);
  for (int l = 0; l < 4; ++l) {
    a.Wq[l] = static_cast<const bf16*>(r->Wq[l]);
    a.bq[l] = static_cast<const bf16*>(r->bq[l]);
    a.Wk[l] = static_cast<const bf16*>(r->Wk[l]);
    a.bk[l] = static_cast<const bf16*>(r->bk[l]);
    a.Wv[l] = static_cast<const bf16*>(r->Wv[l]);
    a.bv[l] = static_cast<const bf16*>(r->bv[l]);
    a.Wo[l] = static_cast<const bf16*>(r->Wo[l]);
    a.bo[l] = static_cast<const bf16*>(r->bo[l]);
    a.gW1[l] = static_cast<const bf16*>(r->gW1[l]);
    a.gb1[l] = static_cast<const bf16*>(r->gb1[l]);
    a.gW2[l] = static_cast<const bf16*>(r->gW2[l]);
    a.gb2[l] = static_cast<const bf16*>(r->gb2[l]);
    a.gln_g[l] = static_cast<const bf16*>(r->gln_g[l]);
    a.gln_b[l] = static_cast<const bf16*>(r->gln_b[l]);
  }
  a.gWout = static_cast<const bf16*>(r->gWout);
  a.gbout = static_cast<const bf16*>(r->gbout);
  a.image_offsets = image_offsets;
  a.I = I;
  a.scope = r->quantile_scope;
  a.gate_inside = r->gate_residual;
  a.rel_q = r->rel_q;
  a.abs_t = r->abs_t;
  a.Q = b.Q;
  a.U2 = b.U2;
  a.cb = b.cb;
  a.S = b.S;
  a.P2 = b.P2;
  a.z = b.z;
  a.O = b.O;
  a.q = b.q;
  a.h = b.h;
  a.u1 = b.u1;
  a.u2 = b.u2;
  a.bar = b.bar;
  a.gate = gate;
  a.mask = mask;
  a.offsets = offsets;
  a.total = total;
  a.status = L.status;
  const size_t smem = router_fused_smem(r->D, r->gate_hidden);
  if (smem > 227 * 1024) return IVC_EUNSUPPORTED;
  if (cudaFuncSetAttribute(router_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return IVC_ECUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, router_fused_kernel, RF_THREADS,
                                                    smem) != cudaSuccess ||
      per_sm < 1)
    return IVC_ECUDA;
  const int grid = num_sms();  // one CTA per SM, all co-resident
  if (cudaMemsetAsync(b.bar, 0, 2 * sizeof(unsigned), L.stream) != cudaSuccess) return IVC_ECUDA;
  TraceScope ts("router.fused", L.stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(RF_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr1[1];
  attr1[0].id = cudaLaunchAttributeCooperative;
  attr1[0].val.cooperative = 1;
  cfg.attrs = attr1;
  cfg.numAttrs = 1;
  return cu_check(cudaLaunchKernelEx(&cfg, router_fused_kernel, a));
}

}  // namespace ivc
