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
//   attend   per 128-token chunk: s[t, h] = x_t . u_h + c_h, running softmax,
//            Zc_h = sum_t exp(s - m) x_t  (mma.sync, fp32 accumulate; x read once)
//   combine  z_h = softmax-weighted merge of the tile's 8 chunks
//   vproj    o_h = Wv_h z_h + bv_h
//   oproj    q = Wo o + bo;  then Q of the next layer = Wq q + bq.
// Gating: u1 = GELU(W1 h + b1), u2 = W2 u1 + b2, then the residual LayerNorm,
// each a phase of its own. This kernel is the default wherever nothing runs
// beside the router (ivc_vir_route, the router-first flow); beside the
// connector, where it would have to wait for every SM, the separate kernels
// are used. IVC_ROUTER_FUSED=1 / 0 forces the choice.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>

#include "ivc_internal.h"
#include "ivc_ptx.cuh"

namespace ivc {
namespace {

constexpr int RF_THREADS = 256;
constexpr int RF_WARPS = RF_THREADS / 32;
constexpr int RF_TOK = 1024;    // tokens per tile
constexpr int RF_HD = 64;       // head width
constexpr int RF_MAXD = 1024;   // widest pooling width (scores staging)
constexpr int RF_MAXK = 2048;   // widest projection input
constexpr int GV_COLS = 8;      // output columns per projection item (one n8 MMA tile)
constexpr int GV_ROWS = 16;     // input rows per projection round (one m16 MMA tile)
constexpr int SC_TOK = 32;      // tokens per staged step of the attention phase

struct RouterFusedArgs {
  // x as {64 ch, T*1024 tokens, D/64 chunks}, box {64, SC_TOK, D/64}, 128-byte
  // swizzle (one request per staged step)
  CUtensorMap xmap3;
  const bf16* x;      // [T, 1024, D]
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
  float* Zp;    // [T, 8 chunks, 16, D] unnormalised weighted sums per chunk
  float* stats; // [2][T, 8 chunks, 16]: running max m, then sum l
  float* z;     // [T, 16, D] merged weighted sums
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
  // > 0: the grid barriers from the one before the gating head on give up
  // after this many clock cycles (failure-detection tests; no bulk copy is
  // in flight at those barriers). 0: every barrier uses IVC_WAIT_CYCLES.
  long long late_wait_cycles;
};

__device__ __forceinline__ float gelu(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

// Grid-wide barrier over co-resident CTAs: one arrival counter that only
// grows (barrier g completes when it reaches (g + 1) * gridDim.x), so no CTA
// has to reset it. Arrival is a release reduction (this CTA's writes, ordered
// by the __syncthreads before it, become visible with it), the wait an
// acquire spin; false after ~1 s without progress.
__device__ bool grid_sync(unsigned* bar, unsigned& gen, long long limit) {
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
      if (clock64() - t0 > limit) {
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

// Bounded wait whose give-up is decided for the whole CTA: every thread waits,
// then one barrier combines the results, so no thread returns while others go
// on to a later CTA barrier.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity) {
  return __syncthreads_and(mbar_wait(bar, parity) ? 1 : 0) != 0;
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
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
// Orders this thread's later async-proxy (bulk copy / TMA) reads of global
// memory after generic writes that other CTAs made before a grid barrier.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// v = hi + lo with hi = bf16(v), lo = bf16(v - hi), two lanes packed per word.
__device__ __forceinline__ void split_bf16x2(float2 v, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 l = __floats2bfloat162_rn(v.x - __low2float(h), v.y - __high2float(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// ------------------------------------------------------------------ projection phase
// Y[m, n] = act(sum_k X(m)[k] W[n, k] + b[n]) for m < M (M = tiles, small).
// Items are GV_COLS = 8 output columns (one n8 MMA tile). Per item the 8
// weight rows (bf16, mbarrier 0) and up to 16 input rows (fp32, mbarrier 1;
// `row(m, c0)` = the input row of output row m for columns c0..c0+7) are
// brought into shared memory with bulk copies; warp w then multiplies the
// k-range [w K/8, (w+1) K/8) with m16n8k16 MMAs, the fp32 inputs split into a
// bf16 hi/lo pair (two MMAs per k-step, fp32 accumulate), and the 8 warps'
// partial tiles are summed through shared memory. Shared memory:
// x [16][K+8] f32 | w [8][K+8] bf16 | partials [8 warps][16][8] f32.
__device__ __forceinline__ size_t gv_x_bytes(int K) {
  return static_cast<size_t>(GV_ROWS) * (K + 8) * 4;
}
__device__ __forceinline__ size_t gv_w_bytes(int K) {
  return static_cast<size_t>(GV_COLS) * (K + 8) * 2;
}

// Warp 0: the weight rows of item `item` into their slot, on mbarrier mb.
__device__ __forceinline__ void gv_issue_w(const bf16* __restrict__ W, int K, int item,
                                           uint8_t* sm, uint64_t* mb) {
  const int lane = threadIdx.x & 31;
  bf16* sw = reinterpret_cast<bf16*>(sm + gv_x_bytes(K));
  if (lane == 0) mbar_arrive_expect_tx(mb, GV_COLS * K * 2);
  __syncwarp();
  if (lane < GV_COLS)
    bulk_load(sw + lane * (K + 8), W + static_cast<size_t>(item * GV_COLS + lane) * K, K * 2, mb);
}

// `pend` tracks the bulk copies this CTA has in flight on mbarriers 0 and 1
// (bits 0 and 1): bit 0 set on entry means the first item's weight rows were
// requested before the grid barrier. A bit is set when copies are issued and
// cleared only when their wait succeeds, so after a give-up (false) the
// kernel's exit still waits for every copy that may land in shared memory.
template <typename RowFn>
__device__ bool gemv_phase(int M, int K, int N, const bf16* __restrict__ W,
                           const bf16* __restrict__ b, float* __restrict__ Y, int ldy, bool act,
                           uint8_t* sm, uint64_t* mb, uint32_t* ph, int& pend, RowFn row) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  const int pitch = K + 8;
  float* sx = reinterpret_cast<float*>(sm);
  const bf16* sw = reinterpret_cast<const bf16*>(sm + gv_x_bytes(K));
  float* red = reinterpret_cast<float*>(sm + gv_x_bytes(K) + gv_w_bytes(K));
  const int n_items = N / GV_COLS;
  const int kw = K / RF_WARPS;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int c0 = item * GV_COLS;
    if (!(pend & 1)) {
      __syncthreads();  // the previous item's reads of the weight slot are done
      if (warp == 0) gv_issue_w(W, K, item, sm, &mb[0]);
      pend |= 1;
    }
    bool w_ready = false;
    for (int m0 = 0; m0 < M; m0 += GV_ROWS) {
      const int rows = min(GV_ROWS, M - m0);
      __syncthreads();  // the previous round's reads of x and the partials are done
      if (warp == 0) {
        if (lane == 0) mbar_arrive_expect_tx(&mb[1], rows * K * 4);
        __syncwarp();
        if (lane < rows) {
          fence_proxy_async_global();
          bulk_load(sx + lane * pitch, row(m0 + lane, c0), K * 4, &mb[1]);
        }
      }
      pend |= 2;
      if (!w_ready) {
        if (!cta_wait(&mb[0], ph[0])) return false;
        ph[0] ^= 1;
        pend &= ~1;
        w_ready = true;
      }
      if (!cta_wait(&mb[1], ph[1])) return false;
      ph[1] ^= 1;
      pend &= ~2;
      // rows >= `rows` of the A tile hold stale values; they only reach
      // output rows that are never stored
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const int kb = warp * kw;
      for (int ks = 0; ks < kw; ks += 16) {
        const int k = kb + ks + t2;
        uint32_t ah[4], al[4], bw[2];
        split_bf16x2(*reinterpret_cast<const float2*>(sx + g * pitch + k), ah[0], al[0]);
        split_bf16x2(*reinterpret_cast<const float2*>(sx + (g + 8) * pitch + k), ah[1], al[1]);
        split_bf16x2(*reinterpret_cast<const float2*>(sx + g * pitch + k + 8), ah[2], al[2]);
        split_bf16x2(*reinterpret_cast<const float2*>(sx + (g + 8) * pitch + k + 8), ah[3], al[3]);
        bw[0] = *reinterpret_cast<const uint32_t*>(sw + g * pitch + k);
        bw[1] = *reinterpret_cast<const uint32_t*>(sw + g * pitch + k + 8);
        mma_bf16_16816(acc, ah, bw);
        mma_bf16_16816(acc, al, bw);
      }
      float* rw = red + warp * (GV_ROWS * GV_COLS);
      rw[g * GV_COLS + t2] = acc[0];
      rw[g * GV_COLS + t2 + 1] = acc[1];
      rw[(g + 8) * GV_COLS + t2] = acc[2];
      rw[(g + 8) * GV_COLS + t2 + 1] = acc[3];
      __syncthreads();
      if (threadIdx.x < GV_ROWS * GV_COLS) {
        const int r = threadIdx.x / GV_COLS, c = threadIdx.x % GV_COLS;
        if (r < rows) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < RF_WARPS; ++w) v += red[w * GV_ROWS * GV_COLS + threadIdx.x];
          if (b) v += __bfloat162float(b[c0 + c]);
          if (act) v = gelu(v);
          Y[static_cast<size_t>(m0 + r) * ldy + c0 + c] = v;
        }
      }
    }
  }
  return true;
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
// The item's 64 x 128 block of Wk arrives by bulk copies on mbarrier 0 (the
// first item's before the grid barrier, see fold_issue_w); Q rows are read
// directly. Shared memory: Wk block [64][128] bf16 | Q block [64][64] f32.
__device__ __forceinline__ void fold_issue_w(const bf16* __restrict__ Wk, int D, int item,
                                             uint8_t* sm, uint64_t* mb) {
  const int lane = threadIdx.x & 31;
  const int cblocks = D / 128;
  const int h = item / cblocks, cbk = item % cblocks;
  bf16* sw = reinterpret_cast<bf16*>(sm);
  if (lane == 0) mbar_arrive_expect_tx(mb, RF_HD * 128 * 2);
  __syncwarp();
  for (int d = lane; d < RF_HD; d += 32)
    bulk_load(sw + d * 128, Wk + static_cast<size_t>(h * RF_HD + d) * D + cbk * 128, 256, mb);
}

// `pend`: as in gemv_phase (bit 0, the Wk block copies on mbarrier 0).
__device__ bool fold_phase(const RouterFusedArgs& a, int l, int Tq, const float* __restrict__ Q,
                           long long ldq, uint8_t* sm, uint64_t* mb, uint32_t* ph, int& pend) {
  const int D = a.D;
  const int cblocks = D / 128;
  const int n_items = cblocks * a.heads;
  const bf16* sw = reinterpret_cast<const bf16*>(sm);
  float* s_q = reinterpret_cast<float*>(sm + RF_HD * 128 * 2);
  const int tid = threadIdx.x & 127;  // column within the block
  const int half = threadIdx.x >> 7;  // two halves share the tiles
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int h = item / cblocks, cbk = item % cblocks;
    const int c = cbk * 128 + tid;
    if (!(pend & 1)) {
      __syncthreads();
      if (threadIdx.x < 32) fold_issue_w(a.Wk[l], D, item, sm, &mb[0]);
      pend |= 1;
    }
    if (!cta_wait(&mb[0], ph[0])) return false;
    ph[0] ^= 1;
    pend &= ~1;
    for (int t0 = 0; t0 < Tq; t0 += 64) {
      const int nt = min(64, Tq - t0);
      __syncthreads();
      for (int i = threadIdx.x; i < nt * RF_HD; i += RF_THREADS)
        s_q[i] = Q[(t0 + i / RF_HD) * ldq + h * RF_HD + i % RF_HD] * 0.125f;
      __syncthreads();
      for (int t = half; t < nt; t += 2) {
        float u = 0.f;
#pragma unroll 16
        for (int d = 0; d < RF_HD; ++d)
          u = fmaf(__bfloat162float(sw[d * 128 + tid]), s_q[t * RF_HD + d], u);
        const bf16 hi = __float2bfloat16_rn(u);
        const bf16 lo = __float2bfloat16_rn(u - __bfloat162float(hi));
        bf16* base = a.U2 + static_cast<size_t>(t0 + t) * 32 * D;
        base[static_cast<size_t>(h) * D + c] = hi;
        base[static_cast<size_t>(16 + h) * D + c] = lo;
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
  return true;
}

// ------------------------------------------------------------------ attention phase
// Scores, softmax and weighted sums of one pooling layer in one pass over x
// (the split-softmax form of single-query attention). Items (tile, chunk of
// AT_CHUNK tokens), a contiguous range per CTA; each item takes its tokens
// SC_TOK at a time, one TMA request per step ({64 channels, 32 tokens, D/64
// chunks}, 128-byte swizzle), double-buffered on mbarriers 2 and 3 across the
// CTA's steps (the first two requested before the grid barrier, x being an
// input; later ones once the scores of the step before them are summed, when
// every warp is done with the slot). Two CTA barriers per step. Per step:
//   1. s[t][j] = x_t . U2[j] for the 32 split rows: warp w multiplies its D/8
//      channels with m16n8k16 MMAs (its U2 fragments in registers for the
//      item), the 8 partial 32x32 tiles, stored column by column, are summed
//      in shared memory;
//      s_h = s[t][h] + s[t][16 + h] + c_h, tokens past valid_len -inf;
//   2. running max m_h and sum l_h, weights e = exp(s - m_h) as a bf16 hi/lo
//      pair;
//   3. Zc[h][c] = Zc[h][c] exp(m_old - m_new) + sum_t e_t x_t[c] (warp w owns
//      channels [w D/8, (w+1) D/8), hi and lo weights into the same fp32
//      accumulators in registers).
// Each item writes its unnormalised Zc to Zp[tile][chunk] and m, l to stats;
// the combine phase merges a tile's chunks. U2 and c are read with plain loads:
// they are written inside this kernel (the fold phase).
// Shared memory: 8 partial score tiles | hi/lo weights | x slots 0 and 1
// (D/64 * 4 KB each, above the fold phase's region since they are filled
// before the barrier that ends it for every CTA).
constexpr int AT_CHUNK = 128;                 // tokens per item
constexpr int AT_NCH = RF_TOK / AT_CHUNK;     // items (partials) per tile
constexpr int AT_RED_PITCH = 36;  // floats per column of a partial score tile
constexpr int AT_P_PITCH = 40;
constexpr int AT_RED_BYTES = RF_WARPS * 32 * AT_RED_PITCH * 4;
constexpr int AT_SLOT0 = ((AT_RED_BYTES + 2 * 16 * AT_P_PITCH * 2 + 1023) / 1024) * 1024;
constexpr int FOLD_SMEM = RF_HD * 128 * 2 + 64 * RF_HD * 4;  // Wk block + Q block
static_assert(AT_SLOT0 >= FOLD_SMEM, "x slots must not overlap the fold phase's staging");

__device__ __forceinline__ void attend_range(const RouterFusedArgs& a, int& i0, int& i1) {
  const int n_items = a.T * AT_NCH;
  i0 = static_cast<int>(static_cast<long long>(blockIdx.x) * n_items / gridDim.x);
  i1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * n_items / gridDim.x);
}

// Steps of an item holding at least one valid token (0: the chunk is padding).
__device__ __forceinline__ int attend_steps(const RouterFusedArgs& a, int item) {
  const int tile = item / AT_NCH, chunk = item % AT_NCH;
  int n = RF_TOK;
  if (a.valid_len) {
    n = a.valid_len[tile];
    n = n < 1 ? 1 : (n > RF_TOK ? RF_TOK : n);
  }
  return max(0, min(AT_CHUNK / SC_TOK, (n - chunk * AT_CHUNK + SC_TOK - 1) / SC_TOK));
}

// Cursor over this CTA's (item, step) sequence, past items without steps.
struct StepCursor {
  int item, st, end;
  __device__ void settle(const RouterFusedArgs& a) {
    while (item < end && st >= attend_steps(a, item)) {
      ++item;
      st = 0;
    }
  }
  __device__ bool valid() const { return item < end; }
  __device__ void next(const RouterFusedArgs& a) {
    ++st;
    settle(a);
  }
};

__device__ __forceinline__ StepCursor attend_first(const RouterFusedArgs& a) {
  StepCursor c;
  attend_range(a, c.item, c.end);
  c.st = 0;
  c.settle(a);
  return c;
}

// Lane 0: x of the cursor's step into slot `slot` (mbarrier 2 + slot).
__device__ __forceinline__ void attend_issue_x(const RouterFusedArgs& a, const StepCursor& c,
                                               int slot, uint8_t* sm, uint64_t* mb) {
  const int slot_bytes = a.D * 64;
  mbar_arrive_expect_tx(&mb[2 + slot], slot_bytes);
  const int tile = c.item / AT_NCH, chunk = c.item % AT_NCH;
  tma_load_3d(sm + AT_SLOT0 + slot * slot_bytes, &a.xmap3, &mb[2 + slot], 0,
              tile * RF_TOK + chunk * AT_CHUNK + c.st * SC_TOK, 0);
}

// Before the grid barrier: this CTA's first two steps. Returns the slots now
// in flight (bit s = slot s).
__device__ __forceinline__ int attend_prefetch_x(const RouterFusedArgs& a, uint8_t* sm,
                                                 uint64_t* mb) {
  __syncthreads();
  StepCursor c = attend_first(a);
  int pending = 0;
  for (int s = 0; s < 2 && c.valid(); ++s, c.next(a)) {
    if (threadIdx.x == 0) attend_issue_x(a, c, s, sm, mb);
    pending |= 1 << s;
  }
  return pending;
}

// KS = D / 128 (the phase is instantiated per width; see attend_phase).
template <int KS>
__device__ __noinline__ bool attend_phase_ks(const RouterFusedArgs& a, bool shared_q, uint8_t* sm,
                                uint64_t* mb, uint32_t* ph, int& x_pending, float* s_m,
                                float* s_l, float* s_scale) {
  constexpr int D = 128 * KS, NT = 2 * KS;
  constexpr int slot_bytes = D * 64;
  constexpr int CHUNK_BYTES = SC_TOK * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t2 = (lane & 3) * 2;
  float* red = reinterpret_cast<float*>(sm);
  bf16* sp = reinterpret_cast<bf16*>(sm + AT_RED_BYTES);  // [hi, lo][16][AT_P_PITCH]
  const int sh = threadIdx.x >> 4, stl = threadIdx.x & 15;  // softmax: head, token pair
  int i0, i1;
  attend_range(a, i0, i1);
  // the issue cursor runs two steps ahead of the consumed ones
  StepCursor ic = attend_first(a);
  for (int s = 0; s < 2 && ic.valid(); ++s) ic.next(a);
  int k = 0;  // steps consumed: slot k & 1
  for (int item = i0; item < i1; ++item) {
    const int tile = item / AT_NCH, chunk = item % AT_NCH;
    const size_t row0 = static_cast<size_t>(item) * 16;
    int n = RF_TOK;
    if (a.valid_len) {
      n = a.valid_len[tile];
      if (n < 1 || n > RF_TOK) {
        if (threadIdx.x == 0 && chunk == 0) atomicOr(a.status, DEV_BAD_VALID_LEN);
        n = n < 1 ? 1 : RF_TOK;
      }
    }
    const int ns = attend_steps(a, item);
    if (ns == 0) {  // every token of the chunk is padding
      if (threadIdx.x < 16) {
        a.stats[row0 + threadIdx.x] = -INFINITY;
        a.stats[static_cast<size_t>(a.T) * AT_NCH * 16 + row0 + threadIdx.x] = 0.f;
      }
      continue;
    }
    // B fragments of the scores (B[k = channel][n = split row] = U2[n][k])
    const bf16* u = a.U2 + (shared_q ? 0 : static_cast<size_t>(tile) * 32 * D);
    uint32_t ub[KS][4][2];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int kk = (warp * KS + ks) * 16 + t2;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int r = nt * 8 + g;
        const bool live = (r & 15) < a.heads;
        const bf16* ur = u + static_cast<size_t>(r) * D + kk;
        ub[ks][nt][0] = live ? *reinterpret_cast<const unsigned*>(ur) : 0u;
        ub[ks][nt][1] = live ? *reinterpret_cast<const unsigned*>(ur + 8) : 0u;
      }
    }
    const float c_h = sh < a.heads ? a.cb[(shared_q ? 0 : tile) * 16 + sh] : 0.f;
    if (threadIdx.x < 16) {
      s_m[threadIdx.x] = -INFINITY;
      s_l[threadIdx.x] = 0.f;
    }
    float accz[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) accz[nt][i] = 0.f;
    for (int st = 0; st < ns; ++st, ++k) {
      const int slot = k & 1;
      const uint8_t* sx = sm + AT_SLOT0 + slot * slot_bytes;
      // the give-up is decided for the whole CTA at the barrier after the scores
      const bool got = mbar_wait(&mb[2 + slot], ph[2 + slot]);
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
          ldsm_x4(af, sx + c * CHUNK_BYTES + ra * 128 + ((ja ^ (ra & 7)) << 4));
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const uint32_t bfr[2] = {ub[ks][nt][0], ub[ks][nt][1]};
            mma_bf16_16816(accs[mt][nt], af, bfr);
          }
        }
      }
      float* rw = red + warp * 32 * AT_RED_PITCH;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const int r = mt * 16 + g, j = nt * 8 + t2;
          rw[j * AT_RED_PITCH + r] = accs[mt][nt][0];
          rw[(j + 1) * AT_RED_PITCH + r] = accs[mt][nt][1];
          rw[j * AT_RED_PITCH + r + 8] = accs[mt][nt][2];
          rw[(j + 1) * AT_RED_PITCH + r + 8] = accs[mt][nt][3];
        }
      // a copy that never landed leaves its bit set (drained at exit)
      if (__syncthreads_and(got ? 1 : 0) == 0) return false;
      ph[2 + slot] ^= 1;
      x_pending &= ~(1 << slot);
      // every warp has finished the previous step's weighted sums: its slot
      // takes the step after this one
      if (k >= 1 && ic.valid()) {
        if (threadIdx.x == 0) attend_issue_x(a, ic, slot ^ 1, sm, mb);
        x_pending |= 1 << (slot ^ 1);
        ic.next(a);
      }
      // 2. running softmax of head sh over tokens 2 stl and 2 stl + 1
      {
        const int tb = chunk * AT_CHUNK + st * SC_TOK;
        // column sh of the hi part and 16 + sh of the lo part, token-contiguous
        float sv[2] = {c_h, c_h};
#pragma unroll
        for (int w = 0; w < RF_WARPS; ++w) {
          const float* rc = red + w * 32 * AT_RED_PITCH;
          const float2 hi = *reinterpret_cast<const float2*>(rc + sh * AT_RED_PITCH + 2 * stl);
          const float2 lo =
              *reinterpret_cast<const float2*>(rc + (16 + sh) * AT_RED_PITCH + 2 * stl);
          sv[0] += hi.x + lo.x;
          sv[1] += hi.y + lo.y;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (!(sh < a.heads && tb + 2 * stl + i < n)) sv[i] = -INFINITY;
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
          sp[sh * AT_P_PITCH + 2 * stl + i] = hi;
          sp[(16 + sh) * AT_P_PITCH + 2 * stl + i] =
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
        for (int kk = 0; kk < SC_TOK / 16; ++kk) {
          uint32_t ah[4], al[4];
          const int pr = lane & 15, pk = kk * 16 + 8 * (lane >> 4);
          ldsm_x4(ah, sp + pr * AT_P_PITCH + pk);
          ldsm_x4(al, sp + (16 + pr) * AT_P_PITCH + pk);
          const int r = kk * 16 + (lane & 15);
#pragma unroll
          for (int nt = 0; nt < NT; nt += 2) {
            const int cw = warp * (D / 8) + 8 * (nt + (lane >> 4));
            const int c = cw >> 6, j = (cw & 63) >> 3;
            uint32_t bf[4];
            ldsm_x4_trans(bf, sx + c * CHUNK_BYTES + r * 128 + ((j ^ (r & 7)) << 4));
            const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
            mma_bf16_16816(accz[nt], ah, b0);
            mma_bf16_16816(accz[nt], al, b0);
            mma_bf16_16816(accz[nt + 1], ah, b1);
            mma_bf16_16816(accz[nt + 1], al, b1);
          }
        }
      }
      // no barrier here: the weights and s_scale are rewritten only after the
      // next step's first barrier, and the score partials were read before the last
    }
    float* zp = a.Zp + row0 * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = warp * (D / 8) + nt * 8 + t2;
      *reinterpret_cast<float2*>(zp + static_cast<size_t>(g) * D + c) =
          make_float2(accz[nt][0], accz[nt][1]);
      *reinterpret_cast<float2*>(zp + static_cast<size_t>(g + 8) * D + c) =
          make_float2(accz[nt][2], accz[nt][3]);
    }
    if (threadIdx.x < 16) {  // s_m / s_l were last written before the final barrier
      a.stats[row0 + threadIdx.x] = s_m[threadIdx.x];
      a.stats[static_cast<size_t>(a.T) * AT_NCH * 16 + row0 + threadIdx.x] = s_l[threadIdx.x];
    }
    __syncthreads();  // stats read before the next item resets them
  }
  return true;
}

__device__ bool attend_phase(const RouterFusedArgs& a, bool shared_q, uint8_t* sm, uint64_t* mb,
                             uint32_t* ph, int& x_pending) {
  __shared__ float s_m[16], s_l[16], s_scale[16];
  switch (a.D / 128) {
    case 1: return attend_phase_ks<1>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    case 2: return attend_phase_ks<2>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    case 3: return attend_phase_ks<3>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    case 4: return attend_phase_ks<4>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    case 5: return attend_phase_ks<5>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    case 6: return attend_phase_ks<6>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    case 7: return attend_phase_ks<7>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
    default: return attend_phase_ks<8>(a, shared_q, sm, mb, ph, x_pending, s_m, s_l, s_scale);
  }
}

// ------------------------------------------------------------------ combine phase
// Items (tile, head): z[tile][h] = sum_c exp(m_c - M) Zc / sum_c exp(m_c - M) l_c
// over the tile's AT_NCH chunks (chunks without a valid token, l = 0, skipped).
__device__ void combine_phase(const RouterFusedArgs& a) {
  const int D = a.D;
  const size_t lofs = static_cast<size_t>(a.T) * AT_NCH * 16;
  const int n_items = a.T * a.heads;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int tile = item / a.heads, h = item % a.heads;
    const size_t r0 = static_cast<size_t>(tile) * AT_NCH * 16 + h;
    float w[AT_NCH];
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < AT_NCH; ++c) {
      w[c] = a.stats[lofs + r0 + 16 * c] > 0.f ? a.stats[r0 + 16 * c] : -INFINITY;
      M = fmaxf(M, w[c]);
    }
    float L = 0.f;
#pragma unroll
    for (int c = 0; c < AT_NCH; ++c) {
      w[c] = w[c] == -INFINITY ? 0.f : expf(w[c] - M);
      L += w[c] * a.stats[lofs + r0 + 16 * c];
    }
    const float inv = 1.0f / L;
    for (int c4 = threadIdx.x * 4; c4 < D; c4 += RF_THREADS * 4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < AT_NCH; ++c) {
        if (w[c] == 0.f) continue;
        const float4 v = *reinterpret_cast<const float4*>(a.Zp + (r0 + 16 * c) * D + c4);
        acc.x = fmaf(w[c], v.x, acc.x);
        acc.y = fmaf(w[c], v.y, acc.y);
        acc.z = fmaf(w[c], v.z, acc.z);
        acc.w = fmaf(w[c], v.w, acc.w);
      }
      *reinterpret_cast<float4*>(a.z + (static_cast<size_t>(tile) * 16 + h) * D + c4) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
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
    int my_nan = 0;
    for (int i = threadIdx.x; i < n; i += RF_THREADS) {
      const double v = static_cast<double>(a.gate[2 * (s + i)]);
      s_vals[i] = v;
      my_nan |= isnan(v) ? 1 : 0;
    }
    // a NaN gate makes the group's quantile NaN (as torch.quantile does), so
    // no tile of the group passes the strict > test; the rank sort, whose
    // ranks assume a total order, is skipped
    const int any_nan = __syncthreads_or(my_nan);
    if (!any_nan) {
      for (int i = threadIdx.x; i < n; i += RF_THREADS) {
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
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled TMA boxes (the launch adds the slack)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* sf = reinterpret_cast<float*>(sm);
  // mbarriers: 0 weights (projections, fold), 1 the projections' input rows,
  // 2 and 3 the two x slots of the attention phase
  __shared__ __align__(8) uint64_t s_mb[4];
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&s_mb[i], 1);
    fence_mbar_init();
    tma_prefetch_desc(&a.xmap3);
  }
  __syncthreads();
  uint32_t ph[4] = {0u, 0u, 0u, 0u};
  unsigned gen = 0;
  bool ok = true;
  // bulk copies in flight on mbarriers 0 (weights) and 1 (projection input
  // rows), bits 0 and 1: set when issued, cleared when their wait succeeds
  int mb_pending = 0;
  int x_pending = 0;       // x slots (bits) requested ahead of their phase
  const int T = a.T, D = a.D, G = a.G;
  long long wait_limit = IVC_WAIT_CYCLES;
  auto sync = [&]() {
    if (ok) ok = grid_sync(a.bar, gen, wait_limit);
    return ok;
  };
  // The weights of the next projection phase do not depend on the previous
  // phase: this CTA's first item's rows are requested before the barrier.
  auto prefetch_w = [&](const bf16* W, int K, int N) {
    __syncthreads();
    if (static_cast<int>(blockIdx.x) < N / GV_COLS) {
      if (warp == 0) gv_issue_w(W, K, blockIdx.x, sm, &s_mb[0]);
      mb_pending |= 1;
    }
  };
  // a phase that does not run (an earlier wait gave up) leaves its
  // prefetched copies to the drain at the end of the kernel
  auto project = [&](int M, int K, int N, const bf16* W, const bf16* b, float* Y, int ldy,
                     bool act, auto row) {
    if (ok) ok = gemv_phase(M, K, N, W, b, Y, ldy, act, sm, s_mb, ph, mb_pending, row);
  };
  // layer 1's query is shared by all tiles: Q1 = Wq_1 query + bq_1 in row 0 of Q
  // (the bf16 query is widened into h first)
  if (blockIdx.x == 0)
    for (int k = threadIdx.x; k < D; k += RF_THREADS) a.h[k] = __bfloat162float(a.query[k]);
  prefetch_w(a.Wq[0], D, D);
  if (sync()) project(1, D, D, a.Wq[0], a.bq[0], a.Q, D, false, [&](int, int) { return a.h; });
  for (int l = 0; l < 4 && ok; ++l) {
    // this CTA's first fold item: its Wk block is requested before the barrier
    __syncthreads();
    if (static_cast<int>(blockIdx.x) < (D / 128) * a.heads) {
      if (warp == 0) fold_issue_w(a.Wk[l], D, blockIdx.x, sm, &s_mb[0]);
      mb_pending |= 1;
    }
    if (!sync()) break;
    const bool shared_q = l == 0;
    if (!fold_phase(a, l, shared_q ? 1 : T, a.Q, shared_q ? 0 : D, sm, s_mb, ph, mb_pending))
      ok = false;
    // the attention phase's first x steps (x is an input) before the barrier
    x_pending = attend_prefetch_x(a, sm, s_mb);
    if (!sync()) break;
    if (!attend_phase(a, shared_q, sm, s_mb, ph, x_pending)) ok = false;
    if (!sync()) break;
    combine_phase(a);
    // o = Wv_h z_h + bv: the input row of output row m for columns of head h is z[m][h]
    prefetch_w(a.Wv[l], D, D);
    if (!sync()) break;
    project(T, D, D, a.Wv[l], a.bv[l], a.O, D, false, [&](int m, int c0) {
      return a.z + (static_cast<size_t>(m) * 16 + c0 / RF_HD) * D;
    });
    prefetch_w(a.Wo[l], D, D);
    if (!sync()) break;
    project(T, D, D, a.Wo[l], a.bo[l], a.q, D, false,
            [&](int m, int) { return a.O + static_cast<size_t>(m) * D; });
    if (l < 3) {
      prefetch_w(a.Wq[l + 1], D, D);
      if (!sync()) break;
      project(T, D, D, a.Wq[l + 1], a.bq[l + 1], a.Q, D, false,
              [&](int m, int) { return a.q + static_cast<size_t>(m) * D; });
    }
  }
  // Gating: h_0 = pooled = q; block b: u1 = GELU(W1 h_b + b1), u2 = W2 u1 + b2,
  // then the residual LayerNorm (rows spread over the CTAs, kept in h).
  for (int b = 0; b < 4 && ok; ++b) {
    const float* hb = b == 0 ? a.q : a.h;
    prefetch_w(a.gW1[b], D, G);
    if (!sync()) break;
    project(T, D, G, a.gW1[b], a.gb1[b], a.u1, G, true,
            [&](int m, int) { return hb + static_cast<size_t>(m) * D; });
    prefetch_w(a.gW2[b], G, D);
    if (!sync()) break;
    project(T, G, D, a.gW2[b], a.gb2[b], a.u2, D, false,
            [&](int m, int) { return a.u1 + static_cast<size_t>(m) * G; });
    if (!sync()) break;
    for (int m = blockIdx.x; m < T; m += gridDim.x) {
      residual_ln_row(hb + static_cast<size_t>(m) * D, a.u2 + static_cast<size_t>(m) * D,
                      a.gln_g[b], a.gln_b[b], sf, D, a.gate_inside);
      __syncthreads();
      for (int i = threadIdx.x; i < D; i += RF_THREADS) a.h[static_cast<size_t>(m) * D + i] = sf[i];
      __syncthreads();
    }
  }
  // head: gate = softmax(Wout h_4 + bout), one warp per tile. From here on no
  // bulk copy is in flight (the last projection's waits succeeded, the
  // attention slots were consumed), so a short test limit may apply.
  if (a.late_wait_cycles > 0) wait_limit = a.late_wait_cycles;
  if (ok && sync()) {
    const int lane = threadIdx.x & 31;
    for (int t = blockIdx.x * RF_WARPS + warp; t < T; t += gridDim.x * RF_WARPS) {
      const float* hr = a.h + static_cast<size_t>(t) * D;
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
    route_phase(a, reinterpret_cast<double*>(sm),
                reinterpret_cast<double*>(sm) + IVC_MAX_QUANTILE_GROUP);
  // copies whose wait never succeeded (a prefetch whose phase never ran, or a
  // phase that gave up with copies in flight): let them land before exit
  if (mb_pending & 1) (void)mbar_wait(&s_mb[0], ph[0]);
  if (mb_pending & 2) (void)mbar_wait(&s_mb[1], ph[1]);
  for (int sl = 0; sl < 2; ++sl)
    if (x_pending & (1 << sl)) (void)mbar_wait(&s_mb[2 + sl], ph[2 + sl]);
  if (!ok && threadIdx.x == 0) atomicOr(a.status, DEV_WAIT_TIMEOUT);
}

size_t router_fused_smem(int D, int G) {
  const size_t K = static_cast<size_t>(D > G ? D : G);
  const size_t gemv = GV_ROWS * (K + 8) * 4 + GV_COLS * (K + 8) * 2 +
                      static_cast<size_t>(RF_WARPS) * GV_ROWS * GV_COLS * 4;
  const size_t route = 2 * static_cast<size_t>(IVC_MAX_QUANTILE_GROUP) * sizeof(double);
  const size_t attend = AT_SLOT0 + 2 * static_cast<size_t>(D) * 64;  // partials, weights, 2 x slots
  const size_t fold = FOLD_SMEM;
  size_t m = gemv;
  for (size_t v : {route, attend, fold, static_cast<size_t>(D) * sizeof(float)})
    if (v > m) m = v;
  return m + 1024;  // alignment slack
}

}  // namespace

// Test limit of the persistent router's late grid barriers (ivc.h,
// ivc_set_router_wait_limit); read at every launch.
static std::atomic<long long> g_late_wait_cycles{0};

long long router_late_wait_cycles() { return g_late_wait_cycles.load(std::memory_order_relaxed); }

void set_router_late_wait_cycles(long long cycles) {
  g_late_wait_cycles.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed);
}

bool router_fused_wanted(bool default_on) {
  static int env = -2;
  if (env == -2) {
    const char* e = std::getenv("IVC_ROUTER_FUSED");
    env = e ? (e[0] == '1' ? 1 : 0) : -1;
  }
  return env < 0 ? default_on : env == 1;
}

bool router_fused_supported(const ivc_router* r) {
  return r->pool_mode == IVC_POOL_FOLDED && r->D % 128 == 0 && r->D <= RF_MAXD &&
         r->heads <= 16 && r->gate_hidden <= RF_MAXK && r->gate_hidden % 128 == 0 &&
         router_fused_smem(r->D, r->gate_hidden) <= 227 * 1024;
}

int launch_router_fused(const ivc_router* r, const void* x, const int32_t* valid_len, int T,
                        const int32_t* image_offsets, int I, float* gate, uint8_t* mask,
                        int32_t* offsets, int32_t* total, const FusedRouterBufs& b,
                        const Launch& L) {
  if (T == 0) return IVC_OK;
  if (!router_fused_supported(r)) return IVC_EUNSUPPORTED;
  RouterFusedArgs a{};
  {
    const unsigned long long D2 = static_cast<unsigned long long>(r->D) * 2;  // row bytes
    const unsigned long long chunks = static_cast<unsigned long long>(r->D) / 64;
    // x: {64 ch, tokens, chunks}, rows of D2 bytes, chunks 128 bytes apart
    const unsigned long long xd[3] = {64, static_cast<unsigned long long>(T) * RF_TOK, chunks};
    const unsigned long long xs[2] = {D2, 128};
    const unsigned xb[3] = {64, SC_TOK, static_cast<unsigned>(chunks)};
    if (map_bf16(&a.xmap3, 3, x, xd, xs, xb) != IVC_OK) return IVC_ECUDA;
  }
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
  a.Zp = b.Zp;
  a.stats = b.stats;
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
  a.late_wait_cycles = router_late_wait_cycles();
  const size_t smem = router_fused_smem(r->D, r->gate_hidden);
  if (smem > 227 * 1024) return IVC_EUNSUPPORTED;
  if (smem_optin(reinterpret_cast<const void*>(router_fused_kernel), smem) != IVC_OK)
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
