// ivc_attend_tc.cu — one folded pooling layer's attention on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM).
//
// InternVL3_5-4B-Flash "Gating and CrossAttentionPooling" article, section 2:
// per layer the learnable query attends, with 16 heads and a padding mask,
// over all tokens of the tile. In the folded form (ivc_router.cu) the key
// projection is folded into the query, so per tile and head the scores are
// s_t = x_t . u_h + c_h over the raw features x, and the weighted sum is
// z_h = sum_t softmax(s)_t x_t (the value projection follows on z_h).
//
// Per (tile, chunk of 128 tokens), like the mma.sync form it replaces, with
// the same outputs: the chunk's unnormalised sums
// Zc_h = sum_t exp(s_t - m_h) x_t, its max m_h and sum l_h (pool_combine
// merges a tile's 8 chunks). Per chunk:
//   scores   S[128 tokens x 32] = X[128 x D] . U2[32 x D]^T   (M 128, N 32;
//            U2 rows 0..15 the bf16 hi parts of u_h, 16..31 the lo parts),
//            x streamed as 32 KB boxes {64 channels, 128 tokens, 2 chunks};
//   softmax  four warps read S from TMEM (thread = token), s_h = S[h] +
//            S[16+h] + c_h, padding tokens -inf, exact max and sum over the
//            chunk, e = exp(s - m) written to shared memory as a bf16 pair
//            hi / lo (rows h and 16+h of P [32 x 128 tokens], K-major,
//            128-byte swizzle);
//   sums     Z^T[128 channels x 32] = X^T[channels x tokens] . P^T per
//            128-channel block (M 128, N 32, K 128 tokens), the x boxes
//            streamed a second time (L2-resident) and read as an MN-major A
//            operand; z_h = Z^T[:, h] + Z^T[:, 16+h].
// TMEM holds S (32 columns) and the D/128 Z^T blocks (32 columns each).
// Warp 0 issues the TMA loads, warp 1 allocates TMEM and issues the MMAs from
// one thread, warps 2..5 do the softmax and the epilogue (warp w reads TMEM
// lanes 32 (w % 4) .. + 31). Every wait is bounded; a wait that runs out sets
// IVC_DEV_WAIT_TIMEOUT and the CTA skips its remaining work. A chunk with no
// valid token loads nothing and leaves l = 0 (the merge skips it).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>

#include "ivc_internal.h"
#include "ivc_ptx.cuh"

namespace ivc {
namespace {

constexpr int AT_THREADS = 192;
constexpr int AT_TOK = 128;     // tokens per chunk (one CTA)
constexpr int AT_NCH = 1024 / AT_TOK;
constexpr int AT_STAGES = 4;    // x boxes in flight
constexpr uint32_t AT_HALF = AT_TOK * 128;   // one 64-channel chunk of a box: 16 KB
constexpr uint32_t AT_BOX = 2 * AT_HALF;     // 32 KB
constexpr uint32_t AT_P = 2 * 32 * 128;      // P: two 64-token halves x 32 rows x 128 B
constexpr int AT_EPI_BAR = 1;   // named barrier of the four softmax / epilogue warps

__device__ __forceinline__ void at_epi_sync() {
  asm volatile("bar.sync %0, 128;" ::"n"(AT_EPI_BAR) : "memory");
}
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int NB>  // NB = D / 128
struct AtSmem {
  static constexpr int D = 128 * NB;
  static constexpr uint32_t RING = AT_STAGES * AT_BOX;
  static constexpr uint32_t U2 = static_cast<uint32_t>(D) * 64;  // 32 rows x D bf16
  static constexpr uint32_t TOTAL = 1024 + RING + U2 + AT_P;
};

// Items are (tile, chunk) pairs, item = tile * 8 + chunk; CTA b takes items
// b, b + gridDim.x, ... (a grid as wide as the SMs the kernel may use), so
// that one item's loads and score MMAs overlap the previous item's weighted
// sums and epilogue. Barriers between the roles, for the k-th item with a
// valid token (phase k & 1): ufull / uempty (the U2 buffer: loaded /
// no longer read by the score MMAs), sfull / sfree (S in TMEM: complete /
// read by the softmax), pfull (P written), zfull / zfree (Z^T in TMEM:
// complete / drained).
struct AtItem {
  int tile, chunk, nvalid;
};

// `status` is non-null in one thread only: the one that reports a length
// outside [1, 1024].
__device__ __forceinline__ AtItem at_item(int item, const int32_t* valid_len, int* status) {
  AtItem r;
  r.tile = item / AT_NCH;
  r.chunk = item % AT_NCH;
  int n = 1024;
  if (valid_len != nullptr) {
    n = valid_len[r.tile];
    if (n < 1 || n > 1024) {
      if (r.chunk == 0 && status != nullptr) atomicOr(status, DEV_BAD_VALID_LEN);
      n = n < 1 ? 1 : 1024;
    }
  }
  r.nvalid = min(AT_TOK, max(0, n - r.chunk * AT_TOK));
  return r;
}

template <int NB>
__global__ void __launch_bounds__(AT_THREADS, 1)
    pool_attend_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                          const __grid_constant__ CUtensorMap umap, int u2_per_tile,
                          const float* __restrict__ cb, int cb_stride,
                          const int32_t* __restrict__ valid_len, int heads, int n_items,
                          float* __restrict__ Zp, float* __restrict__ mstat,
                          float* __restrict__ lstat, int* __restrict__ status) {
  using S = AtSmem<NB>;
  constexpr int D = S::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = sm;
  uint8_t* su2 = sm + S::RING;
  uint8_t* sp = su2 + S::U2;
  __shared__ __align__(8) uint64_t full[AT_STAGES], empty[AT_STAGES];
  __shared__ __align__(8) uint64_t ufull, uempty, sfull, sfree, pfull, zfull, zfree;
  __shared__ uint32_t s_tmem;
  __shared__ float red[2][4][16];  // per-warp max, then sum, of each head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&ufull, 1);
    mbar_init(&uempty, 1);
    mbar_init(&sfull, 1);
    mbar_init(&sfree, 128);
    mbar_init(&pfull, 128);
    mbar_init(&zfull, 1);
    mbar_init(&zfree, 128);
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&umap);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  bool ok = true;
  // the next kernel (the chunk merge) may launch; it waits for this grid
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // x is an input: the first item's first boxes go out before waiting for
      // the previous kernel, which writes U2 (the folded query)
      int g = 0, k = 0;
      bool waited = false;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const AtItem a = at_item(item, valid_len, nullptr);
        if (a.nvalid == 0) continue;
        const int xrow = a.tile * 1024 + a.chunk * AT_TOK;
        if (waited) {  // the U2 buffer is free once the previous item's score MMAs are done
          if (!mbar_wait(&uempty, (k & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&ufull, S::U2);
          tma_load_3d(su2, &umap, &ufull, 0, u2_per_tile ? a.tile * 32 : 0, 0);
        }
        for (int it = 0; it < 2 * NB; ++it, ++g) {
          const int s = g % AT_STAGES;
          if (!mbar_wait(&empty[s], ((g / AT_STAGES) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], AT_BOX);
          tma_load_3d(ring + s * AT_BOX, &xmap, &full[s], 0, xrow, 2 * (it % NB));
          if (!waited && it == (2 * NB < AT_STAGES ? 2 * NB : AT_STAGES) - 1) {
            pdl_wait();
            waited = true;
            mbar_arrive_expect_tx(&ufull, S::U2);
            tma_load_3d(su2, &umap, &ufull, 0, u2_per_tile ? a.tile * 32 : 0, 0);
          }
        }
        ++k;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc_s = idesc_bf16_f32(AT_TOK, 32);              // A, B K-major
      const uint32_t idesc_z = idesc_bf16_f32(128, 32) | (1u << 15);   // A MN-major
      const uint32_t pa = smem_u32(sp);
      int g = 0, k = 0;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const AtItem a = at_item(item, valid_len, nullptr);
        if (a.nvalid == 0) continue;
        const uint32_t ph = k & 1;
        // scores: S += X_box(chunk j) . U2(chunk 2b + j)^T, once U2 is loaded
        // and the softmax has read the previous item's S
        if (!mbar_wait(&ufull, ph) || !mbar_wait(&sfree, ph ^ 1)) { ok = false; break; }
        tc_fence_after();
        for (int b = 0; b < NB && ok; ++b, ++g) {
          const int s = g % AT_STAGES;
          if (!mbar_wait(&full[s], (g / AT_STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xa = smem_u32(ring + s * AT_BOX);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint64_t ad = sw128_kmajor_desc(xa + j * AT_HALF);
            const uint64_t bd = sw128_kmajor_desc(smem_u32(su2) + (2 * b + j) * 4096);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc_s, (b | j | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&sfull);
        umma_commit(&uempty);
        // weighted sums once the softmax weights are in shared memory and the
        // epilogue has drained the previous item's sums
        if (!mbar_wait(&pfull, ph) || !mbar_wait(&zfree, ph ^ 1)) { ok = false; break; }
        tc_fence_after();
        for (int b = 0; b < NB && ok; ++b, ++g) {
          const int s = g % AT_STAGES;
          if (!mbar_wait(&full[s], (g / AT_STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          // A = this box read MN-major: 64-channel atoms 16 KB apart, 8-token
          // groups 1024 B apart; 16 tokens per MMA = 2048 B
          const uint64_t ad = sw128_mnmajor_desc(smem_u32(ring + s * AT_BOX), AT_HALF);
#pragma unroll
          for (int kk = 0; kk < AT_TOK / 16; ++kk) {
            const uint64_t bd = sw128_kmajor_desc(pa + (kk >> 2) * 4096) + 2 * (kk & 3);
            umma_bf16(tmem + 32 + 32 * b, ad + ((2048 * kk) >> 4), bd, idesc_z,
                      kk != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&zfull);
        ++k;
      }
    }
  } else {
    // -------------------------------------------------------- softmax, epilogue
    const int quad = warp & 3;
    const int t = quad * 32 + lane;  // token of the chunk = TMEM lane
    pdl_wait();                      // cb is written by the previous kernel
    int k = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const AtItem a = at_item(item, valid_len, (warp == 2 && lane == 0) ? status : nullptr);
      const size_t row0 = (static_cast<size_t>(a.tile) * AT_NCH + a.chunk) * 16;
      if (a.nvalid == 0) {  // every token of the chunk is padding: l = 0
        if (quad == 0 && lane < 16) {
          mstat[row0 + lane] = -INFINITY;
          lstat[row0 + lane] = 0.f;
        }
        continue;
      }
      const uint32_t ph = k & 1;
      ++k;
      const bool valid = t < a.nvalid;
      float c_h[16];
#pragma unroll
      for (int h = 0; h < 16; ++h)
        c_h[h] = h < heads ? cb[static_cast<size_t>(a.tile) * cb_stride + h] : 0.f;
      // after a wait that ran out the warps keep their named barriers in step
      // (two per item) but do no more work
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sfull, ph));
      if (!ok) {
        at_epi_sync();
        at_epi_sync();
        continue;
      }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16), r);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&sfree);  // S is read: the next item's scores may overwrite it
      float sh[16], e[16], M[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        sh[h] = (valid && h < heads)
                    ? __uint_as_float(r[h]) + __uint_as_float(r[16 + h]) + c_h[h]
                    : -INFINITY;
        float v = sh[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0][quad][h] = v;
      }
      at_epi_sync();
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        M[h] = fmaxf(fmaxf(red[0][0][h], red[0][1][h]), fmaxf(red[0][2][h], red[0][3][h]));
        // token 0 of the chunk is valid, so M is finite for every live head
        e[h] = (valid && h < heads) ? expf(sh[h] - M[h]) : 0.f;
        float v = e[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[1][quad][h] = v;
      }
      // P [32 rows x 128 tokens] bf16, K-major, 128-byte swizzle: row j of
      // token half a at a * 4096 + j * 128, 16-byte unit (t % 64) / 8 XOR j % 8
      // (the previous item's weighted sums, which read P, are complete: its
      // Z^T was drained below before this item's softmax)
      const int ah = t >> 6, tt = t & 63;
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const bf16 hi = __float2bfloat16_rn(e[h]);
        const bf16 lo = __float2bfloat16_rn(e[h] - __bfloat162float(hi));
        const int j0 = h, j1 = 16 + h;
        *reinterpret_cast<bf16*>(sp + ah * 4096 + j0 * 128 + (((tt >> 3) ^ (j0 & 7)) << 4) +
                                 (tt & 7) * 2) = hi;
        *reinterpret_cast<bf16*>(sp + ah * 4096 + j1 * 128 + (((tt >> 3) ^ (j1 & 7)) << 4) +
                                 (tt & 7) * 2) = lo;
      }
      fence_async_shared();
      mbar_arrive(&pfull);
      at_epi_sync();
      if (quad == 0 && lane < 16) {
        float mv = 0.f, lv = 0.f;
#pragma unroll
        for (int h = 0; h < 16; ++h)
          if (h == lane) {
            mv = M[h];
            lv = (red[1][0][h] + red[1][1][h]) + (red[1][2][h] + red[1][3][h]);
          }
        mstat[row0 + lane] = lane < heads ? mv : -INFINITY;
        lstat[row0 + lane] = lane < heads ? lv : 0.f;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&zfull, ph));
      if (!ok) continue;
      tc_fence_after();
#pragma unroll 1
      for (int b = 0; b < NB; ++b) {
        uint32_t z[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + 32 + 32 * b, z);
        tmem_ld_wait();
        const int c = b * 128 + quad * 32 + lane;  // channel = TMEM lane of block b
#pragma unroll
        for (int h = 0; h < 16; ++h)
          if (h < heads)
            Zp[(row0 + h) * D + c] = __uint_as_float(z[h]) + __uint_as_float(z[16 + h]);
      }
      tc_fence_before();
      mbar_arrive(&zfree);  // Z^T is drained: the next item's sums may overwrite it
    }
  }
  if (!ok && status != nullptr) atomicOr(status, DEV_WAIT_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int NB>
int launch_attend_tc_nb(const CUtensorMap& xmap, const CUtensorMap& umap, int u2_per_tile,
                        const float* cb, int cb_stride, const int32_t* valid_len, int T, int heads,
                        float* Zp, float* mstat, float* lstat, const Launch& L) {
  using S = AtSmem<NB>;
  if (smem_optin(reinterpret_cast<const void*>(pool_attend_tc_kernel<NB>), S::TOTAL) != IVC_OK)
    return IVC_ECUDA;
  const int items = T * AT_NCH;
  int grid = L.sm_budget > 0 ? L.sm_budget : num_sms();
  if (grid > items) grid = items;
  return launch_k(pool_attend_tc_kernel<NB>, dim3(grid), dim3(AT_THREADS), S::TOTAL, L.stream, 1,
                  xmap, umap, u2_per_tile, cb, cb_stride, valid_len, heads, items, Zp, mstat, lstat,
                  L.status);
}

}  // namespace

// The attention on tcgen05 unless IVC_ATTEND_TC=0 selects the mma.sync form
// (ivc_router.cu): measured 0.183 against 0.196 ms per ivc_vir_route on the
// 13-tile image, the same within noise inside the dual flow.
bool attend_tc_wanted() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("IVC_ATTEND_TC");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

int pool_attend_tc_chunks() { return AT_NCH; }

bool pool_attend_tc_supported(int D, int heads) {
  return D % 128 == 0 && D <= 1024 && heads >= 1 && heads <= 16 && heads * 64 == D;
}

int launch_pool_attend_tc(const void* x, const bf16* U2, int Tq, const float* cb,
                          const int32_t* valid_len, int T, int D, int heads, float* Zp,
                          float* stats, const Launch& L) {
  if (T == 0) return IVC_OK;
  if (D % 128 != 0 || D > 1024 || heads < 1 || heads > 16 || heads * 64 != D)
    return IVC_EUNSUPPORTED;
  CUtensorMap xmap, umap;
  {
    // x as {64 channels, T*1024 tokens, D/64 chunks}: rows of 2D bytes, chunks 128 B apart
    const unsigned long long d[3] = {64, static_cast<unsigned long long>(T) * 1024,
                                     static_cast<unsigned long long>(D) / 64};
    const unsigned long long st[2] = {static_cast<unsigned long long>(D) * 2, 128};
    const unsigned box[3] = {64, AT_TOK, 2};
    if (map_bf16(&xmap, 3, x, d, st, box) != IVC_OK) return IVC_ECUDA;
  }
  {
    // U2 as {64, Tq*32 rows, D/64 chunks}; one box = a tile's 32 rows
    const unsigned long long d[3] = {64, static_cast<unsigned long long>(Tq) * 32,
                                     static_cast<unsigned long long>(D) / 64};
    const unsigned long long st[2] = {static_cast<unsigned long long>(D) * 2, 128};
    const unsigned box[3] = {64, 32, static_cast<unsigned>(D / 64)};
    if (map_bf16(&umap, 3, U2, d, st, box) != IVC_OK) return IVC_ECUDA;
  }
  float* mstat = stats;
  float* lstat = stats + static_cast<size_t>(T) * AT_NCH * 16;
  const int u2_per_tile = Tq == 1 ? 0 : 1;
  const int cb_stride = Tq == 1 ? 0 : 16;
  TraceScope ts("pool.attend", L.stream);
  switch (D / 128) {
    case 1: return launch_attend_tc_nb<1>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    case 2: return launch_attend_tc_nb<2>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    case 3: return launch_attend_tc_nb<3>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    case 4: return launch_attend_tc_nb<4>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    case 5: return launch_attend_tc_nb<5>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    case 6: return launch_attend_tc_nb<6>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    case 7: return launch_attend_tc_nb<7>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
    default: return launch_attend_tc_nb<8>(xmap, umap, u2_per_tile, cb, cb_stride, valid_len, T, heads, Zp, mstat, lstat, L);
  }
}

}  // namespace ivc
