// ivc_gemm.cuh — the connector / projection GEMM for sm_100a.
//
//   out[m, n] = epilogue( sum_k A[m, k] * B[n, k] )      (B = nn.Linear weight [N, K])
//
// One CTA computes one 128 x BN output tile with the 5th-generation tensor
// cores: TMA streams 128 x 64 A tiles and BN x 64 B tiles (128-byte swizzle)
// through a STAGES-deep shared-memory ring, one thread issues
// tcgen05.mma (M=128, N=BN, K=16) into a TMEM accumulator, and four epilogue
// warps read the accumulator back with tcgen05.ld and apply the fused
// epilogue (LayerNorm fold or bias, then optional GELU) before storing bf16.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
//
// A-operand modes. pixel_shuffle ("Pixel Shuffle 源码逐行解析" of the
// InternVL3-14B-Instruct connector article; table "三档 Token 规模" of the
// InternVL3_5-2B-Flash article) is not materialised: the GEMM row of
// token (tile, a, b) and the column block of grid offset (di, dj) are
// addressed directly in the [T, 32, 32, C] feature tensor through a 5-D TMA
// tensor map, so every A tile is one TMA box:
//   PS_HALF    (factor 0.5):  dims {C, dj:2, b:16, di:2, tile*16+a}, box {64,1,16,1,8}
//   PS_QUARTER (factor 0.25): dims {C, r:4, b:8, q:4, tile*8+a},     box {64,1,8,1,16}
// Column m of the shuffled row is (block*C + c) with block = 2di+dj
// (4q+r for the quarter), so k-step kk loads block kk/(C/64), channels
// 64*(kk%(C/64)).. of each of the 128 tokens of the tile.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ivc_ptx.cuh"

namespace ivc {

enum AMode : int { A_PLAIN = 0, A_PS_HALF = 1, A_PS_QUARTER = 2, A_PS_QUARTER_TWICE = 3 };
enum EpiMode : int { EPI_BIAS = 0, EPI_LNFOLD = 1 };

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_MAX_GROUPS = 8;
constexpr int GEMM_THREADS = 192;

struct alignas(64) GemmMaps {
  CUtensorMap a;
  CUtensorMap b[GEMM_MAX_GROUPS];
};

struct GemmArgs {
  int M, N, K;
  int a_mode;
  int c_blocks;                  // C / 64 for the pixel_shuffle modes
  int epi_mode;
  int gelu;
  int remap;                     // 0: none; 1: transpose 16x16 token grid; 2: 8x8
  int out_f32;                   // 1: store fp32 instead of bf16
  void* out;
  long long ldo;                 // elements
  int group_col_stride;          // output column offset per group (blockIdx.z)
  const __nv_bfloat16* bias[GEMM_MAX_GROUPS];  // EPI_BIAS, per group (may be null)
  const float* colsum;           // EPI_LNFOLD
  const float* fbias;            // EPI_LNFOLD
  const float* row_mean;         // EPI_LNFOLD
  const float* row_rstd;         // EPI_LNFOLD
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr uint32_t B_BYTES = BN * GEMM_BK * 2;
  static constexpr uint32_t RING = STAGES * (A_BYTES + B_BYTES);
  static constexpr uint32_t BARS = (2 * STAGES + 1) * 8 + 16;
  static constexpr uint32_t COLS = 2 * BN * 4;
  static constexpr uint32_t TOTAL = 1024 + RING + BARS + COLS;
};

__device__ __forceinline__ float gelu_erf(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_sm100_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args,
                      int* __restrict__ status) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::A_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::RING);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* accum_bar = empty_bar + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_bar + 1);
  float* s_col0 = reinterpret_cast<float*>(smem + L::RING + L::BARS);
  float* s_col1 = s_col0 + BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.z;
  const int m0 = blockIdx.y * GEMM_BM;
  const int n0 = blockIdx.x * BN;
  const int KT = args.K / GEMM_BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&maps.a);
    tma_prefetch_desc(&maps.b[g]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // Per-column epilogue vectors for this tile, staged once in shared memory.
    for (int i = threadIdx.x - 64; i < BN; i += 128) {
      const int n = n0 + i;
      float c0 = 0.f, c1 = 0.f;
      if (n < args.N) {
        if (args.epi_mode == EPI_LNFOLD) {
          c0 = args.colsum[n];
          c1 = args.fbias[n];
        } else if (args.bias[g] != nullptr) {
          c1 = __bfloat162float(args.bias[g][n]);
        }
      }
      s_col0[i] = c0;
      s_col1[i] = c1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      for (int kk = 0; kk < KT; ++kk) {
        const int s = kk % STAGES;
        const uint32_t ph = (kk / STAGES) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&full_bar[s], L::A_BYTES + L::B_BYTES);
        uint8_t* a_dst = sA + s * L::A_BYTES;
        if (args.a_mode == A_PLAIN) {
          tma_load_2d(a_dst, &maps.a, &full_bar[s], kk * GEMM_BK, m0);
        } else {
          const int blk = kk / args.c_blocks;
          const int c0 = (kk - blk * args.c_blocks) * GEMM_BK;
          if (args.a_mode == A_PS_HALF) {
            tma_load_5d(a_dst, &maps.a, &full_bar[s], c0, blk & 1, 0, blk >> 1, m0 >> 4);
          } else {
            int q, r;
            if (args.a_mode == A_PS_QUARTER) {
              q = blk >> 2;
              r = blk & 3;
            } else {  // two successive factor-0.5 shuffles: blk = 8ei + 4ej + 2di + dj
              q = 2 * (blk >> 3) + ((blk >> 1) & 1);
              r = 2 * ((blk >> 2) & 1) + (blk & 1);
            }
            tma_load_5d(a_dst, &maps.a, &full_bar[s], c0, r, 0, q, m0 >> 3);
          }
        }
        tma_load_2d(sB + s * L::B_BYTES, &maps.b[g], &full_bar[s], kk * GEMM_BK, n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(GEMM_BM, BN);
      for (int kk = 0; kk < KT; ++kk) {
        const int s = kk % STAGES;
        const uint32_t ph = (kk / STAGES) & 1;
        if (!mbar_wait(&full_bar[s], ph)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * L::A_BYTES));
        const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * L::B_BYTES));
#pragma unroll
        for (int k = 0; k < GEMM_BK / 16; ++k) {
          // advance 16 bf16 = 32 bytes (2 x 16 B) along K inside the swizzle atom
          umma_bf16(tmem_base, ad + 2 * k, bd + 2 * k, idesc, (kk | k) != 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[s]);
      }
      umma_commit(accum_bar);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int row = m0 + quad * 32 + lane;
    if (!mbar_wait(accum_bar, 0)) ok = false;
    __syncwarp();
    tc_fence_after();
    float mean = 0.f, rstd = 1.f;
    if (args.epi_mode == EPI_LNFOLD && row < args.M) {
      mean = args.row_mean[row];
      rstd = args.row_rstd[row];
    }
    const float nms = -mean * rstd;
    long long out_row = row;
    if (args.remap == 1) {
      const int t = row & 255;
      out_row = (row & ~255) | ((t & 15) << 4) | (t >> 4);
    } else if (args.remap == 2) {
      const int t = row & 63;
      out_row = (row & ~63) | ((t & 7) << 3) | (t >> 3);
    }
    const long long out_off = out_row * args.ldo + (long long)g * args.group_col_stride + n0;
    const bool ok_any = __all_sync(0xffffffffu, ok);
    if (ok_any) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c, r);
        tmem_ld_wait();
        if (row < args.M && n0 + c < args.N) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float t = __uint_as_float(r[i]);
            if (args.epi_mode == EPI_LNFOLD)
              t = fmaf(rstd, t, nms * s_col0[c + i]) + s_col1[c + i];
            else
              t += s_col1[c + i];
            v[i] = args.gelu ? gelu_erf(t) : t;
          }
          if (args.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.out) + out_off + c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + out_off + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                                  pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                  pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                  pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          }
        }
      }
    }
  }

  if (!ok && status != nullptr) atomicOr(status, 4 /* IVC_DEV_WAIT_TIMEOUT */);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, BN);
  }
}

}  // namespace ivc
