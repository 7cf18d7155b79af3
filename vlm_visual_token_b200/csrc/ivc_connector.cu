// ivc_connector.cu — pixel_shuffle + connector MLP kernels for sm_100a.
//
// LayerNorm ("MLP 连接器源码逐行解析" of the InternVL3-14B-Instruct connector
// article: LayerNorm(4C) -> Linear -> GELU -> Linear) is applied without ever
// writing the normalised rows: with mean mu and rstd of row P,
//   LN(P) W0^T + b0 = rstd * (P (W0*gamma)^T - mu * colsum(W0*gamma)) + (b0 + W0 beta),
// so the first GEMM multiplies the raw pixel-shuffled features (read through
// the 5-D TMA map, see ivc_gemm.cuh) and its epilogue applies rstd, mu and the
// two folded column vectors. ps_stats_kernel computes mu and rstd of every
// shuffled row in one pass over the features.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdlib>
#include <mutex>

#include "ivc_device_once.h"
#include "ivc_gemm.cuh"
#include "ivc_internal.h"

namespace ivc {

// ---------------------------------------------------------------- LN statistics
// A 4x4 block of ViT tokens ("cell") is one factor-0.25 row; its four 2x2
// sub-blocks are four factor-0.5 rows. Each CTA takes PS_CELLS adjacent
// cells; warp w = 4q + r reduces token (4a+q, 4b+r) of each of them over C
// channels (sums shifted by the token's first value to keep the one-pass
// variance well conditioned), all of its loads in flight before their use.
// The token statistics are then merged per row with the pairwise (Chan)
// update in fp64.
constexpr int PS_CELLS = 2;

__device__ __forceinline__ void token_moments(const uint4* __restrict__ v, int pieces, int lane,
                                              float shift, float& s1, float& s2,
                                              const uint4 (&u)[4], int i0) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (i0 + k * 32 + lane >= pieces) continue;
    const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16) - shift;
      const float hi = __uint_as_float(w[j] & 0xffff0000u) - shift;
      s1 += lo + hi;
      s2 = fmaf(lo, lo, fmaf(hi, hi, s2));
    }
  }
  (void)v;
}

__global__ void __launch_bounds__(512) ps_stats_kernel(const bf16* __restrict__ x, int C,
                                                       float* __restrict__ mean_half,
                                                       float* __restrict__ rstd_half,
                                                       float* __restrict__ mean_quarter,
                                                       float* __restrict__ rstd_quarter) {
  __shared__ double s_mean[PS_CELLS][16], s_m2[PS_CELLS][16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp >> 2, r = warp & 3;
  pdl_wait();
  pdl_trigger();
  const int pieces = C / 8;  // 16-byte pieces per token
  const uint4* v[PS_CELLS];
  float shift[PS_CELLS], s1[PS_CELLS], s2[PS_CELLS];
#pragma unroll
  for (int e = 0; e < PS_CELLS; ++e) {
    const int cell = blockIdx.x * PS_CELLS + e;  // tile * 64 + a * 8 + b
    const int tile = cell >> 6, a = (cell >> 3) & 7, b = cell & 7;
    const bf16* tok = x + ((static_cast<long long>(tile) * 32 + 4 * a + q) * 32 + 4 * b + r) * C;
    v[e] = reinterpret_cast<const uint4*>(tok);
    shift[e] = __bfloat162float(tok[0]);
    s1[e] = s2[e] = 0.f;
  }
  for (int i0 = 0; i0 < pieces; i0 += 128) {
    uint4 u[PS_CELLS][4];
#pragma unroll
    for (int e = 0; e < PS_CELLS; ++e)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = i0 + k * 32 + lane;
        // plain loads: x stays in L2 for the GEMMs that follow
        u[e][k] = i < pieces ? __ldg(v[e] + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
    for (int e = 0; e < PS_CELLS; ++e) token_moments(v[e], pieces, lane, shift[e], s1[e], s2[e], u[e], i0);
  }
#pragma unroll
  for (int e = 0; e < PS_CELLS; ++e) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1[e] += __shfl_xor_sync(0xffffffffu, s1[e], o);
      s2[e] += __shfl_xor_sync(0xffffffffu, s2[e], o);
    }
    if (lane == 0) {
      const double n = C;
      s_mean[e][warp] = shift[e] + s1[e] / n;
      s_m2[e][warp] =
          fmax(static_cast<double>(s2[e]) - static_cast<double>(s1[e]) * s1[e] / n, 0.0);
    }
  }
  __syncthreads();
  const double eps = 1e-5;
  if (threadIdx.x < 4 * PS_CELLS && mean_half != nullptr) {
    const int e = threadIdx.x >> 2;
    const int cell = blockIdx.x * PS_CELLS + e;
    const int tile = cell >> 6, a = (cell >> 3) & 7, b = cell & 7;
    const int sa = (threadIdx.x >> 1) & 1, sb = threadIdx.x & 1;
    const int w0 = 4 * (2 * sa) + 2 * sb;  // tokens (2sa+di, 2sb+dj)
    const int ids[4] = {w0, w0 + 1, w0 + 4, w0 + 5};
    double mu = 0.0;
    for (int i = 0; i < 4; ++i) mu += s_mean[e][ids[i]];
    mu *= 0.25;
    double m2 = 0.0;
    for (int i = 0; i < 4; ++i) {
      const double d = s_mean[e][ids[i]] - mu;
      m2 += s_m2[e][ids[i]] + C * d * d;
    }
    const double var = m2 / (4.0 * C);
    const long long row = static_cast<long long>(tile) * 256 + (2 * a + sa) * 16 + (2 * b + sb);
    mean_half[row] = static_cast<float>(mu);
    rstd_half[row] = static_cast<float>(1.0 / sqrt(var + eps));
  }
  if (threadIdx.x >= 32 && threadIdx.x < 32 + PS_CELLS && mean_quarter != nullptr) {
    const int e = threadIdx.x - 32;
    const int cell = blockIdx.x * PS_CELLS + e;
    double mu = 0.0;
    for (int i = 0; i < 16; ++i) mu += s_mean[e][i];
    mu *= 1.0 / 16.0;
    double m2 = 0.0;
    for (int i = 0; i < 16; ++i) {
      const double d = s_mean[e][i] - mu;
      m2 += s_m2[e][i] + C * d * d;
    }
    const double var = m2 / (16.0 * C);
    mean_quarter[cell] = static_cast<float>(mu);
    rstd_quarter[cell] = static_cast<float>(1.0 / sqrt(var + eps));
  }
}

int launch_ps_stats(const bf16* x, int T, int C, float* mean_half, float* rstd_half,
                    float* mean_quarter, float* rstd_quarter, const Launch& L) {
  if (T == 0) return IVC_OK;
  TraceScope ts("ps_stats", L.stream);
  // T * 64 cells, an even number
  return launch_k(ps_stats_kernel, dim3(T * 64 / PS_CELLS), dim3(512), 0, L.stream, 1, x, C,
                  mean_half, rstd_half, mean_quarter, rstd_quarter);
}

// ---------------------------------------------------------------- LN fold
// One warp per output feature n: W_out[n,k] = bf16(W[n,k] * gamma[k]),
// colsum[n] = sum_k W_out[n,k], fbias[n] = b[n] + sum_k W[n,k] * beta[k].
__global__ void __launch_bounds__(256) fold_kernel(const bf16* __restrict__ W,
                                                   const bf16* __restrict__ b,
                                                   const bf16* __restrict__ gamma,
                                                   const bf16* __restrict__ beta, int N, int K,
                                                   bf16* __restrict__ W_out,
                                                   float* __restrict__ colsum,
                                                   float* __restrict__ fbias) {
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (n >= N) return;
  const bf16* w = W + static_cast<long long>(n) * K;
  bf16* wo = W_out + static_cast<long long>(n) * K;
  double cs = 0.0, fb = 0.0;
  for (int k = lane; k < K; k += 32) {
    const float wv = __bfloat162float(w[k]);
    const bf16 scaled = __float2bfloat16_rn(wv * __bfloat162float(gamma[k]));
    wo[k] = scaled;
    cs += static_cast<double>(__bfloat162float(scaled));
    fb += static_cast<double>(wv) * static_cast<double>(__bfloat162float(beta[k]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cs += __shfl_xor_sync(0xffffffffu, cs, o);
    fb += __shfl_xor_sync(0xffffffffu, fb, o);
  }
  if (lane == 0) {
    colsum[n] = static_cast<float>(cs);
    fbias[n] = static_cast<float>(fb + (b ? static_cast<double>(__bfloat162float(b[n])) : 0.0));
  }
}

int launch_fold(const bf16* W, const bf16* b, const bf16* gamma, const bf16* beta, int N, int K,
                bf16* W_out, float* colsum, float* fbias, const Launch& L) {
  TraceScope ts("ln_fold", L.stream);
  return launch_k(fold_kernel, dim3((N + 7) / 8), dim3(256), 0, L.stream, 1, W, b, gamma, beta,
                  N, K, W_out, colsum, fbias);
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

static int encode(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return IVC_ECUDA;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                  strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IVC_OK : IVC_ECUDA;
}

// Row-major [rows, cols] bf16 matrix, box 64 columns x box_rows rows.
static int map_2d(CUtensorMap* m, const void* base, long long rows, long long cols,
                  int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {GEMM_BK, static_cast<cuuint32_t>(box_rows)};
  return encode(m, 2, base, dims, strides, box);
}

int map_rows_2d(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
  return map_2d(m, base, rows, cols, box_rows);
}

int map_bf16(CUtensorMap* m, int rank, const void* base, const unsigned long long* dims,
             const unsigned long long* strides_bytes, const unsigned* box) {
  cuuint64_t d[5], st[4];
  cuuint32_t b[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return encode(m, rank, base, d, st, b);
}

// Batched [batches][rows][inner] bf16 (row stride ld, batch stride bs elements),
// box {box_inner, box_rows, 1}.
static int map_3d(CUtensorMap* m, const void* base, long long batches, long long rows,
                  long long inner, long long ld, long long bs, int box_inner, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batches)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, static_cast<cuuint64_t>(bs) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  return encode(m, 3, base, dims, strides, box);
}

// The [T,32,32,C] features seen as the pixel-shuffled [T*tokens, f*f*C] matrix;
// one box is 128 rows, or (one_tile, f = 4) the 64 rows of one tile.
static int map_ps(CUtensorMap* m, const void* x, int T, int C, int f, bool one_tile = false) {
  const cuuint64_t Cu = static_cast<cuuint64_t>(C);
  const int g = 32 / f;  // output grid side
  cuuint64_t dims[5] = {Cu, static_cast<cuuint64_t>(f), static_cast<cuuint64_t>(g),
                        static_cast<cuuint64_t>(f), static_cast<cuuint64_t>(T) * g};
  // strides (bytes) of dims 1..4: next column in the block, next output
  // column b, next row in the block, next output row (a) / tile.
  cuuint64_t strides[4] = {Cu * 2, Cu * f * 2, Cu * 32 * 2, Cu * 32 * f * 2};
  const int outer = one_tile && g * g < GEMM_BM ? g : GEMM_BM / g;
  cuuint32_t box[5] = {GEMM_BK, 1, static_cast<cuuint32_t>(g), 1, static_cast<cuuint32_t>(outer)};
  return encode(m, 5, x, dims, strides, box);
}

static DeviceTable& device_table() {
  static DeviceTable t;
  return t;
}

int num_sms() {
  static const char key = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = device_table().get(&key, dev);
  if (n > 0) return n;
  int q = 0;
  if (cudaDeviceGetAttribute(&q, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || q <= 0)
    q = 148;
  device_table().raise(&key, dev, q, [] { return 0; });
  return q;
}

int smem_optin(const void* kern, size_t bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return IVC_ECUDA;
  const int rc = device_table().raise(kern, dev, static_cast<int>(bytes), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes)) == cudaSuccess
               ? 0
               : 1;
  });
  return rc == 0 ? IVC_OK : IVC_ECUDA;
}

template <int BN, int STAGES, int CG>
static int run_gemm(const GemmMaps& maps, const GemmArgs& args, const char* tag, int units_cap,
                    const Launch& L) {
  using S = GemmSmem<BN, STAGES, CG>;
  auto kern = gemm_sm100_kernel<BN, STAGES, CG>;
  if (smem_optin(reinterpret_cast<const void*>(kern), S::TOTAL) != IVC_OK) return IVC_ECUDA;
  const long long tiles = static_cast<long long>((args.M + GEMM_BM * CG - 1) / (GEMM_BM * CG)) *
                          ((args.N + BN - 1) / BN) * args.groups;
  const long long units = units_cap;
  // with split-K the last round is cut into slices for every unit
  const int grid = CG * static_cast<int>(tiles < units && args.split_max <= 1 ? tiles : units);
  TraceScope ts(tag ? tag : "gemm", L.stream);
  return launch_k(kern, dim3(grid), dim3(GEMM_THREADS), S::TOTAL, L.stream, CG, maps, args,
                  L.status);
}

// Finishes the split tiles of a GEMM (GemmArgs.split_max): each element of a
// split tile is the sum of its S fp32 k-slice partials, then the epilogue the
// GEMM itself applies (LayerNorm fold or bias, GELU, row remaps, bf16/fp32
// store). Each thread owns 8 consecutive columns of one row. Exits at once
// when the GEMM split nothing (split_s[0] == 1).
__global__ void __launch_bounds__(256)
    splitk_epilogue_kernel(const __grid_constant__ GemmArgs args, int tile_m, int bn) {
  pdl_wait();
  pdl_trigger();
  const int S = args.split_s[0];
  if (S <= 1) return;
  const int first = args.split_s[1], n_split = args.split_s[2];
  int M = args.M;
  if (args.list_count != nullptr) {
    const int c = *args.list_count;
    const long long rows = static_cast<long long>(c < 0 ? 0 : c) * args.item_rows;
    M = rows < M ? static_cast<int>(rows) : M;
  }
  const int m_tiles = (M + tile_m - 1) / tile_m;
  const int n_tiles = (args.N + bn - 1) / bn;
  const int cols8 = bn / 8;
  const long long per_tile = static_cast<long long>(tile_m) * cols8;
  const long long n = n_split * per_tile;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int tt = static_cast<int>(i / per_tile);
    const int in_tile = static_cast<int>(i % per_tile);
    const int lr = in_tile / cols8, lc = (in_tile % cols8) * 8;
    const TileCoord tc = tile_coord(first + tt, m_tiles, n_tiles, tile_m, bn);
    const int row = tc.m0 + lr, c0 = tc.n0 + lc;
    if (row >= M || c0 >= args.N) continue;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const float* p = args.split_part + (static_cast<long long>(tt) * S * tile_m + lr) * bn + lc;
    const long long slice = static_cast<long long>(tile_m) * bn;
#pragma unroll 4
    for (int sl = 0; sl < S; ++sl) {
      const float4 a = __ldcs(reinterpret_cast<const float4*>(p + sl * slice));
      const float4 b = __ldcs(reinterpret_cast<const float4*>(p + sl * slice + 4));
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    if (args.epi_mode == EPI_LNFOLD) {
      const int sr = args.stats_remap
                         ? args.list[row / args.item_rows] * args.item_rows + row % args.item_rows
                         : row;
      const float rstd = args.row_rstd[sr];
      const float nms = -args.row_mean[sr] * rstd;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = fmaf(rstd, v[j], nms * args.colsum[c0 + j]) + args.fbias[c0 + j];
    } else if (args.bias[0] != nullptr) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] += __bfloat162float(args.bias[0][c0 + j]);
    }
    if (args.gelu) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = gelu_erf(v[j]);
    }
    long long out_row = row;
    if (args.remap == 1) {
      const int t = row & 255;
      out_row = (row & ~255) | ((t & 15) << 4) | (t >> 4);
    } else if (args.remap == 2) {
      const int t = row & 63;
      out_row = (row & ~63) | ((t & 7) << 3) | (t >> 3);
    }
    if (args.out_base != nullptr)
      out_row = args.out_base[row / args.item_rows] + out_row % args.item_rows;
    const long long off = out_row * args.ldo + c0;
    if (args.out_f32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.out) + off);
      dst[0] = make_float4(v[0], v[1], v[2], v[3]);
      dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + off) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                     pack_bf16x2(v[6], v[7]));
    }
  }
}

size_t splitk_part_floats() { return static_cast<size_t>(num_sms()) * GEMM_BM * 512; }

// 512-wide pair tiles (see launch_gemm) with IVC_GEMM_WIDE=1. Off by
// default: on the 13-tile image they cut mlp2.fc1 from ~145 to ~106 us, but
// the split-K finishing launches they need (their partials re-read from
// DRAM, ~13-20 us each) cost more than that in the whole step (0.514 against
// 0.497 ms per call).
static bool wide_tiles_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("IVC_GEMM_WIDE");
    on = (e && e[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

// 256-wide tiles run on CTA pairs unless IVC_GEMM_PAIRS=0 (kept for
// comparing the two variants on the same build).
static bool pairs_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("IVC_GEMM_PAIRS");
    on = (e && e[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

// L2 prefetch distance of streamed weights in k-steps (IVC_GEMM_PREFETCH, default 0: measured no gain).
static int prefetch_depth() {
  static int d = -1;
  if (d < 0) {
    const char* e = std::getenv("IVC_GEMM_PREFETCH");
    d = e ? std::atoi(e) : 0;
    if (d < 0) d = 0;
  }
  return d;
}

// Output tile width. Measured on B200 (tcgen05 M=128, TMA-fed ring with
// L2-resident operands): N=256 tiles run at ~1.8-2.2 PFLOP/s, N=128 tiles at
// ~1.08 PFLOP/s, i.e. an N=128 tile takes as long as an N=256 one. So 256 is
// used whenever N > 128, even when it leaves SMs idle.
static int pick_bn(const GemmCall& c) {
  if (c.N <= 32) return 32;
  if (c.N <= 64) return 64;
  if (c.N <= 128) return 128;
  return 256;
}

int launch_gemm(const GemmCall& c, const Launch& L) {
  if (c.M == 0 || c.N == 0) return IVC_OK;
  if (c.K % GEMM_BK != 0 || c.N % 32 != 0 || c.groups < 1 || c.groups > GEMM_MAX_GROUPS)
    return IVC_EUNSUPPORTED;
  if (c.b_mode != B_K2D && (c.b_batch_rows <= 0 || c.b_batch_rows % GEMM_BM != 0))
    return IVC_EUNSUPPORTED;
  if (c.b_mode == B_MN3D && c.N % 64 != 0) return IVC_EUNSUPPORTED;
  int bn = pick_bn(c);
  // CTA pairs (cta_group::2) for 256-wide tiles of plain K-major weights.
  const int cg = (bn == 256 && c.b_mode == B_K2D && pairs_enabled()) ? 2 : 1;
  // 512-wide pair tiles where split-K can still fill the GPU: a host-known
  // row count, split scratch, and at most half as many tiles as pair units
  // (S >= 2). Per CTA and k-step they move 48 KB for 2x the MMA work of a
  // 256-wide tile's 32 KB, and their weight box is one 32 KB request.
  if (cg == 2 && c.N % 512 == 0 && c.list_count == nullptr && c.split_part != nullptr &&
      c.groups == 1 && wide_tiles_enabled()) {
    const long long tiles512 = static_cast<long long>((c.M + 255) / 256) * (c.N / 512);
    if (2 * tiles512 <= num_sms() / 2 && c.K / GEMM_BK >= 16) bn = 512;
  }

  GemmMaps maps;
  int rc;
  switch (c.a_mode) {
    case A_PLAIN: rc = map_2d(&maps.a, c.a, c.M, c.K, GEMM_BM); break;
    case A_PS_HALF: rc = map_ps(&maps.a, c.a, c.T, c.C, 2); break;
    default: rc = map_ps(&maps.a, c.a, c.T, c.C, 4, c.list != nullptr); break;
  }
  if (rc) return rc;
  for (int g = 0; g < c.groups; ++g) {
    if (c.b_mode == B_K2D)
      rc = map_2d(&maps.b[g], c.B[g], c.N, c.K, bn / cg);
    else if (c.b_mode == B_K3D)
      rc = map_3d(&maps.b[g], c.B[g], c.b_batches, c.N, c.K, c.b_ld, c.b_batch_stride, GEMM_BK,
                  bn);
    else
      rc = map_3d(&maps.b[g], c.B[g], c.b_batches, c.K, c.N, c.b_ld, c.b_batch_stride, 64,
                  GEMM_BK);
    if (rc) return rc;
  }
  // persistent units (CTAs, or pairs): all SMs, or fewer when c.reserve_sms
  // leaves room for concurrent work without adding a round of tiles
  int units = num_sms() / cg;
  if (c.reserve_sms > 0) {
    const int tile_m = GEMM_BM * cg;
    const long long tiles = static_cast<long long>((c.M + tile_m - 1) / tile_m) *
                            ((c.N + bn - 1) / bn) * c.groups;
    const int capped = (num_sms() - c.reserve_sms) / cg;
    if (capped > 0 && (tiles + capped - 1) / capped == (tiles + units - 1) / units) units = capped;
  }
  GemmArgs a{};
  a.M = c.M;
  a.N = c.N;
  a.K = c.K;
  a.groups = c.groups;
  a.a_mode = c.a_mode;
  a.b_mode = c.b_mode;
  a.b_batch_rows = c.b_mode == B_K2D ? 0 : c.b_batch_rows;
  a.c_blocks = c.C / GEMM_BK;
  // Weights that stream from HBM once per M-tile row (long K): prefetch the
  // B operand ~16 k-steps ahead into L2 so TMA loads see L2 latency.
  a.b_prefetch = (c.b_mode == B_K2D && c.K >= 2048) ? prefetch_depth() : 0;
  a.epi_mode = c.epi_mode;
  a.gelu = c.gelu;
  a.remap = c.remap;
  a.out = c.out;
  a.out_f32 = c.out_f32;
  a.m_valid = c.m_valid;
  a.ldo = c.ldo;
  a.group_col_stride = c.N;
  for (int g = 0; g < c.groups; ++g) a.bias[g] = c.bias[g];
  a.colsum = c.colsum;
  a.fbias = c.fbias;
  a.row_mean = c.row_mean;
  a.row_rstd = c.row_rstd;
  a.list = c.list;
  a.list_count = c.list_count;
  a.out_base = c.out_base;
  a.item_rows = c.item_rows;
  a.stats_remap = c.stats_remap;
  // Split-K where the output tiles leave SMs idle. With a host-known row
  // count the slice count is fixed here; with a device row count (routed
  // rows) the kernel picks it and the finishing kernel always runs.
  if (c.split_part != nullptr && c.split_s != nullptr && c.groups == 1 && c.b_mode == B_K2D &&
      c.m_valid == 0) {
    const int n_tiles = (c.N + bn - 1) / bn;
    const int KT = c.K / GEMM_BK;
    const int tile_m = GEMM_BM * cg;
    constexpr int kMaxSplit = 8;
    const int split_min = bn > 256 ? 2 : 4;
    a.split_min = split_min;
    if (c.list_count == nullptr) {
      // the kernel's own choice, known here: skip the finishing launch if 1
      const int rem = (((c.M + tile_m - 1) / tile_m) * n_tiles) % units;
      const int S = rem > 0 ? split_count(kMaxSplit, units, rem, KT, split_min) : 1;
      a.split_max = S > 1 ? S : 0;
    } else {
      // the row count is known only on the device: the kernel decides
      a.split_max = KT >= 16 ? kMaxSplit : 0;
    }
    if (a.split_max > 1) {
      if (c.N % 8 != 0) return IVC_EUNSUPPORTED;
      a.split_part = c.split_part;
      a.split_s = c.split_s;
    }
  }
  if (c.list_count != nullptr && (c.item_rows <= 0 || (c.item_rows != 256 && c.item_rows != 64)))
    return IVC_EINVAL;
  if ((c.list != nullptr || c.stats_remap || c.out_base != nullptr) && c.list_count == nullptr)
    return IVC_EINVAL;
  if (c.stats_remap && c.list == nullptr) return IVC_EINVAL;
  a.epi_dep_only = (c.epi_dep_only && a.split_max <= 1 && c.list_count == nullptr) ? 1 : 0;
  int rc2;
  switch (bn) {
    case 512: rc2 = run_gemm<512, 4, 2>(maps, a, c.tag, units, L); break;
    case 256: rc2 = cg == 2 ? run_gemm<256, 6, 2>(maps, a, c.tag, units, L)
                            : run_gemm<256, 4, 1>(maps, a, c.tag, units, L);
      break;
    case 128: rc2 = run_gemm<128, 6, 1>(maps, a, c.tag, units, L); break;
    case 64: rc2 = run_gemm<64, 8, 1>(maps, a, c.tag, units, L); break;
    default: rc2 = run_gemm<32, 8, 1>(maps, a, c.tag, units, L); break;
  }
  if (rc2 != IVC_OK || a.split_max <= 1) return rc2;
  // one thread per 8 output columns of a split tile (at most units tiles of
  // TILE_M x bn), so that every partial load is in flight at once
  const long long items = static_cast<long long>(units) * GEMM_BM * cg * (bn / 8);
  const int blocks = static_cast<int>((items + 255) / 256);
  TraceScope ts("splitk.epilogue", L.stream);
  return launch_k(splitk_epilogue_kernel, dim3(blocks), dim3(256), 0, L.stream, 1, a,
                  GEMM_BM * cg, bn);
}

}  // namespace ivc
