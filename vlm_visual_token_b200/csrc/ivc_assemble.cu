// ivc_assemble.cu — sequence assembly: the compacted visual rows spliced into
// the token sequences for the language model.
//
// InternVL3-14B-Instruct connector article, "视觉 Token 如何注入 Qwen2.5 语言模型":
// the prompt's <IMG_CONTEXT> positions (256 per tile) are replaced, in order,
// by the visual rows. InternVL3_5-4B-Flash article, section 4, and the
// InternVL3_5-2B-Flash article, "路由决策": for a compressed tile 192 of its
// 256 placeholders are deleted from the sequence (the first 64 stay) and the
// position indices follow the shortened sequence.
//
// Two kernels. assemble_scan_kernel (one CTA) walks the batch once with two
// block scans: the running placeholder number j (tile j / 256, slot j % 256)
// and the running count of kept tokens, which is each kept token's output
// row; it records the row's source (visual row or text token) and the new
// sequence offsets. assemble_rows_kernel then moves the rows (16-byte pieces,
// 8 rows per CTA) and writes the position ids.
#include <cuda_runtime.h>

#include "ivc_internal.h"
#include "ivc_ptx.cuh"

namespace ivc {

constexpr int AS_THREADS = 1024;
constexpr int AS_FULL = 256;  // placeholders per tile
constexpr int AS_KEEP = 64;   // kept for a compressed tile

// Workspace after the 256-byte header: src [L] (text: input position; visual:
// -1 - visual row), total [1].
struct AssembleBufs {
  int32_t* src;
  int32_t* total;
};

__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int& block_total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  const int before = warp > 0 ? s_warp[warp - 1] : 0;
  block_total = s_warp[31];
  __syncthreads();  // s_warp is reused by the next scan
  return before + incl - v;
}

constexpr int AS_PER = 4;                       // tokens per thread per pass
constexpr int AS_CHUNK = AS_THREADS * AS_PER;   // tokens per pass
constexpr int AS_ROWS = 8;                      // output rows per CTA of the row copy

__global__ void __launch_bounds__(AS_THREADS)
    assemble_scan_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ seq_off,
                         int B, int L, int32_t img_id, const uint8_t* __restrict__ mask,
                         const int32_t* __restrict__ offsets, int T, int32_t* __restrict__ out_ids,
                         int32_t* __restrict__ out_seq_off, AssembleBufs wb,
                         int* __restrict__ status) {
  __shared__ int s_warp[32];
  __shared__ int s_kept[AS_CHUNK];
  pdl_wait();
  pdl_trigger();
  // sequence offsets must be 0 = s_0 <= ... <= s_B = L
  if (threadIdx.x == 0) {
    bool bad = seq_off[0] != 0 || seq_off[B] != L;
    for (int b = 0; b < B && !bad; ++b) bad = seq_off[b + 1] < seq_off[b];
    if (bad) atomicOr(status, DEV_BAD_PROMPT);
  }
  const long long n_ph = static_cast<long long>(AS_FULL) * T;
  int carry_j = 0, carry_o = 0;
  for (int base = 0; base < L; base += AS_CHUNK) {
    // thread i owns tokens base + AS_PER i .. + AS_PER - 1
    const int p0 = base + AS_PER * threadIdx.x;
    int32_t tok[AS_PER];
    int img[AS_PER], nimg = 0;
#pragma unroll
    for (int e = 0; e < AS_PER; ++e) {
      tok[e] = p0 + e < L ? ids[p0 + e] : 0;
      img[e] = (p0 + e < L && tok[e] == img_id) ? 1 : 0;
      nimg += img[e];
    }
    int tot_j;
    int j = carry_j + block_excl_scan(nimg, s_warp, tot_j);
    int keep[AS_PER], vrow[AS_PER], nkeep = 0;
#pragma unroll
    for (int e = 0; e < AS_PER; ++e) {
      const bool visual = img[e] && j < n_ph;
      const int t = visual ? j / AS_FULL : 0, r = visual ? j % AS_FULL : 0;
      keep[e] = (p0 + e < L && !(visual && mask[t] != 0 && r >= AS_KEEP)) ? 1 : 0;
      vrow[e] = visual ? offsets[t] + r : -1;
      j += img[e];
      nkeep += keep[e];
    }
    int tot_o;
    int o = carry_o + block_excl_scan(nkeep, s_warp, tot_o);
#pragma unroll
    for (int e = 0; e < AS_PER; ++e) {
      s_kept[AS_PER * threadIdx.x + e] = o;  // kept tokens before position p0 + e
      if (keep[e]) {
        out_ids[o] = tok[e];
        wb.src[o] = vrow[e] >= 0 ? -1 - vrow[e] : p0 + e;
      }
      o += keep[e];
    }
    __syncthreads();
    // new offsets of the sequences that start inside this pass
    for (int b = threadIdx.x; b < B; b += AS_THREADS) {
      const int q = seq_off[b];
      if (q >= base && q < base + AS_CHUNK && q < L) out_seq_off[b] = s_kept[q - base];
    }
    __syncthreads();
    carry_j += tot_j;
    carry_o += tot_o;
  }
  // sequences starting at L (empty, at the end), the total, and (malformed
  // offsets, flagged above) starts below 0
  for (int b = threadIdx.x; b <= B; b += AS_THREADS) {
    const int q = seq_off[b];
    if (b == B || q >= L) out_seq_off[b] = carry_o;
    else if (q < 0) out_seq_off[b] = 0;
  }
  if (threadIdx.x == 0) {
    *wb.total = carry_o;
    if (carry_j != n_ph) atomicOr(status, DEV_BAD_PROMPT);
  }
}

// AS_ROWS output rows per CTA (grid = ceil(L / AS_ROWS); rows past the total
// are skipped): every thread first loads all of its 16-byte pieces of the
// CTA's rows, then stores them.
__global__ void __launch_bounds__(256)
    assemble_rows_kernel(const int32_t* __restrict__ ids, int B, const bf16* __restrict__ table,
                         int V, int H, const bf16* __restrict__ visual,
                         const int32_t* __restrict__ out_seq_off, AssembleBufs wb,
                         bf16* __restrict__ out, int32_t* __restrict__ out_pos,
                         int* __restrict__ status) {
  __shared__ const uint4* s_from[AS_ROWS];
  pdl_wait();
  pdl_trigger();
  const int total = *wb.total;
  const int o0 = blockIdx.x * AS_ROWS;
  if (o0 >= total) return;
  const int rows = min(AS_ROWS, total - o0);
  if (threadIdx.x < rows) {
    const int o = o0 + threadIdx.x;
    const int s = wb.src[o];
    const uint4* from = nullptr;
    if (s < 0) {
      from = reinterpret_cast<const uint4*>(visual + static_cast<size_t>(-1 - s) * H);
    } else {
      const int32_t tok = ids[s];
      if (tok >= 0 && tok < V)
        from = reinterpret_cast<const uint4*>(table + static_cast<size_t>(tok) * H);
      else
        atomicOr(status, DEV_BAD_PROMPT);
    }
    s_from[threadIdx.x] = from;
    // position within the sequence: the last sequence starting at or before
    // this row (empty sequences share their start with the next one)
    int lo = 0, hi = B;  // out_seq_off[lo] <= o < out_seq_off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (out_seq_off[mid] <= o) lo = mid; else hi = mid;
    }
    out_pos[o] = o - out_seq_off[lo];
  }
  __syncthreads();
  const int per_row = H / 8;
  const int n = rows * per_row;
  uint4* to = reinterpret_cast<uint4*>(out + static_cast<size_t>(o0) * H);  // rows contiguous
  for (int i0 = 0; i0 < n; i0 += 8 * 256) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + k * 256 + threadIdx.x;
      if (i < n) {
        const uint4* f = s_from[i / per_row];
        u[k] = f ? __ldg(f + i % per_row) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + k * 256 + threadIdx.x;
      if (i < n) __stcs(to + i, u[k]);
    }
  }
}

size_t assemble_ws(int L) {
  return 256 + ((static_cast<size_t>(L) * 4 + 255) & ~static_cast<size_t>(255)) + 256;
}

}  // namespace ivc

using namespace ivc;

extern "C" {

size_t ivc_assemble_workspace_size(int L) { return L < 0 ? 0 : assemble_ws(L); }

int ivc_assemble_sequence(const int32_t* input_ids, const int32_t* seq_offsets, int B, int L,
                          int32_t img_context_id, const void* embed_table, int V, int H,
                          const void* visual, const uint8_t* mask, const int32_t* offsets, int T,
                          int32_t* out_ids, void* out_embeds, int32_t* out_positions,
                          int32_t* out_seq_offsets, void* workspace, size_t ws_bytes,
                          ivc_stream_t stream) {
  if (L < 0 || B < 1 || T < 0 || V <= 0 || H <= 0) return IVC_EINVAL;
  if (H % 8 != 0) return IVC_EUNSUPPORTED;
  if (!seq_offsets || !out_seq_offsets || !workspace) return IVC_EINVAL;
  if (L > 0 && (!input_ids || !embed_table || !out_ids || !out_embeds || !out_positions))
    return IVC_EINVAL;
  if (T > 0 && (!visual || !mask || !offsets)) return IVC_EINVAL;
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al(embed_table) || !al(visual) || !al(out_embeds) || !al(workspace)) return IVC_EALIGN;
  if (ws_bytes < assemble_ws(L)) return IVC_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  char* w = static_cast<char*>(workspace) + 256;
  AssembleBufs wb;
  wb.src = reinterpret_cast<int32_t*>(w);
  wb.total = reinterpret_cast<int32_t*>(w + ((static_cast<size_t>(L) * 4 + 255) & ~static_cast<size_t>(255)));
  {
    TraceScope ts("assemble.scan", s);
    const int rc = launch_k(assemble_scan_kernel, dim3(1), dim3(AS_THREADS), 0, s, 1, input_ids,
                            seq_offsets, B, L, img_context_id, mask, offsets, T, out_ids,
                            out_seq_offsets, wb, status);
    if (rc != IVC_OK) return rc;
  }
  if (L == 0) return IVC_OK;
  TraceScope ts("assemble.rows", s);
  return launch_k(assemble_rows_kernel, dim3((L + AS_ROWS - 1) / AS_ROWS), dim3(256), 0, s, 1,
                  input_ids, B, static_cast<const bf16*>(embed_table), V, H,
                  static_cast<const bf16*>(visual), out_seq_offsets, wb,
                  static_cast<bf16*>(out_embeds), out_positions, status);
}

}  // extern "C"
