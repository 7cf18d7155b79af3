/*
 * ivc.h — C ABI of libivc.so: InternVL visual-token compression on B200.
 *
 * The library implements, for one GPU, the data-parallel hot path that the
 * InternVL pages describe between the vision encoder and the language model:
 *
 *   - pixel_shuffle (space-to-depth, ps_version v2) of each 32x32xC tile grid
 *     at factor 0.5 (1024 -> 256 tokens of 4C channels) and at factor 0.25
 *     (1024 -> 64 tokens of 16C channels), followed by the connector MLP
 *     (mlp1 = LayerNorm -> Linear -> GELU -> Linear; mlp2 = LayerNorm ->
 *     Linear -> GELU -> Linear -> GELU -> Linear);
 *   - the Flash Visual Resolution Router (ViR): CrossAttentionPooling (a
 *     learnable query refined by 4 masked multi-head cross-attention layers
 *     over each tile's tokens), Gating (4 residual MLP blocks, Linear(D,2),
 *     softmax), the double threshold gate > quantile_0.1(gate of the image)
 *     AND gate >= 0.5, and compaction of every tile to 64 or 256 rows.
 *
 * Sources, by page title and section:
 *   [PS]  InternVL3-14B-Instruct, "Pixel Shuffle + MLP connector, line by line":
 *         "Pixel Shuffle 源码逐行解析", "ps_version v1 与 v2",
 *         "MLP 连接器源码逐行解析", "extract_feature() 完整调用链".
 *   [DP]  InternVL3_5-2B-Flash, "1024->256->64 dual-path compression pipeline":
 *         table "三档 Token 规模", "双路压缩管线全流程拆解",
 *         "路由决策：相对 + 绝对双阈值判定", table "核心配置参数速查".
 *   [VIR] InternVL3_5-4B-Flash, "Gating and CrossAttentionPooling":
 *         section 2 (pooling), section 3 (Gating), section 4 (thresholds),
 *         section 5 (data flow).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument named as device memory must point to memory the
 *     caller allocated on the current CUDA device (e.g. by PyTorch). The
 *     library never allocates, frees or retains caller memory. Each call
 *     only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns; results are ready when the stream reaches them.
 *   - Tensors are dense and row-major. bf16 is IEEE bfloat16 stored in
 *     uint16_t. Weights use the nn.Linear layout [out, in]; biases, LayerNorm
 *     gamma/beta and the pooling query are bf16 vectors.
 *   - Device pointers must be 16-byte aligned (the TMA and vector paths need
 *     it); otherwise IVC_EALIGN.
 *   - Scratch memory is the caller's `workspace` of at least
 *     ivc_workspace_size() bytes, 256-byte aligned. Its first 256 bytes hold a
 *     sticky device status word that kernels set when they detect bad device
 *     data (a valid length or image offset out of range) or a bounded wait
 *     that ran out; read and clear it with ivc_device_status().
 *   - Return value: IVC_OK (0) or a negative IVC_E* code; on error nothing was
 *     enqueued unless the code is IVC_ECUDA.
 *   - Calls on different streams with the same workspace race.
 */
#ifndef IVC_H_
#define IVC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* ivc_stream_t; /* cudaStream_t */

enum ivc_status {
  IVC_OK = 0,
  IVC_EINVAL = -1,       /* null pointer, negative count, bad flag or enum */
  IVC_EUNSUPPORTED = -2, /* shape the kernels do not handle (see each call) */
  IVC_EWORKSPACE = -3,   /* workspace smaller than ivc_workspace_size() */
  IVC_ECUDA = -4,        /* a CUDA runtime or driver call failed */
  IVC_EDEVICE = -5,      /* the device status word is set (ivc_device_status) */
  IVC_EALIGN = -6        /* a pointer is not 16-byte aligned */
};

/* Bits of the device status word. */
enum ivc_device_bits {
  IVC_DEV_BAD_VALID_LEN = 1,  /* valid_len[t] outside [1, 1024]; clamped */
  IVC_DEV_BAD_OFFSETS = 2,    /* image_offsets not 0 = o0 <= o1 <= ... = T */
  IVC_DEV_WAIT_TIMEOUT = 4,   /* a pipeline barrier wait ran out; outputs invalid */
  IVC_DEV_GROUP_TOO_LARGE = 8, /* a quantile group above IVC_MAX_QUANTILE_GROUP */
  IVC_DEV_BAD_PROMPT = 16      /* sequence assembly: placeholders != 256 T, a token id
                                  outside [0, V) or seq_offsets not 0 <= ... = L */
};

#define IVC_MAX_QUANTILE_GROUP 8192

/* pixel_shuffle flags ([PS] "ps_version v1 与 v2"; [DP] table). */
enum ivc_ps_flags {
  IVC_PS_V1 = 1,            /* ps_version "v1": output token grid transposed */
  IVC_PS_QUARTER_TWICE = 2  /* factor 0.25 as two factor-0.5 calls (channel order) */
};

/* Connector MLP ([PS] "MLP 连接器源码逐行解析"; [DP] table "三档 Token 规模").
 * n_linear = 2: LN(dims[0]) -> W0 [dims[1],dims[0]] -> GELU -> W1 [dims[2],dims[1]].
 * n_linear = 3: LN(dims[0]) -> W0 -> GELU -> W1 -> GELU -> W2 [dims[3],dims[2]].
 * LayerNorm: biased variance, eps 1e-5; GELU: exact (erf).
 * The `fold_*` fields are optional device pointers written by ivc_mlp_fold()
 * (LayerNorm's affine part folded into W0); when fold_colsum is NULL every call
 * recomputes the fold into its workspace. */
typedef struct ivc_mlp {
  int n_linear;
  int dims[4];
  const void* ln_gamma;      /* bf16 [dims[0]] */
  const void* ln_beta;       /* bf16 [dims[0]] */
  const void* W[3];          /* bf16 [dims[i+1], dims[i]] */
  const void* b[3];          /* bf16 [dims[i+1]] */
  const void* fold_W0;       /* bf16 [dims[1], dims[0]] = W0 * gamma (per input column) */
  const float* fold_colsum;  /* fp32 [dims[1]]: row sums of fold_W0 */
  const float* fold_bias;    /* fp32 [dims[1]]: b0 + W0 beta */
} ivc_mlp;

/* ViR router ([VIR] sections 2-4; [DP] "双路压缩管线全流程拆解" step 3).
 * Pooling: 4 layers, each with its own Wq, Wk, Wv, Wo [D,D] and biases [D];
 * `heads` heads of width D/heads (must be 64); scale 1/sqrt(64); q_0 = query;
 * q_l = Wo_l attn(Wq_l q_{l-1} + bq_l, K_l, V_l) + bo_l; pooled = q_4.
 * Gating: 4 blocks h <- h + LN_b(W2_b GELU(W1_b h + b1_b) + b2_b) with
 * W1 [gate_hidden, D], W2 [D, gate_hidden]; then softmax(Wout h + bout),
 * Wout [2, D]. Routing: tile t is compressed iff
 * gate[t,0] > quantile(gate[.,0] over its group, rel_q) and gate[t,0] >= abs_t,
 * quantile by linear interpolation in fp64; group = image (scope 0) or the
 * whole batch (scope 1).
 * The `fold_*` fields are optional device pointers written by
 * ivc_router_fold() (folded pooling only); all NULL: every call projects the
 * first layer's query and applies Wo and the next Wq one after the other. */
typedef struct ivc_router {
  int D;
  int heads;
  int gate_hidden;
  const void* query;  /* bf16 [D] */
  const void *Wq[4], *bq[4], *Wk[4], *bk[4], *Wv[4], *bv[4], *Wo[4], *bo[4];
  const void *gW1[4], *gb1[4], *gW2[4], *gb2[4], *gln_g[4], *gln_b[4];
  const void *gWout, *gbout;
  double rel_q;       /* flash_relative_threshold, 0.1 */
  double abs_t;       /* flash_absolute_threshold, 0.5 */
  int quantile_scope; /* 0 = per image, 1 = whole batch */
  int pool_mode;      /* IVC_POOL_FOLDED (0) or IVC_POOL_LITERAL (1) */
  int gate_residual;  /* 0: h <- h + LN(u) (the listed block inside the residual);
                         1: h <- LN(h + u) (residual inside the LayerNorm) */
  const void* fold_u1;      /* bf16 [32, D]: layer 1's key-folded query, u_h = Wk_h^T Q_h / 8
                               with Q = Wq_1 query + bq_1; rows h hi, 16 + h lo part */
  const float* fold_c1;     /* fp32 [16]: bk_h . Q_h / 8 */
  const void* fold_wqo[3];  /* bf16 [D, 2D]: P_l = Wq_{l+2} Wo_{l+1}, row n = hi | lo of P_l[n,:] */
  const float* fold_bqo[3]; /* fp32 [D]: Wq_{l+2} bo_{l+1} + bq_{l+2} */
} ivc_router;

/* How CrossAttentionPooling is evaluated; both compute the same function.
 * LITERAL: K_l = X Wk_l^T + bk_l and V_l = X Wv_l^T + bv_l for all tokens (one
 *   grouped tensor-core GEMM, fp32 K/V), then per head softmax(Q.K/8) V.
 * FOLDED: with one query per tile the projections are reassociated exactly:
 *   scores = X (Wk_h^T Q_h / 8) + bk_h.Q_h / 8 and o_h = Wv_h (sum_t p_t x_t) + bv_h,
 *   evaluated in one pass over the raw features per layer (scores, running
 *   softmax and weighted sums per 128-token chunk, the chunks then merged;
 *   ~60x fewer FLOPs, no K/V tensor). The environment variable
 *   IVC_POOL_ATTEND=0 selects the earlier form of the separate kernels
 *   (scores and weighted sums as two tensor-core GEMMs with a softmax kernel
 *   between them). */
enum ivc_pool_mode { IVC_POOL_FOLDED = 0, IVC_POOL_LITERAL = 1 };

enum ivc_op {
  IVC_OP_PS_PROJECT_HALF = 1,    /* ivc_ps_project at factor 0.5 */
  IVC_OP_PS_PROJECT_QUARTER = 2, /* ivc_ps_project at factor 0.25 */
  IVC_OP_VIR_ROUTE = 3,
  IVC_OP_FLASH_COMPRESS = 4
};

/* Text for a status code (static storage). */
const char* ivc_strerror(int status);

/* Library version, major*10000 + minor*100 + patch. */
int ivc_version(void);

/* Workspace bytes that `op` needs for T tiles of width C. `m` is the MLP of
 * ps_project (factor 0.5 or 0.25) or mlp1 of flash_compress, `m2` is mlp2 of
 * flash_compress, `r` the router (NULL where the op has none). Returns 0 for
 * invalid arguments. */
size_t ivc_workspace_size(int op, int T, int C, const ivc_mlp* m, const ivc_mlp* m2,
                          const ivc_router* r);

/* Fold LayerNorm's gamma and beta into the first Linear of `m`, once per set
 * of weights: fold_W0 = W0 * gamma, fold_colsum[n] = sum_k fold_W0[n,k],
 * fold_bias = b0 + W0 beta. The connector then computes
 * LN(P) W0^T + b0 = rstd (P fold_W0^T - mean * fold_colsum) + fold_bias
 * inside the GEMM epilogue (an exact rewrite of the LayerNorm of [PS]).
 * `dst` (device, >= ivc_mlp_fold_size(m) bytes) receives the three arrays;
 * on success m->fold_* point into it. */
size_t ivc_mlp_fold_size(const ivc_mlp* m);
int ivc_mlp_fold(ivc_mlp* m, void* dst, size_t dst_bytes, ivc_stream_t stream);

/* Fold the router's weights once per set of weights (folded pooling,
 * pool_mode = IVC_POOL_FOLDED, only). [VIR] section 2 chains the four pooling
 * layers with nothing between one layer's output projection and the next
 * layer's query projection, and starts from a learnable query, so
 *   layer 1's query Q_1 = Wq_1 query + bq_1 and its key fold u1, c1 depend on
 *   the weights alone, and
 *   Wq_{l+1} (Wo_l o + bo_l) + bq_{l+1} = P_l o + (Wq_{l+1} bo_l + bq_{l+1})
 *   with P_l = Wq_{l+1} Wo_l (l = 1..3),
 * an exact rewrite that saves five dependent launches per call. P_l is formed
 * in fp32 and kept as a bf16 hi | lo pair (about 16 significant bits); the
 * router's vectors stay fp32.
 * `dst` (device, 256-byte aligned, >= ivc_router_fold_size(r) bytes) receives
 * the arrays; on success r->fold_* point into it and every later call with `r`
 * uses them. Returns IVC_EUNSUPPORTED for literal pooling or an unsupported
 * shape, IVC_EINVAL for missing weights, IVC_EWORKSPACE for a short `dst`.
 * Asynchronous on `stream`. */
size_t ivc_router_fold_size(const ivc_router* r);
int ivc_router_fold(ivc_router* r, void* dst, size_t dst_bytes, ivc_stream_t stream);

/* pixel_shuffle + connector MLP ([PS] "extract_feature() 完整调用链" steps 5-8;
 * [DP] table "三档 Token 规模").
 *   x      device bf16 [T, 32, 32, C]: ViT features, CLS dropped.
 *   scale  0.5 (256 tokens of 4C per tile; m->dims[0] must be 4C) or
 *          0.25 (64 tokens of 16C; m->dims[0] must be 16C).
 *   flags  IVC_PS_* bits.
 *   y      device bf16 [T * tokens, m->dims[n_linear]]; token order within a
 *          tile is row-major over the output grid (transposed for IVC_PS_V1).
 * Unsupported (IVC_EUNSUPPORTED): C % 64 != 0, any Linear width % 64 != 0,
 * n_linear not 2 or 3. T == 0 enqueues nothing. */
int ivc_ps_project(const void* x, int T, int C, float scale, int flags, const ivc_mlp* m,
                   void* y, void* workspace, size_t ws_bytes, ivc_stream_t stream);

/* ViR routing ([VIR] sections 2-4).
 *   x              device bf16 [T, 32, 32, D] (tokens row-major over the grid).
 *   valid_len      device int32 [T] (tokens t >= valid_len are padding), or
 *                  NULL for all 1024; values outside [1,1024] set
 *                  IVC_DEV_BAD_VALID_LEN.
 *   image_offsets  device int32 [I+1], 0 = o_0 <= ... <= o_I = T; image i owns
 *                  tiles [o_i, o_{i+1}). Ignored for quantile_scope 1.
 *   gate           device fp32 [T, 2] softmax probabilities; column 0 means
 *                  "compress to 64 tokens".
 *   mask           device uint8 [T]: 1 = compressed (64 rows), 0 = 256 rows.
 *   offsets        device int32 [T+1]: exclusive scan of the row counts;
 *                  offsets[T] = total rows = 256 (T - k) + 64 k.
 * rel_q outside [0, 1] (or NaN) is IVC_EINVAL.
 * Unsupported: D != C, D % 256 != 0, heads * 64 != D, gate_hidden % 256 != 0.
 * The router runs as a chain of kernels overlapped by programmatic dependent
 * launch. With folded pooling, D <= 1024 and at most 16 heads, the
 * environment variable IVC_ROUTER_FUSED=1 selects instead one cooperative
 * persistent kernel that holds every SM until it ends. */
int ivc_vir_route(const void* x, const int32_t* valid_len, int T, int C,
                  const int32_t* image_offsets, int I, const ivc_router* r, float* gate,
                  uint8_t* mask, int32_t* offsets, void* workspace, size_t ws_bytes,
                  ivc_stream_t stream);

/* Routing alone ([VIR] section 4; [DP] "路由决策：相对 + 绝对双阈值判定"): the
 * double threshold and the row-count scan that end ivc_vir_route, applied to
 * a gate vector the caller supplies (for instance gates computed by another
 * implementation of the router). Tile t is compressed iff
 * gate[t,0] > quantile(gate[.,0] over its group, rel_q) and gate[t,0] >= abs_t,
 * the quantile by linear interpolation in fp64, each operation rounded on its
 * own. As with torch.quantile, a NaN gate makes its group's quantile NaN, so
 * no tile of that group is compressed.
 *   gate           device fp32 [T, 2]; only column 0 is read.
 *   image_offsets  device int32 [I+1] as in ivc_vir_route (scope 0); may be
 *                  NULL for scope 1 (one group: the whole batch).
 *   rel_q          in [0, 1], else IVC_EINVAL; abs_t any value.
 *   mask, offsets  as in ivc_vir_route; total: device int32 [1] or NULL.
 *   workspace      >= IVC_ROUTE_WORKSPACE_BYTES (the device status word),
 *                  256-byte aligned. Bad image offsets set IVC_DEV_BAD_OFFSETS
 *                  (nothing compressed); a group above IVC_MAX_QUANTILE_GROUP
 *                  tiles sets IVC_DEV_GROUP_TOO_LARGE (that group uncompressed).
 * One CTA; T == 0 writes offsets[0] = 0 (and *total = 0). */
#define IVC_ROUTE_WORKSPACE_BYTES 256u
int ivc_route(const float* gate, int T, const int32_t* image_offsets, int I, double rel_q,
              double abs_t, int scope, uint8_t* mask, int32_t* offsets, int32_t* total,
              void* workspace, size_t ws_bytes, ivc_stream_t stream);

/* The Flash dual path ([DP] "双路压缩管线全流程拆解"; [VIR] section 5):
 * ivc_ps_project at 0.5 with mlp1 and at 0.25 with mlp2, ivc_vir_route, then
 * compaction: out rows [offsets[t], offsets[t+1]) = the 64 mlp2 rows of tile t
 * if mask[t] else its 256 mlp1 rows, tiles in order.
 *   out    device bf16 [T * 256, H] capacity (H = output width of both MLPs).
 *   total  device int32 [1]: rows written (= offsets[T]).
 * gate, mask, offsets as in ivc_vir_route.
 * The router part runs on a library-owned high-priority stream of the current
 * device (created on the first call, with two events), forked from and joined
 * back into `stream`: to the caller the call is ordered on `stream` alone. */
int ivc_flash_compress(const void* x, const int32_t* valid_len, int T, int C,
                       const int32_t* image_offsets, int I, const ivc_mlp* mlp1,
                       const ivc_mlp* mlp2, const ivc_router* r, void* out, float* gate,
                       uint8_t* mask, int32_t* offsets, int32_t* total, void* workspace,
                       size_t ws_bytes, ivc_stream_t stream);

/* The Flash dual path computed router-first: ivc_vir_route, then each tile
 * only through the path it was routed to (mlp2 at 0.25 for mask[t] = 1, mlp1
 * at 0.5 otherwise), the last Linear of each MLP storing the tile's rows
 * straight at out rows [offsets[t], offsets[t+1]). The pages compute both
 * paths for every tile and then keep one ([DP] "双路压缩管线全流程拆解");
 * the kept rows are the same, the discarded path is never computed.
 * Arguments, results, workspace size (IVC_OP_FLASH_COMPRESS) and errors are
 * those of ivc_flash_compress; every step runs on `stream`, and the router
 * runs as in ivc_vir_route. */
int ivc_flash_compress_routed(const void* x, const int32_t* valid_len, int T, int C,
                              const int32_t* image_offsets, int I, const ivc_mlp* mlp1,
                              const ivc_mlp* mlp2, const ivc_router* r, void* out, float* gate,
                              uint8_t* mask, int32_t* offsets, int32_t* total, void* workspace,
                              size_t ws_bytes, ivc_stream_t stream);

/* Sequence assembly: the compacted visual rows spliced into the token
 * sequences ([PS] "视觉 Token 如何注入 Qwen2.5 语言模型": the prompt's
 * <IMG_CONTEXT> positions take the visual rows in order; [VIR] section 4 and
 * [DP] "路由决策": a compressed tile keeps 64 of its 256 placeholders, the
 * other 192 are deleted and the position indices follow).
 *   input_ids       device int32 [L]: B sequences back to back.
 *   seq_offsets     device int32 [B+1]: 0 = s_0 <= ... <= s_B = L.
 *   img_context_id  the <IMG_CONTEXT> token id. The j-th placeholder of the
 *                   batch is placeholder j % 256 of tile j / 256; a batch
 *                   must hold exactly 256 T of them (else IVC_DEV_BAD_PROMPT,
 *                   and placeholders beyond 256 T are treated as text).
 *   embed_table     device bf16 [V, H]: the language model's token embeddings.
 *   visual          device bf16 [offsets[T], H]: rows of ivc_flash_compress.
 *   mask, offsets   device uint8 [T], int32 [T+1] of ivc_flash_compress.
 *   out_ids         device int32 [L] capacity: the kept token ids.
 *   out_embeds      device bf16 [L, H] capacity: row i = visual row of a kept
 *                   placeholder, else embed_table[out_ids[i]] (a zero row and
 *                   IVC_DEV_BAD_PROMPT for an id outside [0, V)).
 *   out_positions   device int32 [L] capacity: position of row i within its
 *                   sequence (0, 1, ...).
 *   out_seq_offsets device int32 [B+1]: the shortened sequences; the total
 *                   row count L - 192 k is out_seq_offsets[B].
 *   workspace       >= ivc_assemble_workspace_size(L) bytes, status word first.
 * H must be a multiple of 8; pointers to bf16 rows 16-byte aligned. */
size_t ivc_assemble_workspace_size(int L);
int ivc_assemble_sequence(const int32_t* input_ids, const int32_t* seq_offsets, int B, int L,
                          int32_t img_context_id, const void* embed_table, int V, int H,
                          const void* visual, const uint8_t* mask, const int32_t* offsets, int T,
                          int32_t* out_ids, void* out_embeds, int32_t* out_positions,
                          int32_t* out_seq_offsets, void* workspace, size_t ws_bytes,
                          ivc_stream_t stream);

/* Synchronise `stream`, copy the workspace's device status word to *bits and
 * clear it. Returns IVC_OK when no bit was set, IVC_EDEVICE otherwise. */
int ivc_device_status(void* workspace, int* bits, ivc_stream_t stream);

/* Failure detection (diagnostics). Every wait inside the kernels is bounded
 * (about one second of clock cycles): a wait that runs out sets
 * IVC_DEV_WAIT_TIMEOUT in the status word, the kernel skips its remaining
 * work, lets the copies it issued land, and returns; no trap is used and the
 * context stays usable. To exercise that path, `cycles` > 0 makes the
 * persistent router (ivc_vir_route's single-kernel form, IVC_ROUTER_FUSED=1) give up its
 * software grid barriers from the one before the gating head on after that
 * many clock cycles; no bulk copy is in flight at those barriers. With a
 * limit of a few cycles the call's outputs are invalid and the status bit is
 * set. 0 restores the default bound; negative values are IVC_EINVAL.
 * Process-wide, read at each launch. */
int ivc_set_router_wait_limit(long long cycles);

/* ivc_ps_project for callers that cannot allocate device memory.
 * No counterpart on the pages: this is a deployment variant of the call above.
 * Callers such as an inference-engine plugin whose device memory is planned
 * ahead, or a latency-critical loop that cannot afford the synchronisation an
 * allocation may cause, cannot call cudaMalloc to create a workspace. This
 * entry point instead uses a fixed scratch array of IVC_NOALLOC_SCRATCH_BYTES
 * that the library holds in device memory on every GPU that loads it, until
 * the process exits. It allocates nothing itself.
 *   Arguments and results are those of ivc_ps_project, without the workspace.
 *   `m` must already be folded (ivc_mlp_fold); otherwise IVC_EINVAL.
 *   Calls needing more scratch than IVC_NOALLOC_SCRATCH_BYTES (the
 *   ivc_workspace_size of the same op) return IVC_EWORKSPACE and enqueue
 *   nothing: e.g. up to 15 tiles of mlp1 4096->2048->2048 fit.
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture. The
 *   address is looked up again when the device's current context changes
 *   (e.g. after cudaDeviceReset); the first call after such a change must
 *   also come before any capture.
 *   All calls share the one array and it keeps the last call's contents:
 *   calls whose GPU work can overlap (other streams, other host threads on
 *   the same device) race on it. The device status word inside the array is
 *   cleared at the start of every call and cannot be read by the caller. */
#define IVC_NOALLOC_SCRATCH_BYTES (16u << 20)
int ivc_ps_project_noalloc(const void* x, int T, int C, float scale, int flags,
                           const ivc_mlp* m, void* y, ivc_stream_t stream);

/* Per-kernel device timing (diagnostics; off by default). While enabled,
 * every kernel launch is bracketed by two CUDA events on its stream and filed
 * under its role (e.g. "mlp1.fc1", "pool.kv", "pool.attention", "route").
 * ivc_trace_report() waits for the recorded events and writes a JSON object
 * {role: {"launches": n, "ms": total}} into buf (n bytes); IVC_EINVAL if buf
 * is too small. ivc_trace_reset() forgets the records. Not for use while a
 * stream is being captured into a CUDA graph. */
int ivc_trace_enable(int on);
int ivc_trace_reset(void);
int ivc_trace_report(char* buf, size_t n);

#ifdef __cplusplus
}
#endif
#endif /* IVC_H_ */
