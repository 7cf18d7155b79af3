"""fp64 CPU oracle for InternVL's visual-token compression connector and the
Flash Visual Resolution Router (ViR).

TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and
its Python binding) imports, calls or links this module; only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it.

Every function below is the plain definition of one step, written in numpy
float64 with no blocking, fusion or reordering beyond what the step states. A
matrix product (``@``, i.e. BLAS dgemm) and ``scipy.special.erf`` serve as
library primitives. Inputs are the bf16 tensors of ``workloads`` widened to
float64; intermediates are never rounded.

Sources (pages, by title and section):

* [PS]   InternVL3-14B-Instruct "Pixel Shuffle + MLP connector, line by line"
         (zwxr.cn/news/271642): "Pixel Shuffle 源码逐行解析" (pixel_shuffle and
         its three view/permute steps), "ps_version v1 与 v2", "MLP 连接器源码逐行解析"
         (mlp1 = LayerNorm -> Linear -> GELU -> Linear), "extract_feature() 完整调用链".
* [DP]   InternVL3_5-2B-Flash "1024->256->64 dual-path compression pipeline"
         (kwkr.cn/news/620108): table "三档 Token 规模" (factor 0.25 = 0.5^2,
         16C channels, mlp2 with intermediate 4096), "路由决策：相对 + 绝对双阈值判定".
* [VIR]  InternVL3_5-4B-Flash "Gating and CrossAttentionPooling"
         (mrgr.cn/news/14598): section 2 (CrossAttentionPooling: learnable
         query, 4 multi-head cross-attention layers, padding mask), section 3
         (Gating: 4 residual blocks Linear->GELU->Dropout->Linear->Dropout->
         LayerNorm, Linear(hidden,2) + softmax), section 4 (quantile and
         absolute thresholds), section 5 (data flow, splice back into the sequence).

Readings where the pages are silent or garbled (each also listed in the design
notes): one pixel_shuffle call at factor 0.25 for the 64-token path (the
two-call order is a flag); mlp2 = LN -> L -> GELU -> L -> GELU -> L; LayerNorm
eps 1e-5 with biased variance, exact erf GELU; pooling layers are independent
MHA layers with their own Q/K/V/out projections and biases, 16 heads, scale
1/sqrt(64), no residual and no norm between layers, q_l feeds layer l+1; pad
tokens are a suffix and are excluded from the softmax; gating residual wraps
the listed block (h <- h + LN(block(h))), dropout is identity at inference;
quantile by linear interpolation in fp64, per image; gate column 0 means
"compress to 64"; compaction keeps images, tiles and tokens in order;
sequence assembly: the k-th run of 256 placeholders is tile k, a compressed
tile keeps its first 64, positions count the kept tokens per sequence.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np
from scipy.special import erf as _erf

LN_EPS = 1e-5


# ----------------------------------------------------------------------------
# pixel_shuffle  ([PS] "Pixel Shuffle 源码逐行解析"; [DP] table "三档 Token 规模")
# ----------------------------------------------------------------------------
def pixel_shuffle(x: np.ndarray, scale: float, ps_version: str = "v2") -> np.ndarray:
    """Space-to-depth of a [T, G, G, C] grid by factor f = 1/scale.

    Output grid cell (a, b) gathers the f x f block of input cells
    (f*a + di, f*b + dj), di, dj in [0, f); channel block di*f + dj holds input
    cell (f*a+di, f*b+dj). Output tokens are numbered row-major over the
    (G/f) x (G/f) grid: token a*(G/f) + b. This is what the page's
    view -> permute -> view -> permute sequence computes (the first view merges
    f neighbours along the second grid axis into channels, the second view
    merges f neighbours along the first axis in front of them).

    ps_version "v1" omits the final axis swap, so the output grid comes out
    transposed: token b*(G/f) + a holds cell (a, b).

    Returns [T, (G/f)^2, f*f*C].
    """
    T, G, G2, C = x.shape
    assert G == G2
    f = int(round(1.0 / scale))
    assert abs(f * scale - 1.0) < 1e-12 and G % f == 0
    g = G // f
    out = np.empty((T, g * g, f * f * C), dtype=x.dtype)
    for a in range(g):
        for b in range(g):
            tok = a * g + b if ps_version == "v2" else b * g + a
            for di in range(f):
                for dj in range(f):
                    blk = di * f + dj
                    out[:, tok, blk * C:(blk + 1) * C] = x[:, f * a + di, f * b + dj, :]
    return out


def pixel_shuffle_grid(x: np.ndarray, scale: float, ps_version: str = "v2") -> np.ndarray:
    """pixel_shuffle returning the [T, G/f, G/f, f*f*C] grid (for chaining)."""
    T, G, _, C = x.shape
    f = int(round(1.0 / scale))
    return pixel_shuffle(x, scale, ps_version).reshape(T, G // f, G // f, f * f * C)


def pixel_shuffle_quarter(x: np.ndarray, order: str = "single") -> np.ndarray:
    """The 64-token representation of [DP].

    order "single": one pixel_shuffle call at factor 0.25 (the reading taken).
    order "twice":  pixel_shuffle(pixel_shuffle(x, 0.5), 0.5), the page's
                    "equivalent to two pixel_shuffle" remark; same tokens,
                    channels permuted differently.
    """
    if order == "single":
        return pixel_shuffle(x, 0.25)
    once = pixel_shuffle_grid(x, 0.5)
    return pixel_shuffle(once, 0.5)


# ----------------------------------------------------------------------------
# LayerNorm / GELU / Linear / MLP  ([PS] "MLP 连接器源码逐行解析"; [DP])
# ----------------------------------------------------------------------------
def layer_norm(v: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """Normalise the last axis: (v - mean) / sqrt(biased var + eps) * gamma + beta."""
    mu = v.mean(axis=-1, keepdims=True)
    var = ((v - mu) ** 2).mean(axis=-1, keepdims=True)
    return (v - mu) / np.sqrt(var + eps) * gamma + beta


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU: z * Phi(z) = z/2 * (1 + erf(z / sqrt 2))."""
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def linear(v: np.ndarray, W: np.ndarray, b: np.ndarray) -> np.ndarray:
    """nn.Linear with weight [out, in]: v @ W^T + b."""
    return v @ W.T + b


def mlp(P: np.ndarray, ln_g, ln_b, Ws: Sequence[np.ndarray], bs: Sequence[np.ndarray]) -> np.ndarray:
    """LayerNorm, then the Linear layers with GELU between consecutive ones.

    Two layers: mlp1 = LN -> Linear -> GELU -> Linear ([PS]).
    Three layers: mlp2 = LN -> Linear -> GELU -> Linear -> GELU -> Linear ([DP]).
    """
    h = layer_norm(P, ln_g, ln_b)
    for i, (W, b) in enumerate(zip(Ws, bs)):
        h = linear(h, W, b)
        if i + 1 < len(Ws):
            h = gelu(h)
    return h


def ps_project(x: np.ndarray, scale: float, params: dict, ps_version: str = "v2",
               quarter_order: str = "single") -> np.ndarray:
    """pixel_shuffle at `scale` then the MLP; returns [T, tokens, H]."""
    if scale == 0.5:
        P = pixel_shuffle(x, 0.5, ps_version)
    else:
        P = pixel_shuffle_quarter(x, quarter_order)
    T, n, K = P.shape
    Y = mlp(P.reshape(T * n, K), params["ln_g"], params["ln_b"], params["W"], params["b"])
    return Y.reshape(T, n, -1)


# ----------------------------------------------------------------------------
# CrossAttentionPooling  ([VIR] section 2)
# ----------------------------------------------------------------------------
def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = s.max(axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=axis, keepdims=True)


def cross_attention_pooling(X: np.ndarray, valid_len: np.ndarray, r: dict) -> np.ndarray:
    """Pool each tile's tokens into one D-vector with a learnable query.

    X [T, N, D] (N = 1024 raw ViT tokens per tile, row-major over the grid),
    valid_len [T] (tokens t >= valid_len[tile] are padding and get no weight).
    Layer l (l = 1..4): Q = Wq_l q + bq_l; K = X Wk_l^T + bk_l; V = X Wv_l^T + bv_l;
    per head h (head width D/heads): weights = softmax over valid tokens of
    (Q_h . K_h[t]) / sqrt(D/heads); o_h = sum_t weights_t V_h[t];
    q <- Wo_l o + bo_l. q starts as the query token; the output is q after layer 4.
    """
    T, N, D = X.shape
    H = int(r["heads"])
    dh = D // H
    q = np.broadcast_to(r["query"], (T, D)).copy()
    for l in range(len(r["Wq"])):
        Q = linear(q, r["Wq"][l], r["bq"][l])                 # [T, D]
        K = linear(X, r["Wk"][l], r["bk"][l])                 # [T, N, D]
        V = linear(X, r["Wv"][l], r["bv"][l])                 # [T, N, D]
        o = np.zeros((T, D))
        for t in range(T):
            n = int(valid_len[t])
            for h in range(H):
                sl = slice(h * dh, (h + 1) * dh)
                s = K[t, :n, sl] @ Q[t, sl] / math.sqrt(dh)   # [n]
                p = softmax(s)
                o[t, sl] = p @ V[t, :n, sl]
        q = linear(o, r["Wo"][l], r["bo"][l])
    return q


# ----------------------------------------------------------------------------
# Gating  ([VIR] section 3)
# ----------------------------------------------------------------------------
def gating(pooled: np.ndarray, r: dict, residual: str = "outside") -> np.ndarray:
    """Four residual MLP blocks, then Linear(hidden, 2) and a 2-way softmax.

    Block b: u = W2_b GELU(W1_b h + b1_b) + b2_b (dropout is the identity at
    inference). residual "outside": h <- h + LN_b(u) (the reading taken);
    "inside": h <- LN_b(h + u). Returns probabilities [T, 2].
    """
    h = pooled
    for b in range(len(r["gW1"])):
        u = linear(gelu(linear(h, r["gW1"][b], r["gb1"][b])), r["gW2"][b], r["gb2"][b])
        if residual == "outside":
            h = h + layer_norm(u, r["gln_g"][b], r["gln_b"][b])
        else:
            h = layer_norm(h + u, r["gln_g"][b], r["gln_b"][b])
    logits = linear(h, r["gWout"], r["gbout"])
    return softmax(logits, axis=-1)


# ----------------------------------------------------------------------------
# Quantile, double threshold, offsets, compaction  ([VIR] section 4; [DP])
# ----------------------------------------------------------------------------
def quantile_linear(values: np.ndarray, q: float) -> float:
    """Linear-interpolation quantile: sort ascending, pos = q (n - 1),
    lo = floor(pos), hi = ceil(pos), result = v[lo] + (pos - lo) (v[hi] - v[lo]).
    Evaluated in fp64 with each operation rounded separately.

    The threshold of [VIR] section 4 is torch.quantile's, which is NaN as soon
    as one input is NaN (NaN inputs are not skipped); every comparison with a
    NaN threshold is false, so no tile of that group is compressed."""
    v = np.sort(np.asarray(values, dtype=np.float64))
    if np.isnan(v).any():
        return float("nan")
    n = v.shape[0]
    pos = float(q) * float(n - 1)
    lo = int(math.floor(pos))
    hi = int(math.ceil(pos))
    w = pos - lo
    diff = float(v[hi]) - float(v[lo])
    return float(v[lo]) + w * diff


def route(gate0: np.ndarray, image_offsets: np.ndarray, rel_q: float = 0.1,
          abs_t: float = 0.5, scope: str = "image") -> np.ndarray:
    """Compress tile t (to 64 tokens) iff gate0[t] > quantile(gate0 over its
    image, rel_q) and gate0[t] >= abs_t. scope "batch" takes the quantile over
    all tiles at once. Returns uint8 mask [T]."""
    g = np.asarray(gate0, dtype=np.float64)
    T = g.shape[0]
    mask = np.zeros(T, dtype=np.uint8)
    if scope == "batch":
        groups = [(0, T)] if T > 0 else []
    else:
        offs = [int(v) for v in image_offsets]
        groups = [(offs[i], offs[i + 1]) for i in range(len(offs) - 1) if offs[i + 1] > offs[i]]
    for s, e in groups:
        qv = quantile_linear(g[s:e], rel_q)
        for t in range(s, e):
            mask[t] = 1 if (g[t] > qv and g[t] >= abs_t) else 0
    return mask


def compaction_offsets(mask: np.ndarray, full: int = 256, compressed: int = 64) -> np.ndarray:
    """Row offset of each tile in the compacted output; last entry = total rows."""
    counts = np.where(np.asarray(mask) != 0, compressed, full).astype(np.int64)
    offs = np.zeros(counts.shape[0] + 1, dtype=np.int64)
    for t in range(counts.shape[0]):
        offs[t + 1] = offs[t] + counts[t]
    return offs.astype(np.int32)


def compact(Y256: np.ndarray, Y64: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Concatenate, tile by tile, Y64[t] (mask 1) or Y256[t] (mask 0)."""
    parts = [Y64[t] if mask[t] else Y256[t] for t in range(len(mask))]
    if not parts:
        return np.zeros((0, Y256.shape[-1]))
    return np.concatenate(parts, axis=0)


# ----------------------------------------------------------------------------
# Sequence assembly  ([VIR] section 4, compress_visual_tokens_in_sentence:
# a compressed tile keeps 64 of its 256 <IMG_CONTEXT> positions and 192 are
# deleted, the position indices following; [PS] "视觉 Token 如何注入": the
# embedded prompt's <IMG_CONTEXT> positions take the visual rows in order)
# ----------------------------------------------------------------------------
def assemble_sequence(input_ids, seq_offsets, img_context_id: int, embed_table: np.ndarray,
                      visual: np.ndarray, mask, offsets, keep: int = 64,
                      full: int = 256) -> Dict[str, np.ndarray]:
    """Splice the compacted visual rows into a batch of token sequences.

    The j-th <IMG_CONTEXT> placeholder of the batch (sequence order) is
    placeholder r = j % full of tile t = j // full. For a compressed tile
    (mask[t] = 1) placeholders r >= keep are deleted; a kept placeholder takes
    visual row offsets[t] + r; every other token takes its row of the
    embedding table. Position ids count the kept tokens from 0 in each
    sequence. Placeholders beyond full * T (a prompt with more than T tiles)
    are treated as text tokens. Returns ids, embeds, positions, the new
    sequence offsets and the number of placeholders seen."""
    ids = np.asarray(input_ids)
    T = len(mask)
    out_ids: List[int] = []
    rows: List[np.ndarray] = []
    pos: List[int] = []
    new_offs = [0]
    j = 0
    for b in range(len(seq_offsets) - 1):
        start = len(out_ids)
        for p in range(int(seq_offsets[b]), int(seq_offsets[b + 1])):
            tok = int(ids[p])
            if tok == img_context_id:
                jj = j
                j += 1
                if jj < full * T:
                    t, r = divmod(jj, full)
                    if mask[t] and r >= keep:
                        continue  # one of the deleted placeholders
                    out_ids.append(tok)
                    rows.append(visual[int(offsets[t]) + r])
                    pos.append(len(out_ids) - 1 - start)
                    continue
            out_ids.append(tok)
            rows.append(embed_table[tok])
            pos.append(len(out_ids) - 1 - start)
        new_offs.append(len(out_ids))
    H = embed_table.shape[1]
    return {"ids": np.array(out_ids, dtype=np.int64),
            "embeds": np.array(rows).reshape(-1, H),
            "positions": np.array(pos, dtype=np.int64),
            "seq_offsets": np.array(new_offs, dtype=np.int64),
            "placeholders": j}


# ----------------------------------------------------------------------------
# Whole path
# ----------------------------------------------------------------------------
def vir_gate(x: np.ndarray, valid_len: np.ndarray, r: dict, residual: str = "outside") -> np.ndarray:
    """Gate probabilities [T, 2] of the router for features x [T, 32, 32, D]."""
    T, G, _, D = x.shape
    pooled = cross_attention_pooling(x.reshape(T, G * G, D), valid_len, r)
    return gating(pooled, r, residual)


def flash_compress(x, valid_len, image_offsets, mlp1, mlp2, r, rel_q=0.1, abs_t=0.5,
                   gate_override: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Dual path (ps 0.5 -> mlp1, ps 0.25 -> mlp2), router, routing, compaction.

    gate_override: route on a given fp32 gate vector instead of the oracle's
    own (the comparison "given the same gate vector").
    """
    Y256 = ps_project(x, 0.5, mlp1)
    Y64 = ps_project(x, 0.25, mlp2)
    gate = vir_gate(x, valid_len, r)
    g0 = gate[:, 0] if gate_override is None else np.asarray(gate_override, np.float64)
    mask = route(g0, image_offsets, rel_q, abs_t)
    offs = compaction_offsets(mask)
    out = compact(Y256, Y64, mask)
    return {"Y256": Y256, "Y64": Y64, "gate": gate, "mask": mask, "offsets": offs, "out": out}

