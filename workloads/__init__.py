"""Seeded synthetic inputs for the InternVL visual-token compression path.

This module only draws numbers. It holds none of the method's arithmetic
(no pixel_shuffle, no LayerNorm, no matmul, no softmax, no routing): both the
fp64 oracle (``oracle/``) and the CUDA library (``vlm_visual_token_b200``)
receive the very same bf16 tensors from here, so neither side can leak into
the other through its inputs.

Shapes and distributions follow the workloads the pages describe:

* ViT output of one 448x448 tile, CLS dropped and reshaped to a 32x32 grid of
  C-wide features (InternVL3-14B-Instruct Pixel Shuffle + MLP article,
  section "extract_feature() 完整调用链", steps 3-5); C = 1024 for
  InternViT-300M, 3200 for InternViT-6B (InternVL3-38B-Instruct InternViT
  article, section 2).
* 1..12 tiles plus a thumbnail per image (InternVL3_5-2B-Flash dual-path
  article, section "为什么必须压缩").
* Variable-length tiles carry a padding mask; valid tokens form a prefix and
  pad rows are zero (InternVL3_5-4B-Flash Gating/CrossAttentionPooling
  article, section 2).

Features are ~N(0,1); weights ~N(0,0.02); biases 0; LayerNorm gamma=1,
beta=0; the pooling query ~N(0,1). ``affine="random"`` replaces the zero
biases and unit/zero LayerNorm parameters by random ones so that tests catch
a dropped bias or LayerNorm term. Every tensor is drawn in fp32 from a
``torch.Generator`` on the CPU and rounded to bf16 once.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

GRID = 32           # 448 / 14 patches per side
TOKENS = GRID * GRID  # 1024 ViT tokens per tile
POOL_HEADS = 16
POOL_LAYERS = 4
GATE_BLOCKS = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark/parity configuration (dimensions only)."""
    name: str
    path: str                 # "ps_project" (mlp1 only) or "flash" (dual path + router)
    C: int                    # ViT width
    H: int                    # LLM hidden (connector output width)
    tiles_per_image: tuple    # fixed per-image tile counts, or () when drawn
    n_images: int
    mlp2_mid: int = 4096      # mlp2 intermediate width
    D: int = 1024             # pooling width (= C of InternViT-300M)
    gate_hidden: int = 1024   # gating MLP inner width
    var_len_frac: float = 0.0  # fraction of tiles with a padding mask
    var_len_lo: int = 256
    var_len_hi: int = 1024
    draw_tiles: bool = False  # tiles per image ~ U{1..13}
    seed_base: int = 0        # the configuration number, added to the seeds


WORKLOADS: Dict[str, Workload] = {
    # InternVL3.5-2B dims, one tile through ps 0.5 + mlp1 4096->2048->2048.
    "single_tile_2b": Workload("single_tile_2b", "ps_project", C=1024, H=2048,
                               tiles_per_image=(1,), n_images=1, seed_base=1),
    # InternVL3.5-2B-Flash: one image of 12 tiles + thumbnail, both paths + ViR.
    "flash_2b_13tiles": Workload("flash_2b_13tiles", "flash", C=1024, H=2048,
                                 tiles_per_image=(13,), n_images=1, seed_base=2),
    # InternVL3.5-4B-Flash: 16 images x U{1..13} tiles, 10% variable length.
    "flash_4b_batched": Workload("flash_4b_batched", "flash", C=1024, H=2560,
                                 tiles_per_image=(), n_images=16, draw_tiles=True,
                                 var_len_frac=0.10, seed_base=3),
    # InternVL3-14B connector: 64 images x 13 tiles, mlp1 4096->5120->5120.
    "connector_14b_832tiles": Workload("connector_14b_832tiles", "ps_project", C=1024,
                                       H=5120, tiles_per_image=(13,) * 64, n_images=64,
                                       seed_base=4),
    # InternVL3-38B connector (InternViT-6B, C=3200): 32 images x 13 tiles.
    "connector_38b_416tiles": Workload("connector_38b_416tiles", "ps_project", C=3200,
                                       H=5120, tiles_per_image=(13,) * 32, n_images=32,
                                       seed_base=5),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def _bias(g, n, affine, std=0.02):
    if affine == "random":
        return _randn(g, (n,), std)
    return torch.zeros(n, dtype=torch.bfloat16)


def _ln(g, n, affine):
    if affine == "random":
        gamma = (1.0 + torch.randn(n, generator=g) * 0.1).to(torch.bfloat16)
        beta = _randn(g, (n,), 0.1)
        return gamma, beta
    return torch.ones(n, dtype=torch.bfloat16), torch.zeros(n, dtype=torch.bfloat16)


def layout(w: Workload, seed: Optional[int] = None, n_images: Optional[int] = None):
    """Per-image tile counts and per-tile valid lengths.

    Returns (image_offsets int32 [I+1], valid_len int32 [T]).
    """
    g = _gen(777 + w.seed_base if seed is None else seed)
    I = w.n_images if n_images is None else n_images
    if w.draw_tiles:
        counts = torch.randint(1, 14, (I,), generator=g).tolist()
    else:
        counts = list(w.tiles_per_image)[:I]
        if len(counts) < I:
            counts = counts + [counts[-1]] * (I - len(counts))
    offs = [0]
    for c in counts:
        offs.append(offs[-1] + c)
    T = offs[-1]
    valid = torch.full((T,), TOKENS, dtype=torch.int32)
    if w.var_len_frac > 0 and T > 0:
        pick = torch.rand(T, generator=g) < w.var_len_frac
        lens = torch.randint(w.var_len_lo, w.var_len_hi + 1, (T,), generator=g, dtype=torch.int32)
        valid = torch.where(pick, lens, valid)
    return torch.tensor(offs, dtype=torch.int32), valid


def features(T: int, C: int, seed: int, valid_len: Optional[torch.Tensor] = None) -> torch.Tensor:
    """ViT features [T, 32, 32, C] bf16 ~N(0,1); rows past valid_len are zero."""
    g = _gen(seed)
    x = _randn(g, (T, GRID, GRID, C))
    if valid_len is not None:
        idx = torch.arange(TOKENS).view(1, GRID, GRID)
        pad = idx >= valid_len.view(-1, 1, 1).to(torch.int64)
        x[pad] = 0
    return x


def mlp_params(dims: List[int], seed: int, affine: str = "config") -> dict:
    """LayerNorm(dims[0]) then Linear layers dims[i] -> dims[i+1] (nn.Linear [out,in])."""
    g = _gen(seed)
    gamma, beta = _ln(g, dims[0], affine)
    Ws, bs = [], []
    for i in range(len(dims) - 1):
        Ws.append(_randn(g, (dims[i + 1], dims[i]), 0.02))
        bs.append(_bias(g, dims[i + 1], affine))
    return {"dims": list(dims), "ln_g": gamma, "ln_b": beta, "W": Ws, "b": bs}


def router_params(D: int, gate_hidden: int, seed: int, affine: str = "config",
                  heads: int = POOL_HEADS) -> dict:
    """CrossAttentionPooling (query + 4 attention layers) and Gating weights."""
    g = _gen(seed)
    p = {"D": D, "heads": heads, "query": _randn(g, (D,), 1.0)}
    for name in ("Wq", "Wk", "Wv", "Wo"):
        p[name] = []
    for name in ("bq", "bk", "bv", "bo"):
        p[name] = []
    for _ in range(POOL_LAYERS):
        for W, b in (("Wq", "bq"), ("Wk", "bk"), ("Wv", "bv"), ("Wo", "bo")):
            p[W].append(_randn(g, (D, D), 0.02))
            p[b].append(_bias(g, D, affine))
    for name in ("gW1", "gb1", "gW2", "gb2", "gln_g", "gln_b"):
        p[name] = []
    for _ in range(GATE_BLOCKS):
        p["gW1"].append(_randn(g, (gate_hidden, D), 0.02))
        p["gb1"].append(_bias(g, gate_hidden, affine))
        p["gW2"].append(_randn(g, (D, gate_hidden), 0.02))
        p["gb2"].append(_bias(g, D, affine))
        lg, lb = _ln(g, D, affine)
        p["gln_g"].append(lg)
        p["gln_b"].append(lb)
    p["gWout"] = _randn(g, (2, D), 0.02)
    p["gbout"] = _bias(g, 2, affine)
    return p


def make(name_or_w, affine: str = "config", n_images: Optional[int] = None,
         seed_offset: int = 0) -> dict:
    """All inputs of one workload. ``n_images`` truncates the image list (samples)."""
    w = WORKLOADS[name_or_w] if isinstance(name_or_w, str) else name_or_w
    offs, valid = layout(w, seed=777 + w.seed_base + seed_offset, n_images=n_images)
    T = int(offs[-1])
    x = features(T, w.C, 1234 + w.seed_base + seed_offset, valid if w.var_len_frac > 0 else None)
    wseed = 4321 + w.seed_base + seed_offset
    out = {"workload": w, "T": T, "C": w.C, "H": w.H, "x": x, "valid_len": valid,
           "image_offsets": offs,
           "mlp1": mlp_params([4 * w.C, w.H, w.H], wseed, affine)}
    if w.path == "flash":
        out["mlp2"] = mlp_params([16 * w.C, w.mlp2_mid, w.H, w.H], wseed + 1000, affine)
        out["router"] = router_params(w.D, w.gate_hidden, wseed + 2000, affine,
                                      heads=w.D // 64)
    return out
