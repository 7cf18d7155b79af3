"""GPU (libivc.so through its C ABI) against the fp64 oracle on the same
seeded bf16 inputs.

Bars: pixel_shuffle, the routing mask and the compaction offsets bit-exact
(the mask given the same fp32 gate vector), gate probabilities within 1e-3
absolute, connector outputs within relative Frobenius 1e-2 and max-abs 3e-2
(plus half a bf16 ulp where |y| >= 4, see tests/_parity.py).
"""
import dataclasses
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests._parity import GATE_ABS, assert_connector_close, connector_errors, to_np

pytestmark = pytest.mark.gpu


def _ivc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import vlm_visual_token_b200 as ivc
    return ivc


def small_workload(C=128, H=192, mid=320, tiles=(3, 4), var=0.0, gate_hidden=256, name="small"):
    return W.Workload(name, "flash", C=C, H=H, tiles_per_image=tuple(tiles), n_images=len(tiles),
                      mlp2_mid=mid, D=C, gate_hidden=gate_hidden, var_len_frac=var,
                      seed_base=90)


# ------------------------------------------------------------------ connector
@pytest.mark.parametrize("flags", [0, 1])
def test_ps_project_half_small_ragged(flags):
    ivc = _ivc()
    inp = W.make(small_workload(C=128, H=192), affine="random")
    x = inp["x"].cuda()
    m = ivc.Mlp(inp["mlp1"])
    y = ivc.ps_project(x, 0.5, m, flags=flags)
    torch.cuda.synchronize()
    ref = O.ps_project(O.to64(inp["x"]), 0.5, O.to64(inp["mlp1"]),
                       ps_version="v1" if flags & 1 else "v2")
    assert_connector_close(y, ref.reshape(-1, ref.shape[-1]), f"half flags={flags}")


@pytest.mark.parametrize("flags", [0, 1, 2])
def test_ps_project_quarter_small_ragged(flags):
    ivc = _ivc()
    inp = W.make(small_workload(C=128, H=192, tiles=(3,)), affine="random")  # 3*64 rows: ragged
    x = inp["x"].cuda()
    m = ivc.Mlp(inp["mlp2"])
    y = ivc.ps_project(x, 0.25, m, flags=flags)
    torch.cuda.synchronize()
    x64 = O.to64(inp["x"])
    if flags == 2:
        ref = O.ps_project(x64, 0.25, O.to64(inp["mlp2"]), quarter_order="twice")
    else:
        ref = O.ps_project(x64, 0.25, O.to64(inp["mlp2"]), ps_version="v1" if flags else "v2")
        if flags == 1:  # v1 transposes the 8x8 token grid
            ref = ref.reshape(3, 8, 8, -1).transpose(0, 2, 1, 3).reshape(3, 64, -1)
    assert_connector_close(y, ref.reshape(-1, ref.shape[-1]), f"quarter flags={flags}")


def test_prefolded_equals_per_call_fold():
    ivc = _ivc()
    inp = W.make(small_workload(C=64, H=128, tiles=(2,)), affine="random")
    x = inp["x"].cuda()
    a = ivc.ps_project(x, 0.5, ivc.Mlp(inp["mlp1"]))
    b = ivc.ps_project(x, 0.5, ivc.Mlp(inp["mlp1"]).fold())
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_ps_project_deterministic():
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=256, tiles=(5,)), affine="random")
    x = inp["x"].cuda()
    m = ivc.Mlp(inp["mlp2"]).fold()
    a = ivc.ps_project(x, 0.25, m)
    b = ivc.ps_project(x, 0.25, m)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_single_tile_2b_connector_full():
    ivc = _ivc()
    inp = W.make("single_tile_2b")
    m = ivc.Mlp(inp["mlp1"]).fold()
    y = ivc.ps_project(inp["x"].cuda(), 0.5, m)
    torch.cuda.synchronize()
    assert y.shape == (256, 2048)
    ref = O.ps_project(O.to64(inp["x"]), 0.5, O.to64(inp["mlp1"]))
    e = assert_connector_close(y, ref.reshape(256, 2048), "single tile")
    assert e["max_abs"] <= 3e-2, e  # literal bound holds at these magnitudes


def test_ps_project_empty_batch():
    ivc = _ivc()
    inp = W.make(small_workload(C=64, H=128, tiles=(1,)))
    m = ivc.Mlp(inp["mlp1"])
    x = torch.empty(0, 32, 32, 64, dtype=torch.bfloat16, device="cuda")
    y = ivc.ps_project(x, 0.5, m, out=torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert y.numel() == 0


@pytest.mark.parametrize("name", ["connector_14b_832tiles", "connector_38b_416tiles"])
def test_large_connector_sampled_tiles(name):
    """Full-size launch (the sizes the benchmark times); the oracle checks a
    seeded sample of tiles spread over the batch, row by row."""
    ivc = _ivc()
    inp = W.make(name)
    T, C, H = inp["T"], inp["C"], inp["H"]
    x = inp["x"].cuda()
    m = ivc.Mlp(inp["mlp1"]).fold()
    y = ivc.ps_project(x, 0.5, m)
    torch.cuda.synchronize()
    del x
    rng = np.random.default_rng(7)
    tiles = sorted(set([0, T - 1] + rng.choice(T, 4, replace=False).tolist()))
    xs = O.to64(inp["x"][tiles])
    ref = O.ps_project(xs, 0.5, O.to64(inp["mlp1"]))
    got = y.view(T, 256, H)[tiles]
    assert_connector_close(got, ref, name)


# ------------------------------------------------------------------ router
def _route_check(ivc, inp, gate, mask, offsets, sample=None, scope=0, rel_q=0.1, abs_t=0.5):
    x64 = O.to64(inp["x"])
    T = inp["T"]
    tiles = list(range(T)) if sample is None else sample
    r64 = O.to64(inp["router"])
    ref_gate = O.vir_gate(x64[tiles], inp["valid_len"].numpy()[tiles], r64)
    g = to_np(gate)
    assert np.all(np.isfinite(g))
    np.testing.assert_allclose(g[:, 0] + g[:, 1], 1.0, atol=1e-6)
    err = np.abs(g[tiles] - ref_gate).max()
    assert err <= GATE_ABS, err
    # routing and offsets: bit-exact given the GPU's own fp32 gate vector
    ref_mask = O.route(g[:, 0].astype(np.float32).astype(np.float64), inp["image_offsets"].numpy(),
                       rel_q, abs_t, scope="batch" if scope else "image")
    np.testing.assert_array_equal(to_np(mask), ref_mask)
    np.testing.assert_array_equal(to_np(offsets), O.compaction_offsets(ref_mask))
    return err


@pytest.mark.parametrize("pool_mode,fold", [(0, True), (0, False), (1, False)])
def test_vir_route_small_with_padding(pool_mode, fold):
    ivc = _ivc()
    w = small_workload(C=256, H=128, tiles=(3, 1, 5), var=0.6)
    inp = W.make(w, affine="random")
    vl = inp["valid_len"].clone()
    vl[1] = 1   # a single valid token
    inp["valid_len"] = vl
    inp["x"] = W.features(inp["T"], 256, 1234 + 90, vl)
    r = ivc.Router(inp["router"], pool_mode=pool_mode, fold=fold)
    assert (r.folded is not None) == fold
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_VIR_ROUTE, inp["T"], 256, r=r))
    gate, mask, offsets = ivc.vir_route(inp["x"].cuda(), vl.cuda(), inp["image_offsets"].cuda(), r,
                                        workspace=ws)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    _route_check(ivc, inp, gate, mask, offsets)
    assert to_np(mask)[3] == 0  # the one-tile image is never compressed


@pytest.mark.parametrize("pool_mode,fold", [(0, True), (0, False), (1, False)])
def test_vir_route_batch_scope(pool_mode, fold):
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(4, 4)), affine="random")
    r = ivc.Router(inp["router"], scope=1, pool_mode=pool_mode, fold=fold)
    gate, mask, offsets = ivc.vir_route(inp["x"].cuda(), None, inp["image_offsets"].cuda(), r)
    torch.cuda.synchronize()
    _route_check(ivc, inp, gate, mask, offsets, scope=1)


@pytest.mark.parametrize("pool_mode", [0, 1])
def test_vir_route_gating_residual_inside(pool_mode):
    """Reading variant: h <- LN(h + u) in the gating blocks."""
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(3, 2)), affine="random")
    r = ivc.Router(inp["router"], pool_mode=pool_mode, gate_residual=1)
    gate, mask, offsets = ivc.vir_route(inp["x"].cuda(), None, inp["image_offsets"].cuda(), r)
    torch.cuda.synchronize()
    ref = O.vir_gate(O.to64(inp["x"]), inp["valid_len"].numpy(), O.to64(inp["router"]),
                     residual="inside")
    assert np.abs(to_np(gate) - ref).max() <= GATE_ABS
    outside = O.vir_gate(O.to64(inp["x"]), inp["valid_len"].numpy(), O.to64(inp["router"]))
    assert np.abs(ref - outside).max() > 10 * GATE_ABS  # the variant really differs


_GATING_SNIPPET = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
import oracle as O, workloads as W, vlm_visual_token_b200 as ivc
G, inside = {G!r}, {inside!r}
w = W.Workload("gw", "flash", C=256, H=128, tiles_per_image=(3, 18), n_images=2, mlp2_mid=256,
               D=256, gate_hidden=G, seed_base=93)
inp = W.make(w, affine="random")
r = ivc.Router(inp["router"], pool_mode=1, gate_residual=inside)
ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_VIR_ROUTE, inp["T"], 256, r=r))
gate, mask, offsets = ivc.vir_route(inp["x"].cuda(), None, inp["image_offsets"].cuda(), r,
                                    workspace=ws)
torch.cuda.synchronize()
assert ivc.device_status(ws) == 0
ref = O.vir_gate(O.to64(inp["x"]), inp["valid_len"].numpy(), O.to64(inp["router"]),
                 residual="inside" if inside else "outside")
g = gate.cpu().double().numpy()
assert np.abs(g - ref).max() <= {gate_abs!r}, np.abs(g - ref).max()
ref_mask = O.route(g[:, 0], inp["image_offsets"].numpy())
np.testing.assert_array_equal(mask.cpu().numpy(), ref_mask)
np.testing.assert_array_equal(offsets.cpu().numpy(), O.compaction_offsets(ref_mask))
print("gating ok")
"""


@pytest.mark.parametrize("fused", ["0", "1"])
@pytest.mark.parametrize("G,inside", [(512, 0), (2048, 0), (256, 1)])
def test_vir_route_gating_widths(G, inside, fused):
    """The Gating of the separate-kernel router (here through literal
    pooling), as 13 launches or as one cooperative kernel (IVC_GATING_FUSED=1:
    items of 64 or 16 columns, CTAs without an item in one of the two
    projections, 21 rows in two rounds), for a gating width unlike the
    pooling width and for the LN(h + u) reading; in a fresh process since the
    switch is read once."""
    _ivc()
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = _GATING_SNIPPET.format(root=root, G=G, inside=inside, gate_abs=GATE_ABS)
    out = subprocess.run([sys.executable, "-c", code], env={**os.environ, "IVC_GATING_FUSED": fused},
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "gating ok" in out.stdout


def test_bad_valid_len_sets_status_bit():
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(2,)))
    r = ivc.Router(inp["router"])
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_VIR_ROUTE, 2, 256, r=r))
    vl = torch.tensor([0, 1024], dtype=torch.int32, device="cuda")
    ivc.vir_route(inp["x"].cuda(), vl, inp["image_offsets"].cuda(), r, workspace=ws)
    assert ivc.device_status(ws) & 1
    assert ivc.device_status(ws) == 0  # cleared by the read


def test_bad_image_offsets_sets_status_bit():
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(2, 2)))
    r = ivc.Router(inp["router"])
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_VIR_ROUTE, 4, 256, r=r))
    offs = torch.tensor([0, 3, 2], dtype=torch.int32, device="cuda")  # ends at 2 != T
    _, mask, offsets = ivc.vir_route(inp["x"].cuda(), None, offs, r, workspace=ws)
    assert ivc.device_status(ws) & 2
    assert to_np(mask).sum() == 0 and to_np(offsets)[-1] == 4 * 256


# ------------------------------------------------------------------ whole path
def _flash_check(ivc, inp, res, tiles=None, rel_q=0.1, abs_t=0.5):
    T, H = inp["T"], inp["H"]
    x64 = O.to64(inp["x"])
    sel = list(range(T)) if tiles is None else tiles
    Y256 = O.ps_project(x64[sel], 0.5, O.to64(inp["mlp1"]))
    Y64 = O.ps_project(x64[sel], 0.25, O.to64(inp["mlp2"]))
    gate, mask, offsets = res["gate"], res["mask"], res["offsets"]
    _route_check(ivc, inp, gate, mask, offsets, sample=tiles, rel_q=rel_q, abs_t=abs_t)
    offs = to_np(offsets)
    m = to_np(mask)
    assert int(to_np(res["total"])[0]) == offs[-1] == 256 * (T - m.sum()) + 64 * m.sum()
    out = res["out"]
    stats = []
    for i, t in enumerate(sel):
        rows = out[offs[t]:offs[t + 1]]
        ref = Y64[i] if m[t] else Y256[i]
        stats.append(assert_connector_close(rows, ref, f"tile {t}"))
    return stats


@pytest.mark.parametrize("pool_mode,fold", [(0, True), (0, False), (1, False)])
def test_flash_compress_small(pool_mode, fold):
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=192, tiles=(3, 1, 4), var=0.3), affine="random")
    m1, m2 = ivc.Mlp(inp["mlp1"]), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"], pool_mode=pool_mode, fold=fold)
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, inp["T"], 256, m1, m2, r))
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r, workspace=ws)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    _flash_check(ivc, inp, res)


def test_flash_compress_padding_extremes():
    """The dual flow's router kernels on a tile with one valid token, one whose
    second 128-token chunk holds a single valid token, and 4 heads of 64."""
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(3, 2), var=0.6), affine="random")
    vl = inp["valid_len"].clone()
    vl[1] = 1
    vl[3] = 129
    inp["valid_len"] = vl
    inp["x"] = W.features(inp["T"], 256, 1234 + 91, vl)
    m1, m2 = ivc.Mlp(inp["mlp1"]), ivc.Mlp(inp["mlp2"])
    r = ivc.Router(inp["router"])
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, inp["T"], 256, m1, m2, r))
    res = ivc.flash_compress(inp["x"].cuda(), vl.cuda(), inp["image_offsets"].cuda(), m1, m2, r,
                             workspace=ws)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    _flash_check(ivc, inp, res)


def test_flash_compress_empty():
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(1,)))
    m1, m2, r = ivc.Mlp(inp["mlp1"]), ivc.Mlp(inp["mlp2"]), ivc.Router(inp["router"])
    x = torch.empty(0, 32, 32, 256, dtype=torch.bfloat16, device="cuda")
    res = ivc.flash_compress(x, None, torch.zeros(1, dtype=torch.int32, device="cuda"), m1, m2, r)
    torch.cuda.synchronize()
    assert int(res["total"].item()) == 0 and int(res["offsets"][0].item()) == 0


@pytest.mark.parametrize("pool_mode,fold", [(0, True), (0, False), (1, False)])
def test_flash_2b_13tiles_full(pool_mode, fold):
    """The benchmark workload, every output checked against the oracle."""
    ivc = _ivc()
    inp = W.make("flash_2b_13tiles")
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"], pool_mode=pool_mode, fold=fold)
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r)
    torch.cuda.synchronize()
    stats = _flash_check(ivc, inp, res)
    assert max(s["max_abs"] for s in stats) <= 3e-2, stats


@pytest.mark.parametrize("pool_mode", [0, 1])
def test_flash_4b_batched_sampled(pool_mode):
    """16 images with drawn tile counts and 10% padded tiles; the oracle checks
    a seeded sample of tiles (including padded ones); routing and offsets are
    checked for every tile."""
    ivc = _ivc()
    inp = W.make("flash_4b_batched")
    T = inp["T"]
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"], pool_mode=pool_mode)
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, T, 1024, m1, m2, r))
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r, workspace=ws)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    padded = np.nonzero(inp["valid_len"].numpy() < 1024)[0].tolist()
    rng = np.random.default_rng(11)
    tiles = sorted(set(padded[:4] + rng.choice(T, 6, replace=False).tolist() + [T - 1]))
    _flash_check(ivc, inp, res, tiles=tiles)


# ---------------------------------------------------------------- router-first flow
def _routed_vs_dual(ivc, inp, m1, m2, r, routed_res):
    """Rows of tiles routed alike in both flows agree. They are computed by
    the same kernels; only the split-K slicing, chosen per launch from the
    number of rows, can change the fp32 summation order."""
    dual = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                              m1, m2, r)
    torch.cuda.synchronize()
    md, mr = to_np(dual["mask"]), to_np(routed_res["mask"])
    od, orr = to_np(dual["offsets"]), to_np(routed_res["offsets"])
    same = 0
    for t in range(inp["T"]):
        if md[t] != mr[t]:
            continue
        a = dual["out"][od[t]:od[t + 1]]
        b = routed_res["out"][orr[t]:orr[t + 1]]
        torch.testing.assert_close(b.float(), a.float(), rtol=2e-2, atol=2e-2,
                                   msg=lambda m: f"tile {t}: routed vs dual-path rows: {m}")
        same += 1
    assert same > 0


@pytest.mark.parametrize("pool_mode,fold", [(0, True), (0, False), (1, False)])
def test_flash_routed_small(pool_mode, fold):
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=192, tiles=(3, 1, 4), var=0.3), affine="random")
    m1, m2 = ivc.Mlp(inp["mlp1"]), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"], pool_mode=pool_mode, fold=fold)
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, inp["T"], 256, m1, m2, r))
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r, workspace=ws, routed=True)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    _flash_check(ivc, inp, res)
    _routed_vs_dual(ivc, inp, m1, m2, r, res)


@pytest.mark.parametrize("abs_t,rel_q", [(1.5, 0.1), (0.0, 0.0)])
def test_flash_routed_one_path_only(abs_t, rel_q):
    """abs_t 1.5: no tile is compressed (the mlp2 launches see zero rows);
    abs_t 0 with rel_q 0: every tile but each image's lowest gate is."""
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(5, 2), var=0.0))
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"], rel_q=rel_q, abs_t=abs_t)
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r, routed=True)
    torch.cuda.synchronize()
    m = to_np(res["mask"])
    if abs_t > 1:
        assert m.sum() == 0
    else:
        assert m.sum() == inp["T"] - 2
    _flash_check(ivc, inp, res, rel_q=rel_q, abs_t=abs_t)


def test_flash_routed_empty():
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=128, tiles=(1,)))
    m1, m2, r = ivc.Mlp(inp["mlp1"]), ivc.Mlp(inp["mlp2"]), ivc.Router(inp["router"])
    x = torch.empty(0, 32, 32, 256, dtype=torch.bfloat16, device="cuda")
    res = ivc.flash_compress(x, None, torch.zeros(1, dtype=torch.int32, device="cuda"), m1, m2, r,
                             routed=True)
    torch.cuda.synchronize()
    assert int(res["total"].item()) == 0 and int(res["offsets"][0].item()) == 0


def test_flash_routed_2b_13tiles_full():
    """The benchmark workload through the router-first flow, every output
    row checked against the oracle and against the dual-path flow."""
    ivc = _ivc()
    inp = W.make("flash_2b_13tiles")
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"])
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r, routed=True)
    torch.cuda.synchronize()
    stats = _flash_check(ivc, inp, res)
    assert max(s["max_abs"] for s in stats) <= 3e-2, stats
    _routed_vs_dual(ivc, inp, m1, m2, r, res)


def test_flash_routed_4b_batched_sampled():
    """97 tiles in 16 images: odd per-path tile counts, many m-tiles and CTA
    pairs spanning two listed tiles of the factor-0.25 path."""
    ivc = _ivc()
    inp = W.make("flash_4b_batched")
    T = inp["T"]
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"])
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, T, 1024, m1, m2, r))
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r, workspace=ws, routed=True)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    padded = np.nonzero(inp["valid_len"].numpy() < 1024)[0].tolist()
    rng = np.random.default_rng(12)
    tiles = sorted(set(padded[:4] + rng.choice(T, 6, replace=False).tolist() + [T - 1]))
    _flash_check(ivc, inp, res, tiles=tiles)
    _routed_vs_dual(ivc, inp, m1, m2, r, res)


# ---------------------------------------------------------------- sequence assembly
def _prompt_ids(tiles_per_seq, img_id, V, seed, text=(5, 3), extra_img=0):
    rng = np.random.default_rng(seed)
    ids, offs = [], [0]
    for n in tiles_per_seq:
        pre = [int(v) for v in rng.integers(0, V, text[0]) if v != img_id]
        post = [int(v) for v in rng.integers(0, V, text[1]) if v != img_id]
        ids += pre + [img_id] * (256 * n) + post
        offs.append(len(ids))
    ids += [img_id] * extra_img
    offs[-1] = len(ids)
    return np.array(ids, dtype=np.int32), np.array(offs, dtype=np.int32)


def _assemble_check(ivc, ids, offs, img_id, table, visual, mask, v_offs, expect_status=0):
    dev = "cuda"
    res = ivc.assemble_sequence(torch.from_numpy(ids).to(dev), torch.from_numpy(offs).to(dev),
                                img_id, table.to(dev), visual.to(dev),
                                torch.from_numpy(mask.astype(np.uint8)).to(dev),
                                torch.from_numpy(v_offs.astype(np.int32)).to(dev))
    torch.cuda.synchronize()
    assert ivc.device_status(res["workspace"]) == expect_status
    ref = O.assemble_sequence(ids, offs, img_id, table.float().numpy(), visual.float().numpy(),
                              mask, v_offs)
    n = int(ref["seq_offsets"][-1])
    np.testing.assert_array_equal(to_np(res["seq_offsets"]), ref["seq_offsets"])
    np.testing.assert_array_equal(to_np(res["ids"])[:n], ref["ids"])
    np.testing.assert_array_equal(to_np(res["positions"])[:n], ref["positions"])
    # pure data movement: bit-exact rows
    np.testing.assert_array_equal(res["embeds"][:n].float().cpu().numpy(), ref["embeds"])
    return n


@pytest.mark.parametrize("tiles", [(3, 1, 2), (1,), (0, 2, 0)])
def test_assemble_sequence_small(tiles):
    ivc = _ivc()
    T = sum(tiles)
    rng = np.random.default_rng(31 + T)
    mask = (rng.random(T) < 0.5).astype(np.uint8)
    v_offs = O.compaction_offsets(mask)
    V, H, img = 600, 64, 599
    g = torch.Generator().manual_seed(5)
    table = torch.randn(V, H, generator=g).to(torch.bfloat16)
    visual = torch.randn(max(int(v_offs[-1]), 1), H, generator=g).to(torch.bfloat16)
    ids, offs = _prompt_ids(tiles, img, V, seed=T)
    n = _assemble_check(ivc, ids, offs, img, table, visual, mask, v_offs)
    assert n == len(ids) - 192 * int(mask.sum())


def test_assemble_sequence_flags_a_bad_prompt():
    """Two placeholders more than 256 T: flagged, and they stay text rows."""
    ivc = _ivc()
    mask = np.array([1, 0], dtype=np.uint8)
    v_offs = O.compaction_offsets(mask)
    V, H, img = 100, 32, 7
    g = torch.Generator().manual_seed(6)
    table = torch.randn(V, H, generator=g).to(torch.bfloat16)
    visual = torch.randn(int(v_offs[-1]), H, generator=g).to(torch.bfloat16)
    ids, offs = _prompt_ids((2,), img, V, seed=3, extra_img=2)
    _assemble_check(ivc, ids, offs, img, table, visual, mask, v_offs, expect_status=16)


def test_assemble_after_flash_compress():
    """The 13-tile image through ivc_flash_compress, then into a two-turn
    prompt; rows checked against the oracle's splice of the GPU's own rows."""
    ivc = _ivc()
    inp = W.make("flash_2b_13tiles")
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"])
    res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                             m1, m2, r)
    torch.cuda.synchronize()
    mask = to_np(res["mask"])
    v_offs = to_np(res["offsets"])
    total = int(v_offs[-1])
    V, H, img = 4096, inp["H"], 4095
    table = torch.randn(V, H, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    ids, offs = _prompt_ids((13,), img, V, seed=13, text=(40, 12))
    ids2, _ = _prompt_ids((0,), img, V, seed=14, text=(20, 0))
    ids = np.concatenate([ids, ids2]).astype(np.int32)
    offs = np.array([0, offs[1], len(ids)], dtype=np.int32)
    n = _assemble_check(ivc, ids, offs, img, table, res["out"][:total].cpu(), mask, v_offs)
    assert n == len(ids) - 192 * int(mask.sum())


# ---------------------------------------------------------------- opt-in kernel variants
_VARIANT_SNIPPET = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
import oracle as O, workloads as W, vlm_visual_token_b200 as ivc
inp = W.make("flash_2b_13tiles")
m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
r = ivc.Router(inp["router"])
res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(), inp["image_offsets"].cuda(),
                         m1, m2, r)
torch.cuda.synchronize()
from tests._parity import assert_connector_close
x64 = O.to64(inp["x"])
ref_gate = O.vir_gate(x64, inp["valid_len"].numpy(), O.to64(inp["router"]))
g = res["gate"].cpu().double().numpy()
gate_err = np.abs(g - ref_gate).max()
assert gate_err <= {gate_abs!r}, gate_err
mask = res["mask"].cpu().numpy(); offs = res["offsets"].cpu().numpy()
ref_mask = O.route(g[:, 0], inp["image_offsets"].numpy())
np.testing.assert_array_equal(mask, ref_mask)
np.testing.assert_array_equal(offs, O.compaction_offsets(ref_mask))
assert int(res["total"].item()) == offs[-1]
worst = 0.0
for t in range(inp["T"]):
    ref = (O.ps_project(x64[t:t + 1], 0.25, O.to64(inp["mlp2"])) if mask[t]
           else O.ps_project(x64[t:t + 1], 0.5, O.to64(inp["mlp1"]))).reshape(-1, inp["H"])
    e = assert_connector_close(res["out"][offs[t]:offs[t + 1]], ref, f"tile {{t}}")
    worst = max(worst, e["max_abs"])
assert worst <= 3e-2, worst
print("variant ok")
"""


@pytest.mark.parametrize("env", [{"IVC_GEMM_WIDE": "1"}, {"IVC_GEMM_PAIRS": "0"},
                                 {"IVC_ROUTER_FUSED": "1"}, {"IVC_POOL_ATTEND": "0"},
                                 {"IVC_GATING_FUSED": "1"}, {"IVC_POOL_TAIL": "1"},
                                 {"IVC_ATTEND_TC": "0"}, {"IVC_GEMM_GRAPH": "0"},
                                 {"IVC_GRAPH_WIDE": "0"}, {"IVC_GRAPH_WIDE": "2"},
                                 {"IVC_GRAPH_GROUP": "0"}])
def test_flash_kernel_variants(env):
    """The opt-in kernel variants (512-wide pair tiles with split-K, single-CTA
    256-wide tiles, the persistent router inside the dual flow, the pooling as
    tensor-core scores / softmax / weighted-sum kernels; in the single launch
    only 256-wide tiles, 256 x 512 tiles for both first Linears, row-block tile
    order throughout), each in a fresh process since the switches are read
    once."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _VARIANT_SNIPPET.format(root=root, gate_abs=GATE_ABS)],
                         env={**os.environ, **env}, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "variant ok" in out.stdout


# ---------------------------------------------------------------- multi-Linear launch
@pytest.mark.parametrize("flags,scale", [(0, 0.5), (1, 0.5), (0, 0.25), (1, 0.25), (2, 0.25)])
def test_ps_project_single_launch_small(flags, scale):
    """Shapes the single persistent launch of all Linears takes (widths
    multiples of 128): 5 tiles, so the factor-0.25 rows (320) end inside a
    256-row block, every pixel_shuffle flag."""
    ivc = _ivc()
    inp = W.make(small_workload(C=128, H=256, mid=384, tiles=(5,)), affine="random")
    key = "mlp1" if scale == 0.5 else "mlp2"
    y = ivc.ps_project(inp["x"].cuda(), scale, ivc.Mlp(inp[key]).fold(), flags=flags)
    torch.cuda.synchronize()
    x64 = O.to64(inp["x"])
    if flags == 2:
        ref = O.ps_project(x64, 0.25, O.to64(inp[key]), quarter_order="twice")
    else:
        ref = O.ps_project(x64, scale, O.to64(inp[key]), ps_version="v1" if flags else "v2")
        if flags == 1 and scale == 0.25:
            ref = ref.reshape(5, 8, 8, -1).transpose(0, 2, 1, 3).reshape(5, 64, -1)
    assert_connector_close(y, ref.reshape(-1, ref.shape[-1]), f"{key} flags={flags}")


@pytest.mark.parametrize("tiles", [(3, 1, 4), (1,), (9, 8)])
def test_flash_single_launch_small(tiles):
    """Both MLPs in one persistent launch beside the router: 1, 8 and 17
    tiles (1..5 row blocks of 256 for mlp1, ragged ones for mlp2)."""
    ivc = _ivc()
    inp = W.make(small_workload(C=256, H=256, mid=384, tiles=tiles, var=0.3), affine="random")
    m1, m2 = ivc.Mlp(inp["mlp1"]), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"])
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, inp["T"], 256, m1, m2, r))
    for _ in range(2):  # the row-block counters start from zero on every call
        res = ivc.flash_compress(inp["x"].cuda(), inp["valid_len"].cuda(),
                                 inp["image_offsets"].cuda(), m1, m2, r, workspace=ws)
        torch.cuda.synchronize()
        assert ivc.device_status(ws) == 0
        _flash_check(ivc, inp, res)


@pytest.mark.parametrize("env", [{"IVC_GRAPH_WIDE": "2"}, {"IVC_GRAPH_GROUP": "2"},
                                 {"IVC_GRAPH_WIDE": "2", "IVC_GRAPH_GROUP": "3"}])
def test_single_launch_small_tile_forms(env):
    """The single launch's other tile forms on the small shapes above, in a
    fresh process: 256 x 512 tiles on every first Linear (widths of 256 and
    384, so a tile's second half is partly or wholly past N, mixed with the
    256-wide tiles of the later Linears), and tiles in groups of 2 or 3 row
    blocks on every Linear (up to 17 row blocks, so the last group is short)."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                          os.path.join(root, "tests", "test_gpu_parity.py"), "-k",
                          "single_launch_small and not tile_forms"],
                         env={**os.environ, **env}, capture_output=True, text=True,
                         timeout=600, cwd=root)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-2000:]
    assert " passed" in out.stdout
