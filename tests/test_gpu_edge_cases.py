"""GPU parity on the method's edge cases, against the fp64 oracle.

* Routing ([VIR] section 4; [DP] "路由决策：相对 + 绝对双阈值判定", where the
  operators survive as > and >=): ties in the rank sort, gates exactly at the
  quantile and exactly at 0.5, one-tile images, rel_q 0 and 1, groups wider
  than one CTA, a NaN gate (torch.quantile propagates it), a batch-scope
  group above the supported size. Through ivc_route on crafted gate vectors,
  bit-exact against the oracle's route and offsets.
* A router whose head is zero: every gate is exactly 0.5, so every tile ties
  the quantile and the mask is all 0 (both router forms, both flash flows).
* The connector's LayerNorm fold (rstd (x W' - mean colsum(W'))) on features
  with a mean of +20 and outlier channels at +-100 ([PS] "MLP 连接器源码逐行解析":
  LayerNorm first): the subtraction cancels most of the product, so parity is
  checked at the stated tolerances for mlp1 and mlp2.
* Variable-length tiles whose pad rows hold large non-zero values: the pooling
  must ignore them ([VIR] section 2, padding mask), as the oracle does.
* A NaN in one tile's features: the rows it reaches and its gate are NaN, its
  image's quantile is NaN so none of that image's tiles is compressed, every
  other tile and image is unaffected, and the call returns with a clear status.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests._parity import GATE_ABS, assert_connector_close, to_np

pytestmark = pytest.mark.gpu


def _ivc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import vlm_visual_token_b200 as ivc
    return ivc


def _small(C=256, H=128, mid=320, tiles=(3, 4), var=0.0, seed=95):
    return W.Workload("edge", "flash", C=C, H=H, tiles_per_image=tuple(tiles),
                      n_images=len(tiles), mlp2_mid=mid, D=C, gate_hidden=256, var_len_frac=var,
                      seed_base=seed)


def _route_gpu(ivc, g32, offs, rel_q=0.1, abs_t=0.5, scope=0):
    T = g32.shape[0]
    gate = torch.from_numpy(np.stack([g32, 1.0 - g32], axis=1).astype(np.float32)).cuda()
    o = torch.from_numpy(np.asarray(offs, dtype=np.int32)).cuda()
    ws = ivc.new_workspace(ivc.ROUTE_WORKSPACE_BYTES)
    mask, offsets, total = ivc.route(gate, o, rel_q, abs_t, scope, workspace=ws)
    torch.cuda.synchronize()
    return to_np(mask), to_np(offsets), int(to_np(total)[0]), ivc.device_status(ws)


def _route_ref(g32, offs, rel_q=0.1, abs_t=0.5, scope=0):
    m = O.route(g32.astype(np.float64), np.asarray(offs), rel_q, abs_t,
                scope="batch" if scope else "image")
    return m, O.compaction_offsets(m)


def _assert_route(ivc, g32, offs, rel_q=0.1, abs_t=0.5, scope=0):
    mask, offsets, total, st = _route_gpu(ivc, g32, offs, rel_q, abs_t, scope)
    ref_m, ref_o = _route_ref(g32, offs, rel_q, abs_t, scope)
    assert st == 0
    np.testing.assert_array_equal(mask, ref_m)
    np.testing.assert_array_equal(offsets, ref_o)
    assert total == ref_o[-1]
    return mask


# ------------------------------------------------------------------ routing alone
def test_route_all_gates_at_one_half():
    """Every gate ties the quantile (0.5 > 0.5 is false): nothing compressed."""
    ivc = _ivc()
    g = np.full(13, 0.5, dtype=np.float32)
    m = _assert_route(ivc, g, [0, 13])
    assert m.sum() == 0


def test_route_exact_one_half_boundary():
    """Gates exactly 0.5 above a lower quantile are compressed (>= 0.5);
    gates just below 0.5 are not; the gate at the quantile is not (strict >)."""
    ivc = _ivc()
    below = np.nextafter(np.float32(0.5), np.float32(0))
    g = np.array([0.5, 0.7, 0.5, 0.3, 0.6, 0.5, below, 0.9, 0.5, 0.55, 0.5, 0.2, 0.8],
                 dtype=np.float32)
    m = _assert_route(ivc, g, [0, 13])
    assert m[0] == 1 and m[6] == 0 and m[11] == 0
    # the quantile itself lands on 0.5: q = 1.0 puts it at the maximum and
    # rel_q chosen so that pos is integral on a 0.5 value
    _assert_route(ivc, g, [0, 13], rel_q=1.0)
    _assert_route(ivc, g, [0, 13], rel_q=0.0)
    _assert_route(ivc, np.array([0.5, 0.5, 0.6, 0.6, 0.6], dtype=np.float32), [0, 5], rel_q=0.5)


def test_route_ties_random_groups():
    """Gates drawn from a handful of values (many ties, some at 0.5), images of
    1..40 tiles, then one group wider than a CTA (2500 tiles), both scopes."""
    ivc = _ivc()
    rng = np.random.default_rng(17)
    levels = np.array([0.1, 0.3, 0.5, 0.5, 0.55, 0.7, 0.9], dtype=np.float32)
    counts = rng.integers(1, 41, size=60)
    offs = np.concatenate([[0], np.cumsum(counts)])
    g = levels[rng.integers(0, len(levels), size=int(offs[-1]))]
    for rel_q in (0.1, 0.0, 0.35, 1.0):
        _assert_route(ivc, g, offs, rel_q=rel_q)
        _assert_route(ivc, g, offs, rel_q=rel_q, scope=1)
    wide = levels[rng.integers(0, len(levels), size=2500)]
    _assert_route(ivc, wide, [0, 1000, 2500])
    _assert_route(ivc, wide, [0, 2500], scope=1)
    # a one-tile image is never compressed, whatever its gate
    m = _assert_route(ivc, np.array([0.99, 0.2, 0.99, 0.98], dtype=np.float32), [0, 1, 4])
    assert m[0] == 0


def test_route_nan_gate_disables_its_image():
    ivc = _ivc()
    rng = np.random.default_rng(23)
    g = rng.random(20).astype(np.float32)
    g[[2, 14]] = [np.nan, 0.9]
    offs = [0, 7, 13, 20]
    m = _assert_route(ivc, g, offs)
    assert m[0:7].sum() == 0               # the image holding the NaN
    ref_other = _route_ref(g[7:], [0, 6, 13])[0]
    np.testing.assert_array_equal(m[7:], ref_other)
    m = _assert_route(ivc, g, offs, scope=1)
    assert m.sum() == 0


def test_route_status_bits():
    """A batch-scope group above IVC_MAX_QUANTILE_GROUP, and image offsets
    that do not end at T: flagged in the status word, nothing compressed."""
    ivc = _ivc()
    g = np.full(9000, 0.9, dtype=np.float32)
    g[::7] = 0.6
    mask, offsets, total, st = _route_gpu(ivc, g, [0, 9000], scope=1)
    assert st & 8 and mask.sum() == 0 and total == 256 * 9000
    g = np.full(6, 0.9, dtype=np.float32)
    mask, offsets, total, st = _route_gpu(ivc, g, [0, 3, 5])
    assert st & 2 and mask.sum() == 0 and total == 256 * 6


# ------------------------------------------------------------------ zero router head
def _zero_head(inp):
    inp["router"]["gWout"] = torch.zeros_like(inp["router"]["gWout"])
    inp["router"]["gbout"] = torch.zeros_like(inp["router"]["gbout"])
    return inp


@pytest.mark.parametrize("pool_mode", [0, 1])
def test_zero_head_every_gate_exactly_one_half(pool_mode):
    ivc = _ivc()
    inp = _zero_head(W.make(_small(tiles=(5, 1, 4)), affine="random"))
    r = ivc.Router(inp["router"], pool_mode=pool_mode)
    gate, mask, offsets = ivc.vir_route(inp["x"].cuda(), None, inp["image_offsets"].cuda(), r)
    torch.cuda.synchronize()
    assert np.all(to_np(gate) == 0.5)
    assert to_np(mask).sum() == 0
    np.testing.assert_array_equal(to_np(offsets), 256 * np.arange(inp["T"] + 1))
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    for routed in (False, True):
        res = ivc.flash_compress(inp["x"].cuda(), None, inp["image_offsets"].cuda(), m1, m2, r,
                                 routed=routed)
        torch.cuda.synchronize()
        assert np.all(to_np(res["gate"]) == 0.5)
        assert to_np(res["mask"]).sum() == 0
        assert int(res["total"].item()) == 256 * inp["T"]


# ------------------------------------------------------------------ LayerNorm fold cancellation
def _shifted_features(T, C, seed, mean=20.0, outliers=(3, 77, 500, 1000), level=100.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, 32, 32, C, generator=g) + mean
    for i, c in enumerate(outliers):
        if c < C:
            x[..., c] = level if i % 2 == 0 else -level
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("scale", [0.5, 0.25])
def test_connector_large_mean_and_outlier_channels(scale):
    """mean +20, four channels at +-100, InternVL3.5-2B-Flash widths (mlp1
    4096->2048->2048, mlp2 16384->4096->2048->2048), 5 tiles (ragged row tiles)."""
    ivc = _ivc()
    w = W.Workload("shifted", "flash", C=1024, H=2048, tiles_per_image=(5,), n_images=1,
                   seed_base=96)
    inp = W.make(w, affine="random")
    x = _shifted_features(5, 1024, seed=41)
    key = "mlp1" if scale == 0.5 else "mlp2"
    m = ivc.Mlp(inp[key]).fold()
    y = ivc.ps_project(x.cuda(), scale, m)
    torch.cuda.synchronize()
    ref = O.ps_project(O.to64(x), scale, O.to64(inp[key]))
    assert_connector_close(y, ref.reshape(-1, ref.shape[-1]), f"shifted {key}")


# ------------------------------------------------------------------ garbage in pad rows
def _garbage_pads(inp, level=60.0, seed=7):
    """Pad rows (tokens >= valid_len) filled with large non-zero values."""
    vl = inp["valid_len"]
    x = inp["x"].clone().float()
    g = torch.Generator().manual_seed(seed)
    idx = torch.arange(1024).view(1, 32, 32)
    pad = idx >= vl.view(-1, 1, 1).long()
    noise = level + 30.0 * torch.randn(x.shape, generator=g)
    x[pad] = noise[pad]
    inp["x"] = x.to(torch.bfloat16)
    return inp


@pytest.mark.parametrize("pool_mode", [0, 1])
def test_pad_rows_with_large_values_are_ignored(pool_mode):
    ivc = _ivc()
    inp = W.make(_small(tiles=(4, 3), var=0.0), affine="random")
    vl = torch.tensor([1024, 300, 129, 1, 700, 1000, 64], dtype=torch.int32)
    inp["valid_len"] = vl
    inp = _garbage_pads(inp)
    x64 = O.to64(inp["x"])
    ref_gate = O.vir_gate(x64, vl.numpy(), O.to64(inp["router"]))
    r = ivc.Router(inp["router"], pool_mode=pool_mode)
    gate, mask, offsets = ivc.vir_route(inp["x"].cuda(), vl.cuda(), inp["image_offsets"].cuda(), r)
    torch.cuda.synchronize()
    assert np.abs(to_np(gate) - ref_gate).max() <= GATE_ABS
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    res = ivc.flash_compress(inp["x"].cuda(), vl.cuda(), inp["image_offsets"].cuda(), m1, m2, r)
    torch.cuda.synchronize()
    g = to_np(res["gate"])
    assert np.abs(g - ref_gate).max() <= GATE_ABS
    ref_mask = O.route(g[:, 0].astype(np.float32).astype(np.float64), inp["image_offsets"].numpy())
    np.testing.assert_array_equal(to_np(res["mask"]), ref_mask)
    offs = O.compaction_offsets(ref_mask)
    np.testing.assert_array_equal(to_np(res["offsets"]), offs)
    # the connector processes every row of the grid, pad rows included
    Y256 = O.ps_project(x64, 0.5, O.to64(inp["mlp1"]))
    Y64 = O.ps_project(x64, 0.25, O.to64(inp["mlp2"]))
    for t in range(inp["T"]):
        ref = Y64[t] if ref_mask[t] else Y256[t]
        assert_connector_close(res["out"][offs[t]:offs[t + 1]], ref, f"tile {t}")


# ------------------------------------------------------------------ NaN input
@pytest.mark.parametrize("routed", [False, True])
def test_nan_feature_propagates_to_its_tile_and_image_only(routed):
    ivc = _ivc()
    inp = W.make(_small(tiles=(3, 4), var=0.0), affine="random")
    x = inp["x"].clone()
    x[1, 5, 9, 17] = float("nan")          # one channel of one token of tile 1 (image 0)
    inp["x"] = x
    T = inp["T"]
    m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
    r = ivc.Router(inp["router"])
    ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_FLASH, T, 256, m1, m2, r))
    res = ivc.flash_compress(x.cuda(), None, inp["image_offsets"].cuda(), m1, m2, r,
                             workspace=ws, routed=routed)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) == 0
    g = to_np(res["gate"])
    assert np.all(np.isnan(g[1])) and np.all(np.isfinite(np.delete(g, 1, axis=0)))
    x64 = O.to64(x)
    ref_gate = O.vir_gate(x64, inp["valid_len"].numpy(), O.to64(inp["router"]))
    assert np.all(np.isnan(ref_gate[1]))
    assert np.abs(np.delete(g, 1, axis=0) - np.delete(ref_gate, 1, axis=0)).max() <= GATE_ABS
    mask = to_np(res["mask"])
    assert mask[:3].sum() == 0             # image 0 holds the NaN gate
    ref_mask = O.route(g[:, 0].astype(np.float64), inp["image_offsets"].numpy())
    np.testing.assert_array_equal(mask, ref_mask)
    offs = O.compaction_offsets(ref_mask)
    np.testing.assert_array_equal(to_np(res["offsets"]), offs)
    Y256 = O.ps_project(x64, 0.5, O.to64(inp["mlp1"]))
    Y64 = O.ps_project(x64, 0.25, O.to64(inp["mlp2"]))
    for t in range(T):
        ref = (Y64[t] if ref_mask[t] else Y256[t]).reshape(-1, inp["H"])
        got = res["out"][offs[t]:offs[t + 1]].float().cpu().double().numpy()
        # the same rows are NaN on both sides (the row holding the NaN token)
        np.testing.assert_array_equal(np.isnan(got).any(axis=1), np.isnan(ref).any(axis=1))
        keep = ~np.isnan(ref).any(axis=1)
        if t == 1:
            assert (~keep).sum() == 1
        assert_connector_close(torch.from_numpy(got[keep]), ref[keep], f"tile {t}")
