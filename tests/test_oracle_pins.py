"""Pins of the fp64 oracle to things other than itself.

Each test checks the oracle against what the pages print (tests/golden), a
closed form, an invariant, a textbook/library routine (torch.nn modules and
numpy/torch quantile in float64, used here only as test dependencies) or brute
force on tiny inputs. A plausible slip anywhere in the oracle (a dropped term,
a wrong sign or index, a transposed operand) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")))
RNG = np.random.default_rng(20240601)


# ------------------------------------------------------------------ pixel_shuffle
def _ps_by_steps(x, scale, ps_version="v2"):
    """The page's four-step description, restated with torch views and axis
    swaps: merge neighbours along grid axis 2 into channels, swap the grid
    axes, merge neighbours along the (new) axis 2, swap back for v2.
    Returns the intermediate shapes too."""
    t = torch.from_numpy(x)
    n, w, h, c = t.shape
    shapes = [tuple(t.shape)]
    t = t.reshape(n, w, int(h * scale), int(c / scale))
    shapes.append(tuple(t.shape))
    t = t.transpose(1, 2).contiguous()
    shapes.append(tuple(t.shape))
    t = t.reshape(n, int(h * scale), int(w * scale), int(c / (scale * scale)))
    shapes.append(tuple(t.shape))
    if ps_version == "v2":
        t = t.transpose(1, 2).contiguous()
    return t.numpy(), shapes


@pytest.mark.parametrize("scale", [0.5, 0.25])
@pytest.mark.parametrize("ver", ["v2", "v1"])
def test_pixel_shuffle_matches_view_permute_steps(scale, ver):
    x = RNG.standard_normal((2, 32, 32, 8))
    ref, _ = _ps_by_steps(x, scale, ver)
    got = O.pixel_shuffle(x, scale, ver)
    g = int(32 * scale)
    assert got.shape == (2, g * g, int(8 / scale / scale))
    np.testing.assert_array_equal(got, ref.reshape(2, g * g, -1))


def test_pixel_shuffle_step_shapes_from_page():
    x = np.zeros((1, 32, 32, 1024), dtype=np.float32)
    _, shapes = _ps_by_steps(x, 0.5)
    assert [list(s) for s in shapes] == GOLD["pixel_shuffle_step_shapes"]["value"]
    assert O.pixel_shuffle(x, 0.5).shape == (1, 256, 4096)


def test_pixel_shuffle_token_counts_and_channels_from_page():
    tok, ch, grid = (GOLD[k]["value"] for k in ("tokens_per_tile", "channels_per_token", "output_grid"))
    x = np.zeros((1, 32, 32, 1024), dtype=np.float32)
    assert 32 * 32 == tok["vit"] and grid["vit"] == [32, 32]
    for key, s in (("ps_0.5", 0.5), ("ps_0.25", 0.25)):
        y = O.pixel_shuffle(x, s)
        assert y.shape[1] == tok[key] == grid[key][0] * grid[key][1]
        assert y.shape[2] == ch[key]
    q = O.pixel_shuffle_quarter(x)
    assert q.shape == (1, tok["ps_0.25"], ch["ps_0.25"])


@pytest.mark.parametrize("scale", [0.5, 0.25])
def test_pixel_shuffle_is_a_permutation(scale):
    x = np.arange(2 * 32 * 32 * 3, dtype=np.float64).reshape(2, 32, 32, 3)
    y = O.pixel_shuffle(x, scale)
    assert y.size == x.size
    np.testing.assert_array_equal(np.sort(y.ravel()), np.sort(x.ravel()))
    # each output token only holds elements of its own tile
    for t in range(2):
        np.testing.assert_array_equal(np.sort(y[t].ravel()), np.sort(x[t].ravel()))


def test_pixel_shuffle_explicit_entries():
    C = 5
    x = RNG.standard_normal((1, 32, 32, C))
    y = O.pixel_shuffle(x, 0.5)
    # output cell (a, b) = (3, 7), channel block (di, dj) = (1, 0) <- input (7, 14)
    assert y[0, 3 * 16 + 7, (2 * 1 + 0) * C + 4] == x[0, 7, 14, 4]
    assert y[0, 0, 1 * C + 2] == x[0, 0, 1, 2]          # (di,dj)=(0,1)
    assert y[0, 255, 3 * C + 0] == x[0, 31, 31, 0]      # last token, last block
    z = O.pixel_shuffle(x, 0.25)
    # cell (a, b) = (2, 5), (q, r) = (3, 1) <- input (11, 21)
    assert z[0, 2 * 8 + 5, (4 * 3 + 1) * C + 3] == x[0, 11, 21, 3]


@pytest.mark.parametrize("scale", [0.5, 0.25])
def test_pixel_shuffle_v1_is_transpose_of_v2(scale):
    x = RNG.standard_normal((3, 32, 32, 4))
    g = int(32 * scale)
    v1 = O.pixel_shuffle(x, scale, "v1").reshape(3, g, g, -1)
    v2 = O.pixel_shuffle(x, scale, "v2").reshape(3, g, g, -1)
    np.testing.assert_array_equal(v1, v2.transpose(0, 2, 1, 3))
    assert not np.array_equal(v1, v2)


def test_quarter_single_vs_twice_same_tokens_other_channel_order():
    x = RNG.standard_normal((1, 32, 32, 3))
    a = O.pixel_shuffle_quarter(x, "single")
    b = O.pixel_shuffle_quarter(x, "twice")
    assert a.shape == b.shape == (1, 64, 48)
    np.testing.assert_array_equal(np.sort(a, axis=-1), np.sort(b, axis=-1))
    assert not np.array_equal(a, b)


# ------------------------------------------------------------------ LN / GELU / MLP
def test_layer_norm_constant_row_gives_beta_and_library():
    g = RNG.standard_normal(16)
    b = RNG.standard_normal(16)
    v = np.full((3, 16), 2.5)
    np.testing.assert_allclose(O.layer_norm(v, g, b), np.broadcast_to(b, (3, 16)), atol=1e-12)
    v = RNG.standard_normal((5, 16)) * 3 + 1
    ref = torch.nn.functional.layer_norm(torch.from_numpy(v), (16,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-5).numpy()
    np.testing.assert_allclose(O.layer_norm(v, g, b), ref, rtol=1e-12, atol=1e-12)
    u = O.layer_norm(v, np.ones(16), np.zeros(16))
    np.testing.assert_allclose(u.mean(-1), 0, atol=1e-12)
    # biased variance: var(u) = var/(var+eps)
    var = v.var(-1)
    np.testing.assert_allclose(u.var(-1), var / (var + 1e-5), rtol=1e-12)


def test_gelu_closed_forms_and_library():
    assert O.gelu(np.array([0.0]))[0] == 0.0
    # GELU(1) = Phi(1)
    np.testing.assert_allclose(O.gelu(np.array([1.0]))[0], 0.8413447460685429, rtol=1e-15)
    z = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(O.gelu(z) - O.gelu(-z), z, atol=1e-14)
    ref = torch.nn.functional.gelu(torch.from_numpy(z), approximate="none").numpy()
    np.testing.assert_allclose(O.gelu(z), ref, rtol=1e-13, atol=1e-15)


def _mlp_brute(P, g, b, Ws, bs):
    """Textbook loops on tiny shapes."""
    M, K = P.shape
    out = []
    for m in range(M):
        row = list(P[m])
        mu = sum(row) / K
        var = sum((r - mu) ** 2 for r in row) / K
        h = [(row[k] - mu) / math.sqrt(var + 1e-5) * g[k] + b[k] for k in range(K)]
        for i, (Wi, bi) in enumerate(zip(Ws, bs)):
            nh = []
            for n in range(Wi.shape[0]):
                acc = bi[n]
                for k in range(Wi.shape[1]):
                    acc += Wi[n, k] * h[k]
                if i + 1 < len(Ws):
                    acc = 0.5 * acc * (1 + math.erf(acc / math.sqrt(2)))
                nh.append(acc)
            h = nh
        out.append(h)
    return np.array(out)


@pytest.mark.parametrize("dims", [[8, 6, 6], [12, 7, 5, 4]])
def test_mlp_brute_force(dims):
    P = RNG.standard_normal((5, dims[0])) * 2 + 0.3
    g = 1 + 0.1 * RNG.standard_normal(dims[0])
    b = 0.1 * RNG.standard_normal(dims[0])
    Ws = [RNG.standard_normal((dims[i + 1], dims[i])) * 0.5 for i in range(len(dims) - 1)]
    bs = [RNG.standard_normal(dims[i + 1]) * 0.1 for i in range(len(dims) - 1)]
    np.testing.assert_allclose(O.mlp(P, g, b, Ws, bs), _mlp_brute(P, g, b, Ws, bs), rtol=1e-12, atol=1e-12)


def test_mlp1_matches_torch_sequential():
    K, H = 32, 24
    seq = torch.nn.Sequential(torch.nn.LayerNorm(K), torch.nn.Linear(K, H), torch.nn.GELU(),
                              torch.nn.Linear(H, H)).double()
    with torch.no_grad():
        for p in seq.parameters():
            p.copy_(torch.randn(p.shape, dtype=torch.float64) * 0.3)
    P = RNG.standard_normal((9, K))
    ref = seq(torch.from_numpy(P)).detach().numpy()
    got = O.mlp(P, seq[0].weight.detach().numpy(), seq[0].bias.detach().numpy(),
                [seq[1].weight.detach().numpy(), seq[3].weight.detach().numpy()],
                [seq[1].bias.detach().numpy(), seq[3].bias.detach().numpy()])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_mlp1_param_count_and_num_image_token_from_page():
    gold = GOLD["mlp1_params_14b"]["value"]
    w = W.WORKLOADS["connector_14b_832tiles"]
    shapes = [(w.H, 4 * w.C), (w.H, w.H)]  # the weight shapes the oracle's mlp1 consumes
    count = sum(a * b for a, b in shapes)
    assert (4 * w.C, w.H) == (gold["in"], gold["hidden"])
    assert count == 47_185_920 and round(count / 1e6, 1) == gold["params_millions"]
    nit = GOLD["num_image_token"]["value"]
    x = np.zeros((1, nit["image_size"] // nit["patch_size"], nit["image_size"] // nit["patch_size"], 2))
    assert O.pixel_shuffle(x, nit["downsample_ratio"]).shape[1] == nit["tokens"]
    w4 = W.WORKLOADS["flash_4b_batched"]
    assert (4 * w4.C, w4.H) == tuple(GOLD["mlp1_dims_4b"]["value"].values())
    m2 = GOLD["mlp2_dims_2b_flash"]["value"]
    w2 = W.WORKLOADS["flash_2b_13tiles"]
    assert (16 * w2.C, w2.mlp2_mid, w2.H) == (m2["in"], m2["mid"], m2["out"])


def test_ps_project_end_to_end_tiny_brute():
    C, H = 2, 3
    x = RNG.standard_normal((1, 32, 32, C))
    prm = {"ln_g": 1 + 0.1 * RNG.standard_normal(4 * C), "ln_b": 0.1 * RNG.standard_normal(4 * C),
           "W": [RNG.standard_normal((H, 4 * C)), RNG.standard_normal((H, H))],
           "b": [RNG.standard_normal(H), RNG.standard_normal(H)]}
    Y = O.ps_project(x, 0.5, prm)
    # token (a,b) = (5, 9): gather the 2x2 block by hand, then brute-force MLP
    a, b = 5, 9
    P = np.concatenate([x[0, 2 * a + di, 2 * b + dj] for di in range(2) for dj in range(2)])[None]
    np.testing.assert_allclose(Y[0, a * 16 + b], _mlp_brute(P, prm["ln_g"], prm["ln_b"], prm["W"], prm["b"])[0],
                               rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ pooling
def _router(D=32, heads=4, layers=4, blocks=4, hid=24, seed=0):
    r = np.random.default_rng(seed)
    p = {"D": D, "heads": heads, "query": r.standard_normal(D)}
    for k in ("Wq", "Wk", "Wv", "Wo"):
        p[k] = [r.standard_normal((D, D)) * 0.3 for _ in range(layers)]
    for k in ("bq", "bk", "bv", "bo"):
        p[k] = [r.standard_normal(D) * 0.1 for _ in range(layers)]
    p["gW1"] = [r.standard_normal((hid, D)) * 0.3 for _ in range(blocks)]
    p["gb1"] = [r.standard_normal(hid) * 0.1 for _ in range(blocks)]
    p["gW2"] = [r.standard_normal((D, hid)) * 0.3 for _ in range(blocks)]
    p["gb2"] = [r.standard_normal(D) * 0.1 for _ in range(blocks)]
    p["gln_g"] = [1 + 0.1 * r.standard_normal(D) for _ in range(blocks)]
    p["gln_b"] = [0.1 * r.standard_normal(D) for _ in range(blocks)]
    p["gWout"] = r.standard_normal((2, D)) * 0.3
    p["gbout"] = r.standard_normal(2) * 0.1
    return p


def test_pooling_single_valid_token_reduces_to_out_proj_of_v():
    r = _router()
    X = RNG.standard_normal((3, 10, 32))
    lens = np.array([1, 1, 1])
    got = O.cross_attention_pooling(X, lens, r)
    for t in range(3):
        v = r["Wv"][3] @ X[t, 0] + r["bv"][3]
        np.testing.assert_allclose(got[t], r["Wo"][3] @ v + r["bo"][3], rtol=1e-12, atol=1e-12)


def test_pooling_zero_keys_give_mean_of_values():
    r = _router(layers=1)
    r["Wk"][0][:] = 0
    r["bk"][0][:] = 0
    X = RNG.standard_normal((2, 12, 32))
    lens = np.array([12, 5])
    got = O.cross_attention_pooling(X, lens, r)
    for t, n in enumerate(lens):
        v = X[t, :n] @ r["Wv"][0].T + r["bv"][0]
        np.testing.assert_allclose(got[t], r["Wo"][0] @ v.mean(0) + r["bo"][0], rtol=1e-12, atol=1e-12)


def test_pooling_ignores_padding_values():
    r = _router()
    X = RNG.standard_normal((2, 16, 32))
    lens = np.array([16, 9])
    a = O.cross_attention_pooling(X, lens, r)
    X2 = X.copy()
    X2[1, 9:] = 1e3 * RNG.standard_normal((7, 32))
    b = O.cross_attention_pooling(X2, lens, r)
    np.testing.assert_array_equal(a, b)


def test_pooling_matches_torch_multihead_attention_chain():
    D, Hh = 32, 4
    r = _router(D=D, heads=Hh)
    X = RNG.standard_normal((3, 20, D))
    lens = np.array([20, 13, 1])
    mask = torch.from_numpy(np.arange(20)[None, :] >= lens[:, None])
    q = torch.from_numpy(np.broadcast_to(r["query"], (3, 1, D)).copy())
    Xt = torch.from_numpy(X)
    for l in range(4):
        mha = torch.nn.MultiheadAttention(D, Hh, batch_first=True, dtype=torch.float64)
        with torch.no_grad():
            mha.in_proj_weight.copy_(torch.from_numpy(np.concatenate([r["Wq"][l], r["Wk"][l], r["Wv"][l]])))
            mha.in_proj_bias.copy_(torch.from_numpy(np.concatenate([r["bq"][l], r["bk"][l], r["bv"][l]])))
            mha.out_proj.weight.copy_(torch.from_numpy(r["Wo"][l]))
            mha.out_proj.bias.copy_(torch.from_numpy(r["bo"][l]))
        q, _ = mha(q, Xt, Xt, key_padding_mask=mask, need_weights=False)
    np.testing.assert_allclose(O.cross_attention_pooling(X, lens, r), q[:, 0].detach().numpy(),
                               rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------------ gating
def _pool_chunked(X, valid_len, r, rescale=True, merge=True, chunk=128, step=32):
    """Single-query pooling in the single-pass form (fp64): per layer and head
    the key projection folded into the query (u, c), per chunk of `chunk` tokens
    a running max m and sum l over steps of `step` tokens with the weighted sum
    kept relative to m, chunks without a valid token skipped, chunks merged
    with weights exp(m_c - M); the value projection applied to the merged sum."""
    T, N, D = X.shape
    H = int(r["heads"])
    dh = D // H
    q = np.broadcast_to(r["query"], (T, D)).copy()
    for l in range(len(r["Wq"])):
        Q = q @ r["Wq"][l].T + r["bq"][l]
        o = np.zeros((T, D))
        for t in range(T):
            n = int(valid_len[t])
            for h in range(H):
                sl = slice(h * dh, (h + 1) * dh)
                u = r["Wk"][l][sl].T @ Q[t, sl] / math.sqrt(dh)
                c = r["bk"][l][sl] @ Q[t, sl] / math.sqrt(dh)
                parts = []
                for c0 in range(0, N, chunk):
                    m, lsum, z = -math.inf, 0.0, np.zeros(D)
                    for s0 in range(c0, min(c0 + chunk, n), step):
                        xs = X[t, s0:min(s0 + step, n)]
                        sc = xs @ u + c
                        m_new = max(m, float(sc.max()))
                        f = math.exp(m - m_new) if rescale else 1.0
                        e = np.exp(sc - m_new)
                        lsum, z, m = lsum * f + e.sum(), z * f + e @ xs, m_new
                    if lsum > 0:
                        parts.append((m, lsum, z))
                M = max(pm for pm, _, _ in parts)
                w = [math.exp(pm - M) if merge else 1.0 for pm, _, _ in parts]
                zt = sum(wi * pz for wi, (_, _, pz) in zip(w, parts)) / \
                    sum(wi * pl for wi, (_, pl, _) in zip(w, parts))
                o[t, sl] = r["Wv"][l][sl] @ zt + r["bv"][l][sl]
        q = o @ r["Wo"][l].T + r["bo"][l]
    return q


def test_pooling_single_pass_form_equals_definition():
    """The reassociation the pooling kernels compute (folded key projection,
    running softmax per 128-token chunk, chunks merged) equals the oracle's
    attention to rounding, including a one-token tile and a tile whose second
    chunk holds a single valid token; dropping the running rescale or the
    max-relative merge weights breaks it."""
    rng = np.random.default_rng(11)
    T, N, D, H = 3, 1024, 128, 2

    def mat(o, i):
        return rng.normal(size=(o, i)) / math.sqrt(i)

    r = {"heads": H, "query": rng.normal(size=D)}
    for k in ("Wq", "Wk", "Wv", "Wo"):
        r[k] = [mat(D, D) for _ in range(4)]
    for k in ("bq", "bk", "bv", "bo"):
        r[k] = [0.1 * rng.normal(size=D) for _ in range(4)]
    # growing scale along the tokens: the running max changes from chunk to chunk
    X = rng.normal(size=(T, N, D)) * np.linspace(1.0, 4.0, N)[None, :, None]
    vl = np.array([1, 129, 1024])
    ref = O.cross_attention_pooling(X, vl, r)
    np.testing.assert_allclose(_pool_chunked(X, vl, r), ref, rtol=1e-9, atol=1e-12)
    assert not np.allclose(_pool_chunked(X, vl, r, rescale=False), ref, rtol=1e-3)
    assert not np.allclose(_pool_chunked(X, vl, r, merge=False), ref, rtol=1e-3)


def test_gating_rows_sum_to_one_and_sigmoid_identity():
    r = _router()
    h = RNG.standard_normal((7, 32))
    p = O.gating(h, r)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-15)
    # recompute the logits' difference through the 2-way softmax identity
    z = np.log(p[:, 0]) - np.log(p[:, 1])
    np.testing.assert_allclose(p[:, 0], 1 / (1 + np.exp(-z)), rtol=1e-14)


def test_gating_matches_torch_modules():
    D, hid = 32, 24
    r = _router(D=D, hid=hid)
    h0 = RNG.standard_normal((6, D))
    h = torch.from_numpy(h0)
    for b in range(4):
        l1 = torch.nn.Linear(D, hid).double()
        l2 = torch.nn.Linear(hid, D).double()
        ln = torch.nn.LayerNorm(D).double()
        with torch.no_grad():
            l1.weight.copy_(torch.from_numpy(r["gW1"][b])); l1.bias.copy_(torch.from_numpy(r["gb1"][b]))
            l2.weight.copy_(torch.from_numpy(r["gW2"][b])); l2.bias.copy_(torch.from_numpy(r["gb2"][b]))
            ln.weight.copy_(torch.from_numpy(r["gln_g"][b])); ln.bias.copy_(torch.from_numpy(r["gln_b"][b]))
        blk = torch.nn.Sequential(l1, torch.nn.GELU(), torch.nn.Dropout(0.1), l2, torch.nn.Dropout(0.1), ln).eval()
        h = h + blk(h)
    out = torch.nn.Linear(D, 2).double()
    with torch.no_grad():
        out.weight.copy_(torch.from_numpy(r["gWout"])); out.bias.copy_(torch.from_numpy(r["gbout"]))
    ref = torch.softmax(out(h), dim=-1).detach().numpy()
    np.testing.assert_allclose(O.gating(h0, r), ref, rtol=1e-12, atol=1e-14)


def test_gating_inside_variant_matches_torch_modules():
    """The other reading of a Gating block: LayerNorm applied to the residual
    sum, h <- LN(h + W2 GELU(W1 h + b1) + b2), checked against torch modules."""
    D, hid = 32, 24
    r = _router(D=D, hid=hid)
    h0 = RNG.standard_normal((5, D))
    h = torch.from_numpy(h0)
    for b in range(4):
        l1 = torch.nn.Linear(D, hid).double()
        l2 = torch.nn.Linear(hid, D).double()
        ln = torch.nn.LayerNorm(D).double()
        with torch.no_grad():
            l1.weight.copy_(torch.from_numpy(r["gW1"][b])); l1.bias.copy_(torch.from_numpy(r["gb1"][b]))
            l2.weight.copy_(torch.from_numpy(r["gW2"][b])); l2.bias.copy_(torch.from_numpy(r["gb2"][b]))
            ln.weight.copy_(torch.from_numpy(r["gln_g"][b])); ln.bias.copy_(torch.from_numpy(r["gln_b"][b]))
            h = ln(h + l2(torch.nn.functional.gelu(l1(h))))
    out = torch.nn.Linear(D, 2).double()
    with torch.no_grad():
        out.weight.copy_(torch.from_numpy(r["gWout"])); out.bias.copy_(torch.from_numpy(r["gbout"]))
    ref = torch.softmax(out(h), dim=-1).detach().numpy()
    got = O.gating(h0, r, residual="inside")
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    # the two readings differ (a swapped branch would pass one test, not both)
    assert np.abs(got - O.gating(h0, r)).max() > 1e-3


# ------------------------------------------------------------------ quantile / routing
@pytest.mark.parametrize("n", [1, 2, 3, 5, 11, 13, 64, 257])
def test_quantile_matches_numpy_and_torch(n):
    v = RNG.random(n)
    for q in (0.0, 0.1, 0.37, 0.5, 1.0):
        got = O.quantile_linear(v, q)
        np.testing.assert_allclose(got, np.quantile(v, q, method="linear"), rtol=1e-15, atol=1e-16)
        np.testing.assert_allclose(got, torch.quantile(torch.from_numpy(v), q).item(), rtol=1e-15, atol=1e-16)


def test_quantile_nan_propagates_like_torch():
    """A NaN gate makes torch.quantile NaN (the pages' threshold); the oracle
    follows, and then no tile of the group passes the strict > test."""
    rng = np.random.default_rng(5)
    for n in (1, 2, 5, 13):
        v = rng.random(n)
        v[rng.integers(n)] = np.nan
        ref = torch.quantile(torch.from_numpy(v), 0.1).item()
        assert math.isnan(ref)
        assert math.isnan(O.quantile_linear(v, 0.1))
        mask = O.route(np.concatenate([v, [0.9, 0.8, 0.3]]), np.array([0, n, n + 3]))
        assert mask[:n].sum() == 0               # the image holding the NaN
        assert mask[n:].tolist() == [1, 1, 0]     # the other image is untouched
    # batch scope: one NaN anywhere disables compression for the batch
    g = np.array([0.9, 0.8, np.nan, 0.7])
    assert O.route(g, np.array([0, 4]), scope="batch").sum() == 0


def test_quantile_brute_cases():
    assert O.quantile_linear([0.7], 0.1) == 0.7
    v = np.array([5., 1., 4., 2., 3., 9., 8., 7., 6., 0., 10.])  # n = 11, pos = 1.0 exactly
    assert O.quantile_linear(v, 0.1) == 1.0
    assert O.quantile_linear(v, 0.0) == 0.0 and O.quantile_linear(v, 1.0) == 10.0
    # n = 13 (12 tiles + thumbnail): pos = 1.2 -> v[1] + 0.2 (v[2] - v[1])
    v13 = np.arange(13, dtype=np.float64) * 0.05
    np.testing.assert_allclose(O.quantile_linear(v13[::-1], 0.1), 0.05 + 0.2 * 0.05, rtol=1e-14)


def test_route_semantics():
    th = GOLD["thresholds"]["value"]
    rel, ab = th["flash_relative_threshold"], th["flash_absolute_threshold"]
    # single-tile image: g > quantile(g) is false -> never compressed
    assert O.route(np.array([0.99]), np.array([0, 1]), rel, ab).tolist() == [0]
    # strict > at the quantile, >= at 0.5
    g = np.array([0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5])
    assert O.route(g, np.array([0, 11]), rel, ab).sum() == 0       # all tie the quantile
    g = np.array([0.4, 0.5, 0.5, 0.6, 0.7, 0.8, 0.9, 0.95, 0.96, 0.97, 0.98])  # q = 0.5 (pos=1)
    m = O.route(g, np.array([0, 11]), rel, ab)
    assert m.tolist() == [0, 0, 0, 1, 1, 1, 1, 1, 1, 1, 1]
    g = np.array([0.1, 0.2, 0.3, 0.45, 0.49])
    assert O.route(g, np.array([0, 5]), rel, ab).sum() == 0      # all below 0.5
    # per image vs whole batch
    g = np.array([0.9, 0.95, 0.6, 0.7])
    per = O.route(g, np.array([0, 2, 4]), rel, ab)
    bat = O.route(g, np.array([0, 2, 4]), rel, ab, scope="batch")
    assert per.tolist() == [0, 1, 0, 1] and bat.tolist() == [1, 1, 0, 1]


def test_compaction_length_and_rows():
    gold = GOLD["compressed_tile"]["value"]
    T, H = 9, 3
    Y256 = RNG.standard_normal((T, 256, H))
    Y64 = RNG.standard_normal((T, 64, H))
    mask = np.array([1, 0, 0, 1, 1, 0, 1, 0, 0], dtype=np.uint8)
    offs = O.compaction_offsets(mask)
    k = int(mask.sum())
    assert offs[-1] == 256 * (T - k) + 64 * k == T * gold["placeholders"] - k * gold["deleted"]
    out = O.compact(Y256, Y64, mask)
    assert out.shape == (offs[-1], H)
    for t in range(T):
        src = Y64[t] if mask[t] else Y256[t]
        np.testing.assert_array_equal(out[offs[t]:offs[t + 1]], src)
    wc = GOLD["worst_case_image_tokens"]["value"]
    assert O.compaction_offsets(np.zeros(wc["tiles"], np.uint8))[-1] == wc["after"]
    assert wc["tiles"] * 1024 == wc["before"]


def test_flash_compress_small_composes_steps():
    D = 32
    r = _router(D=D, heads=4)
    x = RNG.standard_normal((4, 32, 32, D))
    lens = np.array([1024, 700, 1024, 300])
    offs = np.array([0, 3, 4])
    mlp1 = {"ln_g": np.ones(4 * D), "ln_b": np.zeros(4 * D),
            "W": [RNG.standard_normal((16, 4 * D)) * 0.1, RNG.standard_normal((16, 16)) * 0.1],
            "b": [np.zeros(16), np.zeros(16)]}
    mlp2 = {"ln_g": np.ones(16 * D), "ln_b": np.zeros(16 * D),
            "W": [RNG.standard_normal((24, 16 * D)) * 0.1, RNG.standard_normal((16, 24)) * 0.1,
                  RNG.standard_normal((16, 16)) * 0.1],
            "b": [np.zeros(24), np.zeros(16), np.zeros(16)]}
    res = O.flash_compress(x, lens, offs, mlp1, mlp2, r)
    k = int(res["mask"].sum())
    assert res["out"].shape == (256 * (4 - k) + 64 * k, 16)
    assert res["Y256"].shape == (4, 256, 16) and res["Y64"].shape == (4, 64, 16)
    np.testing.assert_allclose(res["gate"].sum(-1), 1, atol=1e-15)
    # gate override routes on the given vector
    res2 = O.flash_compress(x, lens, offs, mlp1, mlp2, r, gate_override=np.array([0.9, 0.95, 0.99, 0.2]))
    assert res2["mask"].tolist() == [0, 1, 1, 0]


# ------------------------------------------------------------------ sequence assembly
def test_assemble_worked_example_scaled_down():
    """Hand-built example with 4 placeholders per tile, 1 kept when compressed
    (the same rule as 256 / 64, scaled down): ids 5 [9 9 9 9] [9 9 9 9] 7 with
    tile 0 compressed gives 5 9 9 9 9 9 7; tile 0's one row, then tile 1's
    four rows, then the table row of 7."""
    tab = np.arange(10 * 3, dtype=np.float64).reshape(10, 3)
    vis = 100.0 + np.arange(5 * 3, dtype=np.float64).reshape(5, 3)
    ids = np.array([5, 9, 9, 9, 9, 9, 9, 9, 9, 7])
    res = O.assemble_sequence(ids, [0, 10], 9, tab, vis, mask=[1, 0], offsets=[0, 1, 5],
                              keep=1, full=4)
    np.testing.assert_array_equal(res["ids"], [5, 9, 9, 9, 9, 9, 7])
    expect = np.stack([tab[5], vis[0], vis[1], vis[2], vis[3], vis[4], tab[7]])
    np.testing.assert_array_equal(res["embeds"], expect)
    np.testing.assert_array_equal(res["positions"], np.arange(7))
    np.testing.assert_array_equal(res["seq_offsets"], [0, 7])
    assert res["placeholders"] == 8


def _prompt(tiles_per_seq, text=(3, 2), img_id=7, V=50, seed=0):
    rng = np.random.default_rng(seed)
    ids, offs = [], [0]
    for n in tiles_per_seq:
        seq = list(rng.integers(10, V, text[0])) + [img_id] * (256 * n) + list(rng.integers(10, V, text[1]))
        ids += seq
        offs.append(len(ids))
    return np.array(ids), np.array(offs)


def test_assemble_lengths_follow_the_page_counts():
    """Every compressed tile removes 192 of its 256 placeholders; uncompressed
    tiles keep all 256 (page numbers in tests/golden)."""
    g = GOLD["compressed_tile"]["value"]
    tiles = [3, 1, 2]
    ids, offs = _prompt(tiles)
    T = sum(tiles)
    mask = np.array([1, 0, 1, 0, 0, 1])
    vis_offs = O.compaction_offsets(mask)
    H = 4
    tab = RNG.standard_normal((50, H))
    vis = RNG.standard_normal((int(vis_offs[-1]), H))
    res = O.assemble_sequence(ids, offs, 7, tab, vis, mask, vis_offs)
    k = int(mask.sum())
    assert len(res["ids"]) == len(ids) - g["deleted"] * k
    # per sequence: the tiles of sequence b are consecutive
    t0 = 0
    for b, n in enumerate(tiles):
        kb = int(mask[t0:t0 + n].sum())
        assert res["seq_offsets"][b + 1] - res["seq_offsets"][b] == (offs[b + 1] - offs[b]) - 192 * kb
        seg = res["positions"][res["seq_offsets"][b]:res["seq_offsets"][b + 1]]
        np.testing.assert_array_equal(seg, np.arange(len(seg)))
        t0 += n
    # the kept placeholders take every visual row exactly once, in order
    sel = res["ids"] == 7
    np.testing.assert_array_equal(res["embeds"][sel], vis)
    assert sel.sum() == g["placeholders"] * (T - k) + g["kept"] * k
    np.testing.assert_array_equal(res["embeds"][~sel], tab[res["ids"][~sel]])


def test_assemble_no_compression_is_plain_injection():
    """With no tile compressed the result is the plain injection of [PS]
    "视觉 Token 如何注入": input_embeds[ids == IMG_CONTEXT] = visual rows."""
    ids, offs = _prompt([2])
    H = 3
    tab = RNG.standard_normal((50, H))
    vis = RNG.standard_normal((512, H))
    res = O.assemble_sequence(ids, offs, 7, tab, vis, [0, 0], [0, 256, 512])
    ref = tab[ids].copy()
    ref[ids == 7] = vis
    np.testing.assert_array_equal(res["ids"], ids)
    np.testing.assert_array_equal(res["embeds"], ref)


def test_assemble_extra_placeholders_stay_text():
    ids, offs = _prompt([1])
    ids = np.concatenate([ids, [7, 7]])
    offs = np.array([0, len(ids)])
    tab = RNG.standard_normal((50, 2))
    vis = RNG.standard_normal((64, 2))
    res = O.assemble_sequence(ids, offs, 7, tab, vis, [1], [0, 64])
    assert res["placeholders"] == 258
    np.testing.assert_array_equal(res["embeds"][-2:], tab[[7, 7]])
