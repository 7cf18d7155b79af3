"""The C ABI loads and exports what include/ivc.h declares; host-side argument
checks return their codes before any GPU work (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ivc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ivc_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_three_calls():
    names = _declared()
    for n in ("ivc_ps_project", "ivc_vir_route", "ivc_flash_compress", "ivc_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    for n in _declared():
        assert hasattr(L, n), n
    assert L.ivc_version() >= 100


def test_trace_without_records_needs_no_gpu():
    """The tracing calls only touch CUDA for recorded launches: with none, the
    report is an empty object and a too-small buffer is refused."""
    import vlm_visual_token_b200 as ivc
    ivc.trace_enable(False)
    ivc.trace_reset()
    assert ivc.trace_report() == {}
    with pytest.raises(ivc.IvcError):
        ivc.trace_report(max_bytes=1)


def test_status_strings():
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert L.ivc_strerror(code).decode() not in ("", "unknown status")


def _mlp(dims):
    import vlm_visual_token_b200 as ivc
    c = ivc._CMlp()
    c.n_linear = len(dims) - 1
    for i, d in enumerate(dims):
        c.dims[i] = d
    c.ln_gamma = c.ln_beta = 256
    for i in range(c.n_linear):
        c.W[i] = 256 * (i + 2)
        c.b[i] = 256
    return c


def test_workspace_size_and_shape_checks():
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    m1 = _mlp([4096, 2048, 2048])
    m2 = _mlp([16384, 4096, 2048, 2048])
    n1 = L.ivc_workspace_size(ivc.OP_PS_HALF, 13, 1024, ctypes.byref(m1), None, None)
    n2 = L.ivc_workspace_size(ivc.OP_PS_HALF, 26, 1024, ctypes.byref(m1), None, None)
    assert n1 > 0 and n2 > n1
    # at least the hidden activations [T*256, H] bf16 and the row statistics
    assert n1 >= 13 * 256 * 2048 * 2 + 2 * 13 * 256 * 4
    assert L.ivc_workspace_size(ivc.OP_PS_QUARTER, 13, 1024, ctypes.byref(m2), None, None) > 0
    bad = _mlp([4096, 2000, 2048])   # width not a multiple of 64
    assert L.ivc_workspace_size(ivc.OP_PS_HALF, 1, 1024, ctypes.byref(bad), None, None) == 0
    assert L.ivc_workspace_size(99, 1, 1024, ctypes.byref(m1), None, None) == 0
    assert L.ivc_workspace_size(ivc.OP_PS_HALF, -1, 1024, ctypes.byref(m1), None, None) == 0


def test_entry_points_reject_bad_arguments_without_touching_the_gpu():
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    m1 = _mlp([4096, 2048, 2048])
    ws = ctypes.c_void_p(1 << 20)
    x = ctypes.c_void_p(1 << 24)
    y = ctypes.c_void_p(1 << 26)
    P = ctypes.byref
    # bad scale, bad flags
    assert L.ivc_ps_project(x, 1, 1024, ctypes.c_float(0.3), 0, P(m1), y, ws, 1 << 40, None) == -1
    assert L.ivc_ps_project(x, 1, 1024, ctypes.c_float(0.5), 8, P(m1), y, ws, 1 << 40, None) == -1
    # C not a multiple of 64; dims[0] != 4C
    assert L.ivc_ps_project(x, 1, 1000, ctypes.c_float(0.5), 0, P(m1), y, ws, 1 << 40, None) == -2
    assert L.ivc_ps_project(x, 1, 512, ctypes.c_float(0.5), 0, P(m1), y, ws, 1 << 40, None) == -2
    # null input, misaligned input, small workspace
    assert L.ivc_ps_project(None, 1, 1024, ctypes.c_float(0.5), 0, P(m1), y, ws, 1 << 40, None) == -1
    assert L.ivc_ps_project(ctypes.c_void_p((1 << 24) + 8), 1, 1024, ctypes.c_float(0.5), 0, P(m1),
                            y, ws, 1 << 40, None) == -6
    assert L.ivc_ps_project(x, 1, 1024, ctypes.c_float(0.5), 0, P(m1), y, ws, 16, None) == -3
    # negative tile count
    assert L.ivc_ps_project(x, -2, 1024, ctypes.c_float(0.5), 0, P(m1), y, ws, 1 << 40, None) == -1
    # router: D must equal C and be 64 x heads
    r = ivc._CRouter()
    r.D, r.heads, r.gate_hidden = 1024, 8, 1024
    assert L.ivc_vir_route(x, None, 1, 1024, x, 1, P(r), y, y, y, ws, 1 << 40, None) == -2
    r.heads = 16
    assert L.ivc_vir_route(x, None, 1, 512, x, 1, P(r), y, y, y, ws, 1 << 40, None) == -2
    r.quantile_scope = 3
    assert L.ivc_vir_route(x, None, 1, 1024, x, 1, P(r), y, y, y, ws, 1 << 40, None) == -1


@pytest.mark.parametrize("name", ["ivc_flash_compress", "ivc_flash_compress_routed"])
def test_flash_entry_points_reject_bad_arguments(name):
    """Both flash flows share their argument checks; none reaches the GPU."""
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    fn = getattr(L, name)
    m1 = _mlp([4096, 2048, 2048])
    m2 = _mlp([16384, 4096, 2048, 2048])
    m2_bad = _mlp([16384, 4096, 2048, 1024])  # output width differs from mlp1's
    r = ivc._CRouter()
    r.D, r.heads, r.gate_hidden = 1024, 16, 1024
    r.query = r.gWout = 1 << 28
    for k in ("Wq", "Wk", "Wv", "Wo", "gW1", "gW2", "gln_g", "gln_b"):
        arr = getattr(r, k)
        for l in range(4):
            arr[l] = 1 << 28
    ws = ctypes.c_void_p(1 << 20)
    x = ctypes.c_void_p(1 << 24)
    y = ctypes.c_void_p(1 << 26)
    P = ctypes.byref

    def call(T=1, C=1024, mlp2=m2, out=y, nbytes=1 << 40, xx=x):
        return fn(xx, None, T, C, x, 1, P(m1), P(mlp2), P(r), out, y, y, y, y, ws, nbytes, None)

    assert call(T=-1) == -1
    assert call(mlp2=m2_bad) == -2
    assert call(C=512) == -2
    assert call(out=None) == -1
    assert call(out=ctypes.c_void_p((1 << 26) + 4)) == -6
    assert call(nbytes=64) == -3
    assert call(xx=ctypes.c_void_p((1 << 24) + 2)) == -6


def test_route_rejects_bad_arguments_without_touching_the_gpu():
    """ivc_route (the double threshold on a given gate vector) checks its
    arguments on the host; rel_q outside [0, 1] would index past the sorted
    gates, so it is refused, for ivc_vir_route too."""
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    g = ctypes.c_void_p(1 << 24)
    o = ctypes.c_void_p(1 << 25)
    m = ctypes.c_void_p(1 << 26)
    ws = ctypes.c_void_p(1 << 20)

    def call(T=4, offs=o, I=1, rel_q=0.1, scope=0, mask=m, offsets=o, ws=ws, nbytes=256):
        return L.ivc_route(g, T, offs, I, rel_q, 0.5, scope, mask, offsets, None, ws, nbytes, None)

    assert call(rel_q=1.5) == -1
    assert call(rel_q=-0.1) == -1
    assert call(rel_q=float("nan")) == -1
    assert call(scope=2) == -1
    assert call(T=-1) == -1
    assert call(offsets=None) == -1
    assert call(mask=None) == -1
    assert call(offs=None) == -1                 # per-image scope needs the offsets
    assert call(nbytes=128) == -3                # the status word needs 256 bytes
    assert call(ws=ctypes.c_void_p((1 << 20) + 64)) == -6
    r = ivc._CRouter()
    r.D, r.heads, r.gate_hidden = 1024, 16, 1024
    r.rel_q = 2.0
    x = ctypes.c_void_p(1 << 24)
    y = ctypes.c_void_p(1 << 26)
    assert L.ivc_vir_route(x, None, 1, 1024, x, 1, ctypes.byref(r), y, y, y, ws, 1 << 40,
                           None) == -1


def _router_struct(ivc, D=1024):
    r = ivc._CRouter()
    r.D, r.heads, r.gate_hidden = D, D // 64, 1024
    r.query = r.gWout = 1 << 28
    for k in ("Wq", "Wk", "Wv", "Wo", "gW1", "gW2", "gln_g", "gln_b"):
        arr = getattr(r, k)
        for l in range(4):
            arr[l] = 1 << 28
    return r


def test_router_fold_size_and_argument_checks_without_touching_the_gpu():
    """ivc_router_fold (InternVL3_5-4B-Flash article, section 2: the pooling
    layers chain with nothing between Wo_l and Wq_{l+1}): its buffer holds the
    first layer's query (fp32 D), its split key fold (bf16 32 x D) and bias
    term (fp32 16), and per later layer P = Wq Wo as a bf16 hi | lo pair
    (D x 2D) with its fp32 bias (D), each piece 256-byte aligned. Every check
    runs before the GPU is touched."""
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    P = ctypes.byref
    r = _router_struct(ivc)

    def a(n):
        return (n + 255) // 256 * 256

    D = 1024
    want = a(4 * D) + a(2 * 32 * D) + a(4 * 16) + 3 * (a(2 * 2 * D * D) + a(4 * D))
    assert L.ivc_router_fold_size(P(r)) == want
    lit = _router_struct(ivc)
    lit.pool_mode = 1
    assert L.ivc_router_fold_size(P(lit)) == 0
    dst = ctypes.c_void_p(1 << 30)
    assert L.ivc_router_fold(P(lit), dst, want, None) == -2
    assert L.ivc_router_fold(P(r), None, want, None) == -1
    assert L.ivc_router_fold(P(r), ctypes.c_void_p((1 << 30) + 16), want, None) == -6
    assert L.ivc_router_fold(P(r), dst, want - 1, None) == -3
    no_query = _router_struct(ivc)
    no_query.query = None
    assert L.ivc_router_fold(P(no_query), dst, want, None) == -1
    # the fold fields are all or none, and only with folded pooling
    part = _router_struct(ivc)
    part.fold_u1 = 1 << 29
    x = ctypes.c_void_p(1 << 24)
    y = ctypes.c_void_p(1 << 26)
    ws = ctypes.c_void_p(1 << 20)
    assert L.ivc_vir_route(x, None, 1, 1024, x, 1, P(part), y, y, y, ws, 1 << 40, None) == -1
    full = _router_struct(ivc)
    full.fold_u1 = full.fold_c1 = 1 << 29
    for l in range(3):
        full.fold_wqo[l] = full.fold_bqo[l] = 1 << 29
    full.pool_mode = 1
    assert L.ivc_vir_route(x, None, 1, 1024, x, 1, P(full), y, y, y, ws, 1 << 40, None) == -1
    full.fold_c1 = (1 << 29) + 4
    full.pool_mode = 0
    assert L.ivc_vir_route(x, None, 1, 1024, x, 1, P(full), y, y, y, ws, 1 << 40, None) == -6
