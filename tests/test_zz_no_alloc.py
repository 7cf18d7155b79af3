"""ivc_ps_project_noalloc: the connector call for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Called through the C ABI and compared, on two calls in a row, with the
ordinary ivc_ps_project on the same inputs (the parity tolerance of the other
connector tests, and the kernels are the same, so the outputs also match
bit for bit). Kept in a file that pytest collects last."""
import ctypes

import pytest
import torch

import workloads as W
from tests._parity import assert_connector_close

pytestmark = pytest.mark.gpu


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import vlm_visual_token_b200 as ivc
    L = ivc.lib()
    f = L.ivc_ps_project_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                  ctypes.POINTER(ivc._CMlp), ctypes.c_void_p, ctypes.c_void_p]
    return ivc, f


def _noalloc(ivc, f, x, scale, m, flags=0):
    T = x.shape[0]
    rows = T * (256 if scale == 0.5 else 64)
    y = torch.full((rows, m.out_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    rc = f(ctypes.c_void_p(x.data_ptr()), T, x.shape[-1], ctypes.c_float(scale), flags,
           ctypes.byref(m.c), ctypes.c_void_p(y.data_ptr()),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, ivc.lib().ivc_strerror(rc)
    return y


@pytest.mark.parametrize("scale,key,name", [(0.5, "mlp1", "single_tile_2b"),
                                            (0.25, "mlp2", "flash_2b_13tiles")])
def test_noalloc_matches_workspace_call_twice(scale, key, name):
    ivc, f = _lib()
    inp = W.make(name, affine="random", n_images=1)
    x = inp["x"][:3].cuda().contiguous() if scale == 0.25 else inp["x"].cuda()
    m = ivc.Mlp(inp[key]).fold()
    ref = ivc.ps_project(x, scale, m)
    for _ in range(2):
        got = _noalloc(ivc, f, x, scale, m)
        torch.cuda.synchronize()
        assert_connector_close(got, ref.double().cpu().numpy(), "noalloc vs ps_project")
        assert torch.equal(got, ref)


def test_noalloc_rejects_what_does_not_fit_and_unfolded_weights():
    ivc, f = _lib()
    inp = W.make("single_tile_2b")
    m = ivc.Mlp(inp["mlp1"])
    x = inp["x"].cuda()
    y = torch.empty(256, 2048, dtype=torch.bfloat16, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # not folded
    assert f(ctypes.c_void_p(x.data_ptr()), 1, 1024, ctypes.c_float(0.5), 0, ctypes.byref(m.c),
             ctypes.c_void_p(y.data_ptr()), s) == -1
    m.fold()
    # 64 tiles of hidden activations need ~64 MiB of scratch: more than the array holds
    assert f(ctypes.c_void_p(x.data_ptr()), 64, 1024, ctypes.c_float(0.5), 0, ctypes.byref(m.c),
             ctypes.c_void_p(y.data_ptr()), s) == -3
