"""Failure detection on the GPU without a fault: the persistent router's
grid barriers after the gating are given a limit of a few clock cycles, so
their waits run out (the other blocks have not arrived yet). The call must
return, set IVC_DEV_WAIT_TIMEOUT in the workspace status word, and leave the
context usable: the next call with the default limit matches the oracle.
No bulk copy is in flight at those barriers; every other wait keeps its
normal bound. The persistent router is selected with IVC_ROUTER_FUSED=1,
read once per process, so the check runs in a fresh one."""
import os
import subprocess
import sys

import pytest
import torch

from tests._parity import GATE_ABS

pytestmark = pytest.mark.gpu

_SNIPPET = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
import oracle as O, workloads as W, vlm_visual_token_b200 as ivc
L = ivc.lib()
w = W.Workload("fail", "flash", C=256, H=128, tiles_per_image=(3, 2), n_images=2,
               mlp2_mid=256, D=256, gate_hidden=256, seed_base=97)
inp = W.make(w, affine="random")
r = ivc.Router(inp["router"])
ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_VIR_ROUTE, inp["T"], 256, r=r))
x, offs = inp["x"].cuda(), inp["image_offsets"].cuda()
assert L.ivc_set_router_wait_limit(-1) == -1
assert L.ivc_set_router_wait_limit(4) == 0
try:
    ivc.vir_route(x, None, offs, r, workspace=ws)
    torch.cuda.synchronize()
    assert ivc.device_status(ws) & 4          # IVC_DEV_WAIT_TIMEOUT
finally:
    assert L.ivc_set_router_wait_limit(0) == 0
assert ivc.device_status(ws) == 0             # cleared by the read
gate, mask, offsets = ivc.vir_route(x, None, offs, r, workspace=ws)
torch.cuda.synchronize()
assert ivc.device_status(ws) == 0
ref_gate = O.vir_gate(O.to64(inp["x"]), inp["valid_len"].numpy(), O.to64(inp["router"]))
g = gate.cpu().double().numpy()
assert np.abs(g - ref_gate).max() <= {gate_abs!r}
ref_mask = O.route(g[:, 0], inp["image_offsets"].numpy())
np.testing.assert_array_equal(mask.cpu().numpy(), ref_mask)
np.testing.assert_array_equal(offsets.cpu().numpy(), O.compaction_offsets(ref_mask))
print("failure path ok")
"""


def test_router_barrier_timeout_sets_status_and_recovers():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _SNIPPET.format(root=root, gate_abs=GATE_ABS)],
                         env={**os.environ, "IVC_ROUTER_FUSED": "1"}, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "failure path ok" in out.stdout
