"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""
import numpy as np
import torch

# Tolerances of the connector outputs: relative Frobenius error 1e-2 and
# max-abs error 3e-2. The outputs are bf16; where |y| >= 4 one bf16 ulp is
# >= 2^-5, so rounding the exact result to bf16 alone can use up to half an
# ulp (1/64 on [4,8), 1/32 on [8,16)). For those elements the bound is
# 3e-2 plus half an ulp of the oracle value; below 4 it is 3e-2 flat.
REL_FRO = 1e-2
MAX_ABS = 3e-2
GATE_ABS = 1e-3


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 2.0 ** -126)
    e = np.floor(np.log2(a))
    return 0.5 * 2.0 ** (e - 7)


def connector_errors(got: torch.Tensor, ref: np.ndarray) -> dict:
    g = got.detach().float().cpu().double().numpy().reshape(ref.shape)
    err = g - ref
    fro = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    absmax = float(np.abs(err).max()) if err.size else 0.0
    allowed = MAX_ABS + np.where(np.abs(ref) >= 4.0, bf16_half_ulp(ref), 0.0)
    excess = float((np.abs(err) - allowed).max()) if err.size else -1.0
    return {"rel_fro": fro, "max_abs": absmax, "max_excess": excess, "n": int(err.size)}


def assert_connector_close(got, ref, what=""):
    e = connector_errors(got, ref)
    assert np.isfinite(e["rel_fro"]), (what, e)
    assert e["rel_fro"] <= REL_FRO, (what, e)
    assert e["max_excess"] <= 0.0, (what, e)
    return e


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16, torch.float32):
        return t.double().numpy()
    return t.numpy()
