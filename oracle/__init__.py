"""fp64 CPU oracle of the visual-token compression path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package. The product path never does.
"""
from . import ivc_oracle
from .ivc_oracle import *  # noqa: F401,F403


def to64(t):
    """A bf16/fp32 torch tensor (or list of them) widened to float64 numpy."""
    import numpy as np
    if isinstance(t, (list, tuple)):
        return [to64(v) for v in t]
    if isinstance(t, dict):
        return {k: to64(v) for k, v in t.items()}
    if hasattr(t, "detach"):
        import torch
        if t.dtype in (torch.int32, torch.int64, torch.uint8):
            return t.detach().cpu().numpy()
        return t.detach().cpu().to(torch.float64).numpy()
    return t
