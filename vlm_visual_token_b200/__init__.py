"""Python binding of libivc.so — InternVL visual-token compression on B200.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. PyTorch provides device memory and the current CUDA stream. The
functions keep the C names without the ``ivc_`` prefix:

    ps_project(x, scale, mlp, flags=0)           -> y [T*tokens, H] bf16
    vir_route(x, valid_len, image_offsets, r)    -> gate, mask, offsets
    route(gate, image_offsets)                   -> mask, offsets, total
    flash_compress(x, valid_len, image_offsets, mlp1, mlp2, r) -> dict

Importing this module fails loudly when the shared library is missing; there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import json
import os
from typing import Optional, Sequence

import torch

POOL_FOLDED, POOL_LITERAL = 0, 1

__all__ = ["Mlp", "Router", "POOL_FOLDED", "POOL_LITERAL", "ps_project", "vir_route", "route",
           "flash_compress", "assemble_sequence", "workspace_size",
           "device_status", "IvcError", "lib", "LIB_PATH", "PS_V1", "PS_QUARTER_TWICE",
           "OP_PS_HALF", "OP_PS_QUARTER", "OP_VIR_ROUTE", "OP_FLASH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libivc.so")

PS_V1 = 1
PS_QUARTER_TWICE = 2
OP_PS_HALF, OP_PS_QUARTER, OP_VIR_ROUTE, OP_FLASH = 1, 2, 3, 4

_vp = ctypes.c_void_p


class _CMlp(ctypes.Structure):
    _fields_ = [("n_linear", ctypes.c_int), ("dims", ctypes.c_int * 4),
                ("ln_gamma", _vp), ("ln_beta", _vp), ("W", _vp * 3), ("b", _vp * 3),
                ("fold_W0", _vp), ("fold_colsum", _vp), ("fold_bias", _vp)]


class _CRouter(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("heads", ctypes.c_int), ("gate_hidden", ctypes.c_int),
                ("query", _vp),
                ("Wq", _vp * 4), ("bq", _vp * 4), ("Wk", _vp * 4), ("bk", _vp * 4),
                ("Wv", _vp * 4), ("bv", _vp * 4), ("Wo", _vp * 4), ("bo", _vp * 4),
                ("gW1", _vp * 4), ("gb1", _vp * 4), ("gW2", _vp * 4), ("gb2", _vp * 4),
                ("gln_g", _vp * 4), ("gln_b", _vp * 4), ("gWout", _vp), ("gbout", _vp),
                ("rel_q", ctypes.c_double), ("abs_t", ctypes.c_double),
                ("quantile_scope", ctypes.c_int), ("pool_mode", ctypes.c_int),
                ("gate_residual", ctypes.c_int),
                ("fold_u1", _vp), ("fold_c1", _vp), ("fold_wqo", _vp * 3), ("fold_bqo", _vp * 3)]


class IvcError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {lib().ivc_strerror(code).decode()} ({code})")
        self.code = code


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libivc.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libivc.so not built at {LIB_PATH}; run "
                              "`python -m vlm_visual_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.ivc_strerror.restype = ctypes.c_char_p
        L.ivc_strerror.argtypes = [ctypes.c_int]
        L.ivc_version.restype = ctypes.c_int
        L.ivc_workspace_size.restype = ctypes.c_size_t
        L.ivc_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(_CMlp), ctypes.POINTER(_CMlp),
                                         ctypes.POINTER(_CRouter)]
        L.ivc_mlp_fold_size.restype = ctypes.c_size_t
        L.ivc_mlp_fold_size.argtypes = [ctypes.POINTER(_CMlp)]
        L.ivc_mlp_fold.restype = ctypes.c_int
        L.ivc_mlp_fold.argtypes = [ctypes.POINTER(_CMlp), _vp, ctypes.c_size_t, _vp]
        L.ivc_router_fold_size.restype = ctypes.c_size_t
        L.ivc_router_fold_size.argtypes = [ctypes.POINTER(_CRouter)]
        L.ivc_router_fold.restype = ctypes.c_int
        L.ivc_router_fold.argtypes = [ctypes.POINTER(_CRouter), _vp, ctypes.c_size_t, _vp]
        L.ivc_ps_project.restype = ctypes.c_int
        L.ivc_ps_project.argtypes = [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                     ctypes.POINTER(_CMlp), _vp, _vp, ctypes.c_size_t, _vp]
        L.ivc_vir_route.restype = ctypes.c_int
        L.ivc_vir_route.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int,
                                    ctypes.POINTER(_CRouter), _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                    _vp]
        L.ivc_route.restype = ctypes.c_int
        L.ivc_route.argtypes = [_vp, ctypes.c_int, _vp, ctypes.c_int, ctypes.c_double,
                                ctypes.c_double, ctypes.c_int, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                _vp]
        L.ivc_flash_compress.restype = ctypes.c_int
        L.ivc_flash_compress.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int,
                                         ctypes.POINTER(_CMlp), ctypes.POINTER(_CMlp),
                                         ctypes.POINTER(_CRouter), _vp, _vp, _vp, _vp, _vp, _vp,
                                         ctypes.c_size_t, _vp]
        L.ivc_flash_compress_routed.restype = ctypes.c_int
        L.ivc_flash_compress_routed.argtypes = L.ivc_flash_compress.argtypes
        L.ivc_assemble_workspace_size.restype = ctypes.c_size_t
        L.ivc_assemble_workspace_size.argtypes = [ctypes.c_int]
        L.ivc_assemble_sequence.restype = ctypes.c_int
        L.ivc_assemble_sequence.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int32,
                                            _vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp,
                                            ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                            ctypes.c_size_t, _vp]
        L.ivc_set_router_wait_limit.restype = ctypes.c_int
        L.ivc_set_router_wait_limit.argtypes = [ctypes.c_longlong]
        L.ivc_device_status.restype = ctypes.c_int
        L.ivc_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_int), _vp]
        L.ivc_trace_enable.restype = ctypes.c_int
        L.ivc_trace_enable.argtypes = [ctypes.c_int]
        L.ivc_trace_reset.restype = ctypes.c_int
        L.ivc_trace_reset.argtypes = []
        L.ivc_trace_report.restype = ctypes.c_int
        L.ivc_trace_report.argtypes = [ctypes.c_char_p, ctypes.c_size_t]
        _LIB = L
    return _LIB


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise IvcError(rc, what)


class Mlp:
    """Connector MLP weights on the device plus their C descriptor.

    params: {"dims": [...], "ln_g", "ln_b", "W": [...], "b": [...]} of bf16 tensors.
    """

    def __init__(self, params: dict, device="cuda"):
        def dev(t):
            return t.to(device=device, dtype=torch.bfloat16).contiguous()
        self.dims = list(params["dims"])
        self.ln_g = dev(params["ln_g"])
        self.ln_b = dev(params["ln_b"])
        self.W = [dev(w) for w in params["W"]]
        self.b = [dev(b) for b in params["b"]]
        self.folded = None
        c = _CMlp()
        c.n_linear = len(self.W)
        for i, d in enumerate(self.dims):
            c.dims[i] = d
        c.ln_gamma = self.ln_g.data_ptr()
        c.ln_beta = self.ln_b.data_ptr()
        for i in range(len(self.W)):
            c.W[i] = self.W[i].data_ptr()
            c.b[i] = self.b[i].data_ptr()
        self.c = c

    @property
    def out_dim(self) -> int:
        return self.dims[-1]

    def fold(self, stream=None) -> "Mlp":
        """Fold LayerNorm's gamma/beta into the first Linear once (ivc_mlp_fold)."""
        n = lib().ivc_mlp_fold_size(ctypes.byref(self.c))
        self.folded = torch.empty(n, dtype=torch.uint8, device=self.W[0].device)
        _check(lib().ivc_mlp_fold(ctypes.byref(self.c), _ptr(self.folded), n, _stream(stream)),
               "ivc_mlp_fold")
        return self


class Router:
    """ViR router weights (CrossAttentionPooling + Gating) and thresholds.

    With `fold` (the default) and folded pooling on a CUDA device, the weight
    folds of ivc_router_fold are formed once here."""

    def __init__(self, params: dict, rel_q: float = 0.1, abs_t: float = 0.5, scope: int = 0,
                 device="cuda", pool_mode: int = 0, gate_residual: int = 0, fold: bool = True):
        def dev(t):
            return t.to(device=device, dtype=torch.bfloat16).contiguous()
        self.t = {}
        c = _CRouter()
        c.D = int(params["D"])
        c.heads = int(params["heads"])
        c.gate_hidden = int(params["gW1"][0].shape[0])
        self.t["query"] = dev(params["query"])
        c.query = self.t["query"].data_ptr()
        for k in ("Wq", "bq", "Wk", "bk", "Wv", "bv", "Wo", "bo",
                  "gW1", "gb1", "gW2", "gb2", "gln_g", "gln_b"):
            self.t[k] = [dev(v) for v in params[k]]
            arr = getattr(c, k)
            for i, v in enumerate(self.t[k]):
                arr[i] = v.data_ptr()
        self.t["gWout"] = dev(params["gWout"])
        self.t["gbout"] = dev(params["gbout"])
        c.gWout = self.t["gWout"].data_ptr()
        c.gbout = self.t["gbout"].data_ptr()
        c.rel_q = float(rel_q)
        c.abs_t = float(abs_t)
        c.quantile_scope = int(scope)
        c.pool_mode = int(pool_mode)
        c.gate_residual = int(gate_residual)
        self.c = c
        self.folded = None
        if fold and c.pool_mode == 0 and torch.device(device).type == "cuda":
            self.fold()

    def fold(self, stream=None) -> "Router":
        """Form the weight folds once (ivc_router_fold)."""
        n = lib().ivc_router_fold_size(ctypes.byref(self.c))
        if n == 0:
            raise IvcError(-3, "ivc_router_fold_size")
        self.folded = torch.empty(n, dtype=torch.uint8, device=self.t["query"].device)
        _check(lib().ivc_router_fold(ctypes.byref(self.c), _ptr(self.folded), n, _stream(stream)),
               "ivc_router_fold")
        return self


def workspace_size(op: int, T: int, C: int, m: Optional[Mlp] = None, m2: Optional[Mlp] = None,
                   r: Optional[Router] = None) -> int:
    n = lib().ivc_workspace_size(op, T, C, ctypes.byref(m.c) if m else None,
                                 ctypes.byref(m2.c) if m2 else None,
                                 ctypes.byref(r.c) if r else None)
    if n == 0:
        raise IvcError(-2, "ivc_workspace_size")
    return n


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    # zeroed so that the status word in its header starts clear
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def ps_project(x: torch.Tensor, scale: float, mlp: Mlp, flags: int = 0,
               out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    T, G, G2, C = x.shape
    rows = T * (256 if scale == 0.5 else 64)
    if out is None:
        out = torch.empty(rows, mlp.out_dim, dtype=torch.bfloat16, device=x.device)
    op = OP_PS_HALF if scale == 0.5 else OP_PS_QUARTER
    need = workspace_size(op, T, C, mlp)
    if workspace is None:
        workspace = new_workspace(need, x.device)
    _check(lib().ivc_ps_project(_ptr(x), T, C, float(scale), int(flags), ctypes.byref(mlp.c),
                                _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "ivc_ps_project")
    return out


def vir_route(x: torch.Tensor, valid_len: Optional[torch.Tensor], image_offsets: torch.Tensor,
              r: Router, workspace: Optional[torch.Tensor] = None, stream=None):
    T, _, _, C = x.shape
    dev = x.device
    gate = torch.empty(T, 2, dtype=torch.float32, device=dev)
    mask = torch.empty(T, dtype=torch.uint8, device=dev)
    offsets = torch.empty(T + 1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_VIR_ROUTE, T, C, r=r), dev)
    I = int(image_offsets.numel()) - 1
    _check(lib().ivc_vir_route(_ptr(x), _ptr(valid_len), T, C, _ptr(image_offsets), I,
                               ctypes.byref(r.c), _ptr(gate), _ptr(mask), _ptr(offsets),
                               _ptr(workspace), workspace.numel(), _stream(stream)),
           "ivc_vir_route")
    return gate, mask, offsets


ROUTE_WORKSPACE_BYTES = 256


def route(gate: torch.Tensor, image_offsets: Optional[torch.Tensor], rel_q: float = 0.1,
          abs_t: float = 0.5, scope: int = 0, workspace: Optional[torch.Tensor] = None,
          stream=None):
    """ivc_route: the double threshold and row offsets for a given fp32 gate
    [T, 2]. Returns mask [T] uint8, offsets [T+1] int32, total [1] int32."""
    T = int(gate.shape[0])
    dev = gate.device
    mask = torch.empty(T, dtype=torch.uint8, device=dev)
    offsets = torch.empty(T + 1, dtype=torch.int32, device=dev)
    total = torch.empty(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(ROUTE_WORKSPACE_BYTES, dev)
    I = int(image_offsets.numel()) - 1 if image_offsets is not None else 0
    _check(lib().ivc_route(_ptr(gate), T, _ptr(image_offsets), I, float(rel_q), float(abs_t),
                           int(scope), _ptr(mask), _ptr(offsets), _ptr(total), _ptr(workspace),
                           workspace.numel(), _stream(stream)),
           "ivc_route")
    return mask, offsets, total


def flash_compress(x: torch.Tensor, valid_len: Optional[torch.Tensor], image_offsets: torch.Tensor,
                   mlp1: Mlp, mlp2: Mlp, r: Router, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, bufs: Optional[dict] = None,
                   stream=None, routed: bool = False) -> dict:
    """ivc_flash_compress (both paths for every tile, then compaction), or with
    routed=True ivc_flash_compress_routed (router first, each tile through its
    selected path only); same results."""
    T, _, _, C = x.shape
    dev = x.device
    H = mlp1.out_dim
    if bufs is None:
        bufs = {"gate": torch.empty(T, 2, dtype=torch.float32, device=dev),
                "mask": torch.empty(T, dtype=torch.uint8, device=dev),
                "offsets": torch.empty(T + 1, dtype=torch.int32, device=dev),
                "total": torch.empty(1, dtype=torch.int32, device=dev)}
    if out is None:
        out = torch.empty(max(T, 1) * 256, H, dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_FLASH, T, C, mlp1, mlp2, r), dev)
    I = int(image_offsets.numel()) - 1
    fn = lib().ivc_flash_compress_routed if routed else lib().ivc_flash_compress
    _check(fn(_ptr(x), _ptr(valid_len), T, C, _ptr(image_offsets), I,
              ctypes.byref(mlp1.c), ctypes.byref(mlp2.c), ctypes.byref(r.c),
              _ptr(out), _ptr(bufs["gate"]), _ptr(bufs["mask"]),
              _ptr(bufs["offsets"]), _ptr(bufs["total"]), _ptr(workspace),
              workspace.numel(), _stream(stream)),
           "ivc_flash_compress_routed" if routed else "ivc_flash_compress")
    res = dict(bufs)
    res["out"] = out
    return res


def assemble_sequence(input_ids: torch.Tensor, seq_offsets: torch.Tensor, img_context_id: int,
                      embed_table: torch.Tensor, visual: torch.Tensor, mask: torch.Tensor,
                      offsets: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                      out: Optional[dict] = None, stream=None) -> dict:
    """ivc_assemble_sequence: the visual rows spliced into the token sequences
    (compressed tiles keep 64 of their 256 placeholders). Returns device
    tensors at full capacity L; the kept length is seq_offsets[-1]."""
    L = int(input_ids.numel())
    B = int(seq_offsets.numel()) - 1
    V, H = embed_table.shape
    T = int(mask.numel())
    dev = input_ids.device
    if out is None:
        out = {"ids": torch.empty(max(L, 1), dtype=torch.int32, device=dev),
               "embeds": torch.empty(max(L, 1), H, dtype=torch.bfloat16, device=dev),
               "positions": torch.empty(max(L, 1), dtype=torch.int32, device=dev),
               "seq_offsets": torch.empty(B + 1, dtype=torch.int32, device=dev)}
    if workspace is None:
        workspace = new_workspace(lib().ivc_assemble_workspace_size(L), dev)
    _check(lib().ivc_assemble_sequence(_ptr(input_ids), _ptr(seq_offsets), B, L,
                                       int(img_context_id), _ptr(embed_table), V, H, _ptr(visual),
                                       _ptr(mask), _ptr(offsets), T, _ptr(out["ids"]),
                                       _ptr(out["embeds"]), _ptr(out["positions"]),
                                       _ptr(out["seq_offsets"]), _ptr(workspace),
                                       workspace.numel(), _stream(stream)),
           "ivc_assemble_sequence")
    res = dict(out)
    res["workspace"] = workspace
    return res


def device_status(workspace: torch.Tensor, stream=None) -> int:
    """Bits of the workspace's device status word (then cleared)."""
    bits = ctypes.c_int(0)
    rc = lib().ivc_device_status(_ptr(workspace), ctypes.byref(bits), _stream(stream))
    if rc not in (0, -5):
        raise IvcError(rc, "ivc_device_status")
    return bits.value


def trace_enable(on: bool = True) -> None:
    """Start (or stop) recording the device time of each of the library's launches."""
    _check(lib().ivc_trace_enable(1 if on else 0), "ivc_trace_enable")


def trace_reset() -> None:
    """Forget the recorded launches."""
    _check(lib().ivc_trace_reset(), "ivc_trace_reset")


def trace_report(max_bytes: int = 1 << 16) -> dict:
    """{role: {"launches": n, "ms": total device ms}} of the launches recorded
    since the last reset (waits for them to finish)."""
    buf = ctypes.create_string_buffer(max_bytes)
    _check(lib().ivc_trace_report(buf, len(buf)), "ivc_trace_report")
    return json.loads(buf.value.decode())
