"""Python binding of the C ABI in ``include/moe.h`` (ctypes; argument marshalling only).

Every function here forwards to the CUDA library ``libmoe_b200.so``: the work of each step
runs in its kernels. Tensors are torch CUDA tensors (device memory and streams come from
PyTorch); the binding passes their data pointers and the current CUDA stream. There is no
fallback: if the library is missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

from .configs import MoEConfig

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(5)
DEVERR_NONE, DEVERR_WAIT_TIMEOUT, DEVERR_BAD_INDEX = range(3)

# Every symbol include/moe.h declares.
EXPORTS = ("moe_capacity", "moe_workspace_size", "moe_workspace_size_host", "moe_route",
           "moe_route_ex", "moe_dispatch", "moe_dispatch_noalloc", "moe_expert_ffn",
           "moe_expert_up", "moe_expert_down", "moe_combine", "moe_forward", "moe_forward_ex",
           "moe_forward_host", "moe_expert_up_w8", "moe_expert_down_w8", "moe_forward_w8",
           "moe_pack_w8", "moe_expert_up_w8p", "moe_expert_down_w8p", "moe_forward_w8p",
           "moe_gather_rows", "moe_forward_host_many", "moe_selftest_wait_timeout",
           "moe_balance_loss", "moe_drop_rate",
           "moe_workspace_init", "moe_get_device_error", "moe_status_string", "moe_last_error",
           "moe_version")


class moe_problem(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("D", ctypes.c_int64), ("F", ctypes.c_int64),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("capacity_factor", ctypes.c_double), ("renormalize", ctypes.c_int32),
                ("activation", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("capacity_order", ctypes.c_int32), ("drop_policy", ctypes.c_int32),
                ("routing_mode", ctypes.c_int32), ("min_capacity", ctypes.c_int64),
                ("reserved", ctypes.c_int32)]


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"moe status {status}: {msg}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m top_routing_expert_fp32_b200.build`"
                          " (or __graft_entry__.build()) first")
    L = ctypes.CDLL(LIB_PATH)
    P, S, I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
    PP = ctypes.POINTER(moe_problem)
    sig = {
        "moe_capacity": [PP, ctypes.POINTER(ctypes.c_int64)],
        "moe_workspace_size": [PP, ctypes.POINTER(S)],
        "moe_workspace_size_host": [PP, ctypes.POINTER(S)],
        "moe_route": [PP, P, P, P, P, P, P, P, P, S, P],
        "moe_dispatch": [PP, P, P, P, P, P, P, P, P, P, S, P],
        "moe_dispatch_noalloc": [PP, P, P, P, P, P, P, P, P, P],
        "moe_expert_ffn": [PP, P, P, P, P, P, P, P, P, S, P],
        "moe_expert_up": [PP, P, P, P, P, P, P, S, P],
        "moe_expert_down": [PP, P, P, P, P, P, S, P],
        "moe_combine": [PP, P, P, P, P, P, P, P, P],
        "moe_forward": [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "moe_forward_host": [PP, P, P, P, P, P, P, P, P, S, P],
        "moe_route_ex": [PP, P, P, P, P, P, P, P, P, P, P, S, P],
        "moe_forward_ex": [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "moe_expert_up_w8": [PP, P, P, P, P, P, P, P, P, S, P],
        "moe_expert_down_w8": [PP, P, P, P, P, P, P, S, P],
        "moe_forward_w8": [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "moe_pack_w8": [PP, P, P, P, P, P, P, P],
        "moe_gather_rows": [P, I64, P, I64, I64, P, P, S, P],
        "moe_forward_host_many": [PP, I64, P, P, P, P, P, P, P, P, S, P],
        "moe_selftest_wait_timeout": [P, S, I64, P],
        "moe_balance_loss": [PP, P, P, ctypes.POINTER(ctypes.c_double)],
        "moe_drop_rate": [PP, P, ctypes.POINTER(ctypes.c_double)],
        "moe_expert_up_w8p": [PP, P, P, P, P, P, P, P, P, S, P],
        "moe_expert_down_w8p": [PP, P, P, P, P, P, P, S, P],
        "moe_forward_w8p": [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "moe_workspace_init": [P, S, P],
        "moe_get_device_error": [P, P, ctypes.POINTER(ctypes.c_int32)],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_last_error.argtypes = []
    L.moe_last_error.restype = ctypes.c_char_p
    L.moe_version.argtypes = []
    L.moe_version.restype = ctypes.c_int32
    return L


lib = _load()


def _check(status: int):
    if status != MOE_OK:
        raise MoEError(status, lib.moe_last_error().decode(errors="replace"))


def problem(cfg: MoEConfig, N: Optional[int] = None) -> moe_problem:
    return moe_problem(N=cfg.N if N is None else N, D=cfg.D, F=cfg.F, E=cfg.E, k=cfg.k,
                       capacity_factor=float(cfg.capacity_factor), renormalize=cfg.renormalize,
                       activation=cfg.activation, dtype=cfg.dtype,
                       capacity_order=cfg.capacity_order, drop_policy=cfg.drop_policy,
                       routing_mode=cfg.routing_mode, min_capacity=cfg.min_capacity, reserved=0)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def capacity(p: moe_problem) -> int:
    c = ctypes.c_int64()
    _check(lib.moe_capacity(ctypes.byref(p), ctypes.byref(c)))
    return c.value


def workspace_size(p: moe_problem, host: bool = False) -> int:
    b = ctypes.c_size_t()
    fn = lib.moe_workspace_size_host if host else lib.moe_workspace_size
    _check(fn(ctypes.byref(p), ctypes.byref(b)))
    return b.value


def workspace(p: moe_problem, device="cuda", host: bool = False) -> torch.Tensor:
    """A device workspace of the required size with its error word zeroed."""
    n = workspace_size(p, host)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    _check(lib.moe_workspace_init(ws.data_ptr(), ws.numel(), _stream(None)))
    return ws


def route(p, X, W_r, bias, logits, topk_idx, topk_gate, prob_colsum, ws, stream=None):
    _check(lib.moe_route(ctypes.byref(p), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(logits),
                         _ptr(topk_idx), _ptr(topk_gate), _ptr(prob_colsum), _ptr(ws),
                         ws.numel(), _stream(stream)))


def route_ex(p, X, W_r, bias, noise, logits, topk_idx, topk_gate, prob_colsum, z_loss, ws,
             stream=None):
    _check(lib.moe_route_ex(ctypes.byref(p), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(noise),
                            _ptr(logits), _ptr(topk_idx), _ptr(topk_gate), _ptr(prob_colsum),
                            _ptr(z_loss), _ptr(ws), ws.numel(), _stream(stream)))


def dispatch(p, X, topk_idx, load, offsets, pos, dropped, row_token, X_perm, ws, stream=None):
    _check(lib.moe_dispatch(ctypes.byref(p), _ptr(X), _ptr(topk_idx), _ptr(load), _ptr(offsets),
                            _ptr(pos), _ptr(dropped), _ptr(row_token), _ptr(X_perm), _ptr(ws),
                            ws.numel(), _stream(stream)))


def dispatch_noalloc(p, X, topk_idx, load, offsets, pos, dropped, row_token, X_perm,
                     stream=None):
    """moe_dispatch without a workspace (counters in a fixed array inside the library)."""
    _check(lib.moe_dispatch_noalloc(ctypes.byref(p), _ptr(X), _ptr(topk_idx), _ptr(load),
                                    _ptr(offsets), _ptr(pos), _ptr(dropped), _ptr(row_token),
                                    _ptr(X_perm), _stream(stream)))


def expert_ffn(p, X_perm, offsets, W1, W2, W3, H, Y, ws, stream=None):
    _check(lib.moe_expert_ffn(ctypes.byref(p), _ptr(X_perm), _ptr(offsets), _ptr(W1), _ptr(W2),
                              _ptr(W3), _ptr(H), _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))


def expert_up(p, X_perm, offsets, W1, W2, H, ws, stream=None):
    _check(lib.moe_expert_up(ctypes.byref(p), _ptr(X_perm), _ptr(offsets), _ptr(W1), _ptr(W2),
                             _ptr(H), _ptr(ws), ws.numel(), _stream(stream)))


def expert_down(p, H, offsets, W3, Y, ws, stream=None):
    _check(lib.moe_expert_down(ctypes.byref(p), _ptr(H), _ptr(offsets), _ptr(W3), _ptr(Y),
                               _ptr(ws), ws.numel(), _stream(stream)))


def combine(p, Y, topk_idx, topk_gate, offsets, pos, dropped, out, stream=None):
    _check(lib.moe_combine(ctypes.byref(p), _ptr(Y), _ptr(topk_idx), _ptr(topk_gate),
                           _ptr(offsets), _ptr(pos), _ptr(dropped), _ptr(out), _stream(stream)))


def forward(p, X, W_r, bias, W1, W2, W3, out, ws, *, logits=None, topk_idx=None, topk_gate=None,
            load=None, offsets=None, pos=None, dropped=None, prob_colsum=None, stream=None):
    _check(lib.moe_forward(ctypes.byref(p), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(W1), _ptr(W2),
                           _ptr(W3), _ptr(out), _ptr(logits), _ptr(topk_idx), _ptr(topk_gate),
                           _ptr(load), _ptr(offsets), _ptr(pos), _ptr(dropped),
                           _ptr(prob_colsum), _ptr(ws), ws.numel(), _stream(stream)))


def forward_ex(p, X, W_r, bias, noise, W1, W2, W3, out, ws, *, logits=None, topk_idx=None,
               topk_gate=None, load=None, offsets=None, pos=None, dropped=None, prob_colsum=None,
               z_loss=None, stream=None):
    _check(lib.moe_forward_ex(ctypes.byref(p), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(noise),
                              _ptr(W1), _ptr(W2), _ptr(W3), _ptr(out), _ptr(logits),
                              _ptr(topk_idx), _ptr(topk_gate), _ptr(load), _ptr(offsets),
                              _ptr(pos), _ptr(dropped), _ptr(prob_colsum), _ptr(z_loss),
                              _ptr(ws), ws.numel(), _stream(stream)))


def expert_up_w8(p, X_perm, offsets, W1q, S1, W2q, S2, H, ws, stream=None):
    _check(lib.moe_expert_up_w8(ctypes.byref(p), _ptr(X_perm), _ptr(offsets), _ptr(W1q), _ptr(S1),
                                _ptr(W2q), _ptr(S2), _ptr(H), _ptr(ws), ws.numel(),
                                _stream(stream)))


def expert_down_w8(p, H, offsets, W3q, S3, Y, ws, stream=None):
    _check(lib.moe_expert_down_w8(ctypes.byref(p), _ptr(H), _ptr(offsets), _ptr(W3q), _ptr(S3),
                                  _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))


def gather_rows(src, index, dst, ws, stream=None):
    """dst[i] = src[index[i]] (row-wise); src / dst: 2-D device tensors of equal row size."""
    rb = math.prod(dst.shape[1:]) * dst.element_size()
    _check(lib.moe_gather_rows(_ptr(src), src.shape[0], _ptr(index), index.numel(), rb, _ptr(dst),
                               _ptr(ws), ws.numel(), _stream(stream)))


def pack_w8(p, W1q, W2q, W3q, W1p, W2p, W3p, stream=None):
    _check(lib.moe_pack_w8(ctypes.byref(p), _ptr(W1q), _ptr(W2q), _ptr(W3q), _ptr(W1p),
                           _ptr(W2p), _ptr(W3p), _stream(stream)))


def expert_up_w8p(p, X_perm, offsets, W1p, S1, W2p, S2, H, ws, stream=None):
    _check(lib.moe_expert_up_w8p(ctypes.byref(p), _ptr(X_perm), _ptr(offsets), _ptr(W1p),
                                 _ptr(S1), _ptr(W2p), _ptr(S2), _ptr(H), _ptr(ws), ws.numel(),
                                 _stream(stream)))


def expert_down_w8p(p, H, offsets, W3p, S3, Y, ws, stream=None):
    _check(lib.moe_expert_down_w8p(ctypes.byref(p), _ptr(H), _ptr(offsets), _ptr(W3p), _ptr(S3),
                                   _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)))


def forward_w8(p, X, W_r, bias, w8, out, ws, *, logits=None, topk_idx=None, topk_gate=None,
               load=None, offsets=None, pos=None, dropped=None, prob_colsum=None, packed=False,
               stream=None):
    """w8: an object with W1q, S1, W2q, S2, W3q, S3 (e.g. inputs.MoEWeights8); packed=True:
    its W1q, W2q, W3q are the K-contiguous copies written by pack_w8 (moe_forward_w8p)."""
    fn = lib.moe_forward_w8p if packed else lib.moe_forward_w8
    _check(fn(ctypes.byref(p), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(w8.W1q),
                              _ptr(w8.S1), _ptr(w8.W2q), _ptr(w8.S2), _ptr(w8.W3q), _ptr(w8.S3),
                              _ptr(out), _ptr(logits), _ptr(topk_idx), _ptr(topk_gate),
                              _ptr(load), _ptr(offsets), _ptr(pos), _ptr(dropped),
                              _ptr(prob_colsum), _ptr(ws), ws.numel(), _stream(stream)))


def forward_host(p, X_host: torch.Tensor, W_r, bias, W1, W2, W3, out_host: torch.Tensor, ws,
                 stream=None):
    """X_host / out_host are CPU tensors (pinned for asynchronous copies)."""
    _check(lib.moe_forward_host(ctypes.byref(p), _ptr(X_host), _ptr(W_r), _ptr(bias), _ptr(W1),
                                _ptr(W2), _ptr(W3), _ptr(out_host), _ptr(ws), ws.numel(),
                                _stream(stream)))


def forward_host_many(p, X_host: torch.Tensor, W_r, bias, W1, W2, W3, out_host: torch.Tensor, ws,
                      stream=None):
    """X_host / out_host: CPU tensors [n_batches, N, D] (pinned for asynchronous copies)."""
    nb = X_host.shape[0] if X_host.dim() == 3 else 1
    _check(lib.moe_forward_host_many(ctypes.byref(p), nb, _ptr(X_host), _ptr(W_r), _ptr(bias),
                                     _ptr(W1), _ptr(W2), _ptr(W3), _ptr(out_host), _ptr(ws),
                                     ws.numel(), _stream(stream)))


def balance_loss(p, load, prob_colsum) -> float:
    """load [E] int32, prob_colsum [E] fp32: host tensors (device tensors are copied)."""
    ld = load.detach().to("cpu", torch.int32).contiguous()
    cs = prob_colsum.detach().to("cpu", torch.float32).contiguous()
    out = ctypes.c_double()
    _check(lib.moe_balance_loss(ctypes.byref(p), _ptr(ld), _ptr(cs), ctypes.byref(out)))
    return out.value


def drop_rate(p, dropped) -> float:
    """dropped [N,k] uint8: a host tensor (a device tensor is copied)."""
    d = dropped.detach().to("cpu", torch.uint8).contiguous()
    out = ctypes.c_double()
    _check(lib.moe_drop_rate(ctypes.byref(p), _ptr(d), ctypes.byref(out)))
    return out.value


def selftest_wait_timeout(ws, timeout_us: int, stream=None):
    _check(lib.moe_selftest_wait_timeout(_ptr(ws), ws.numel(), int(timeout_us), _stream(stream)))


def device_error(ws, stream=None) -> int:
    code = ctypes.c_int32()
    st = lib.moe_get_device_error(_ptr(ws), _stream(stream), ctypes.byref(code))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        _check(st)
    return code.value


class Layer:
    """Convenience holder: a problem, its workspace and the forward call."""

    def __init__(self, cfg: MoEConfig, device="cuda"):
        self.cfg = cfg
        self.p = problem(cfg)
        self.ws = workspace(self.p, device)

    def forward(self, X, W_r, bias, W1, W2, W3, out=None, **exports):
        if out is None:
            out = torch.empty_like(X)
        forward(self.p, X, W_r, bias, W1, W2, W3, out, self.ws, **exports)
        return out
