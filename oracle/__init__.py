"""CPU oracle of the MoE FFN forward layer -- TEST INFRASTRUCTURE ONLY.

A ctypes wrapper around ``moe_oracle.c`` (plain fp64 loops written from the pages). Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import this
package; the product library never does, and shares no code with it.

Arrays are numpy; bf16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1
SILU, GELU_ERF, GELU_TANH = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP). Building the checker is not using it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=gnu11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.oracle_capacity.argtypes = [i64, i32, i32, f64]
        L.oracle_capacity.restype = i64
        L.oracle_capacity_min.argtypes = [i64, i32, i32, f64, i64]
        L.oracle_capacity_min.restype = i64
        L.oracle_dispatch_order.argtypes = [i64, i32, i32, i64, i32, P, P, P, P, P, P]
        L.oracle_dispatch_order.restype = None
        L.oracle_combine_policy.argtypes = [i64, i32, i64, P, P, i32, P, P]
        L.oracle_combine_policy.restype = None
        L.oracle_router_logits.argtypes = [i64, i64, i32, P, i32, P, P, P, P]
        L.oracle_router_logits.restype = None
        L.oracle_route.argtypes = [i64, i32, i32, i32, P, P, P, P, P]
        L.oracle_route.restype = ctypes.c_int
        L.oracle_route_ex.argtypes = [i64, i32, i32, i32, i32, P, P, P, P, P, P, P]
        L.oracle_route_ex.restype = ctypes.c_int
        L.oracle_topk_margin.argtypes = [i64, i32, i32, P, P]
        L.oracle_topk_margin.restype = None
        L.oracle_dispatch.argtypes = [i64, i32, i32, i64, P, P, P, P, P, P]
        L.oracle_dispatch.restype = None
        L.oracle_expert_ffn.argtypes = [i64, P, P, i64, i64, P, P, P, P, i32, i32, P]
        L.oracle_expert_ffn.restype = None
        L.oracle_combine.argtypes = [i64, i32, i64, P, P, P, P]
        L.oracle_combine.restype = None
        L.oracle_balance_loss.argtypes = [i64, i32, i32, P, P, i32]
        L.oracle_balance_loss.restype = f64
        L.oracle_drop_rate.argtypes = [i64, i32, P]
        L.oracle_drop_rate.restype = f64
        L.oracle_forward.argtypes = [i64, i64, i64, i32, i32, f64, i64, i32, i32, i32, i32,
                                     i32, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.oracle_forward.restype = ctypes.c_int
        L.oracle_forward_w8.argtypes = [i64, i64, i64, i32, i32, f64, i64, i32, i32, i32, i32,
                                        i32, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                        P]
        L.oracle_forward_w8.restype = ctypes.c_int
        L.oracle_expert_ffn_w8.argtypes = [i64, P, P, i64, i64, P, i32, P, P, P, P, P, P, i32, P]
        L.oracle_expert_ffn_w8.restype = None
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _elems(a, dtype: int):
    """X / W1..W3 arrays: fp32 values (dtype F32) or bf16 bit patterns as uint16 (BF16)."""
    if dtype == F32:
        return np.ascontiguousarray(a, dtype=np.float32)
    if dtype == BF16:
        if a.dtype != np.uint16:
            raise TypeError("bf16 arrays must be passed as uint16 bit patterns")
        return np.ascontiguousarray(a)
    raise ValueError(f"unknown dtype {dtype}")


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# Capacity policies: slot order of the position assignment, and what a token's kept slots
# weigh when another of its slots was dropped.
SLOT_MAJOR, TOKEN_MAJOR = 0, 1
DROP_ZERO, DROP_RENORM_KEPT = 0, 1


def capacity(N: int, k: int, E: int, cf: float, min_capacity: int = 0) -> int:
    return int(lib().oracle_capacity_min(N, k, E, float(cf), int(min_capacity)))


def router_logits(X: np.ndarray, x_dtype: int, W_r: np.ndarray, bias=None):
    """Returns (logits fp64 [N,E], logits fp32 [N,E])."""
    N, D = X.shape
    E = W_r.shape[1]
    X = _elems(X, x_dtype)
    W_r = _c(W_r, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    l64 = np.empty((N, E), np.float64)
    l32 = np.empty((N, E), np.float32)
    lib().oracle_router_logits(N, D, E, _p(X), x_dtype, _p(W_r), _p(b), _p(l64), _p(l32))
    return l64, l32


def route(logits32: np.ndarray, k: int, renorm: int, want_probs: bool = False):
    """Returns dict(idx [N,k] int32, gate [N,k] f64, colsum [E] f64, probs [N,E] or None)."""
    logits32 = _c(logits32, np.float32)
    N, E = logits32.shape
    idx = np.empty((N, k), np.int32)
    gate = np.empty((N, k), np.float64)
    colsum = np.empty((E,), np.float64)
    probs = np.empty((N, E), np.float64) if want_probs else None
    rc = lib().oracle_route(N, E, k, renorm, _p(logits32), _p(idx), _p(gate), _p(probs),
                            _p(colsum))
    if rc != 0:
        raise ValueError("oracle_route: non-finite logits")
    return dict(idx=idx, gate=gate, colsum=colsum, probs=probs)


# Routing modes (training-time variants of the selection).
ROUTE_TOPK, ROUTE_NOISY_TOPK, ROUTE_GSHARD_RANDOM = 0, 1, 2


def route_ex(logits32: np.ndarray, k: int, renorm: int, mode: int = ROUTE_TOPK, noise=None,
             want_probs: bool = False):
    """route() with the training-time variants and the z-loss. Returns dict(idx, gate, colsum,
    probs, zloss) where zloss = mean over tokens of (log sum exp logits)^2."""
    logits32 = _c(logits32, np.float32)
    N, E = logits32.shape
    nz = None if noise is None else _c(noise, np.float32)
    idx = np.empty((N, k), np.int32)
    gate = np.empty((N, k), np.float64)
    colsum = np.empty((E,), np.float64)
    probs = np.empty((N, E), np.float64) if want_probs else None
    z = np.zeros((1,), np.float64)
    rc = lib().oracle_route_ex(N, E, k, renorm, mode, _p(logits32), _p(nz), _p(idx), _p(gate),
                               _p(probs), _p(colsum), _p(z))
    if rc != 0:
        raise ValueError("oracle_route_ex: non-finite logits or noise, or missing noise")
    return dict(idx=idx, gate=gate, colsum=colsum, probs=probs, zloss=float(z[0]))


def topk_margin(logits64: np.ndarray, k: int) -> np.ndarray:
    logits64 = _c(logits64, np.float64)
    N, E = logits64.shape
    m = np.empty((N,), np.float64)
    lib().oracle_topk_margin(N, E, k, _p(logits64), _p(m))
    return m


def dispatch(idx: np.ndarray, E: int, C: int, order: int = SLOT_MAJOR):
    """Capacity dispatch (slot-major or token-major). Returns dict(load, offsets, pos, dropped,
    row_token)."""
    idx = _c(idx, np.int32)
    N, k = idx.shape
    load = np.empty((E,), np.int32)
    offsets = np.empty((E + 1,), np.int32)
    pos = np.empty((N, k), np.int32)
    dropped = np.empty((N, k), np.uint8)
    row_token = np.full((N * k,), -1, np.int32)
    lib().oracle_dispatch_order(N, k, E, C, order, _p(idx), _p(load), _p(offsets), _p(pos),
                                _p(dropped), _p(row_token))
    return dict(load=load, offsets=offsets, pos=pos, dropped=dropped,
                row_token=row_token[: int(offsets[E])].copy())


def expert_ffn(rec_token, rec_expert, X, W1, W2, W3, dtype: int, act: int) -> np.ndarray:
    """fp64 gated expert output of each record. X [N,D]; W1,W2 [E,D,F]; W3 [E,F,D]."""
    rec_token = _c(rec_token, np.int32)
    rec_expert = _c(rec_expert, np.int32)
    X, W1, W2, W3 = (_elems(a, dtype) for a in (X, W1, W2, W3))
    n = rec_token.shape[0]
    D = X.shape[1]
    F = W1.shape[2]
    Y = np.empty((n, D), np.float64)
    lib().oracle_expert_ffn(n, _p(rec_token), _p(rec_expert), D, F, _p(X), _p(W1), _p(W2),
                            _p(W3), dtype, act, _p(Y))
    return Y


def expert_ffn_w8(rec_token, rec_expert, X, x_dtype: int, W1q, S1, W2q, S2, W3q, S3,
                  act: int) -> np.ndarray:
    """fp64 gated expert output with 8-bit weights: W = q * s, s per expert and output column.
    W1q, W2q [E,D,F] int8, W3q [E,F,D] int8; S1, S2 [E,F], S3 [E,D] fp32."""
    rec_token = _c(rec_token, np.int32)
    rec_expert = _c(rec_expert, np.int32)
    X = _elems(X, x_dtype)
    W1q, W2q, W3q = (_c(w, np.int8) for w in (W1q, W2q, W3q))
    S1, S2, S3 = (_c(s, np.float32) for s in (S1, S2, S3))
    n = rec_token.shape[0]
    D = X.shape[1]
    F = W1q.shape[2]
    Y = np.empty((n, D), np.float64)
    lib().oracle_expert_ffn_w8(n, _p(rec_token), _p(rec_expert), D, F, _p(X), x_dtype, _p(W1q),
                               _p(S1), _p(W2q), _p(S2), _p(W3q), _p(S3), act, _p(Y))
    return Y


def combine(gate, dropped, Yrec, policy: int = DROP_ZERO) -> np.ndarray:
    gate = _c(gate, np.float64)
    N, k = gate.shape
    Yrec = _c(Yrec, np.float64)
    D = Yrec.shape[-1]
    dr = None if dropped is None else _c(dropped, np.uint8)
    out = np.empty((N, D), np.float64)
    lib().oracle_combine_policy(N, k, D, _p(gate), _p(dr), policy, _p(Yrec.reshape(N * k, D)),
                                _p(out))
    return out


def balance_loss(N: int, k: int, load, colsum, nk_denominator: bool = True) -> float:
    load = _c(load, np.int32)
    colsum = _c(colsum, np.float64)
    return float(lib().oracle_balance_loss(N, k, load.shape[0], _p(load), _p(colsum),
                                           1 if nk_denominator else 0))


def drop_rate(dropped) -> float:
    dropped = _c(dropped, np.uint8)
    N, k = dropped.shape
    return float(lib().oracle_drop_rate(N, k, _p(dropped)))


def forward(X, W_r, bias, W1, W2, W3, *, k: int, cf: float, renorm: int, act: int,
            dtype: int, min_capacity: int = 0, order: int = SLOT_MAJOR,
            drop_policy: int = DROP_ZERO):
    """Whole layer in fp64. Returns dict(out [N,D] f64, logits32, idx, gate, load, offsets,
    pos, dropped, colsum)."""
    X, W1, W2, W3 = (_elems(a, dtype) for a in (X, W1, W2, W3))
    N, D = X.shape
    E = W_r.shape[1]
    F = W1.shape[2]
    W_r = _c(W_r, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((N, D), np.float64)
    l32 = np.empty((N, E), np.float32)
    idx = np.empty((N, k), np.int32)
    gate = np.empty((N, k), np.float64)
    load = np.empty((E,), np.int32)
    offsets = np.empty((E + 1,), np.int32)
    pos = np.empty((N, k), np.int32)
    dropped = np.empty((N, k), np.uint8)
    colsum = np.empty((E,), np.float64)
    rc = lib().oracle_forward(N, D, F, E, k, float(cf), int(min_capacity), order, drop_policy,
                              renorm, act, dtype, _p(X), _p(W_r),
                              _p(b), _p(W1), _p(W2), _p(W3), _p(out), _p(l32), _p(idx),
                              _p(gate), _p(load), _p(offsets), _p(pos), _p(dropped),
                              _p(colsum))
    if rc != 0:
        raise ValueError("oracle_forward: non-finite logits")
    return dict(out=out, logits32=l32, idx=idx, gate=gate, load=load, offsets=offsets,
                pos=pos, dropped=dropped, colsum=colsum)


def forward_w8(X, W_r, bias, W1q, S1, W2q, S2, W3q, S3, *, k: int, cf: float, renorm: int,
               act: int, dtype: int, min_capacity: int = 0, order: int = SLOT_MAJOR,
               drop_policy: int = DROP_ZERO):
    """Whole layer in fp64 with 8-bit expert weights (W = q * s per expert and output column).
    Returns the same dict as forward()."""
    X = _elems(X, dtype)
    W1q, W2q, W3q = (_c(w, np.int8) for w in (W1q, W2q, W3q))
    S1, S2, S3 = (_c(s, np.float32) for s in (S1, S2, S3))
    N, D = X.shape
    E = W_r.shape[1]
    F = W1q.shape[2]
    W_r = _c(W_r, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((N, D), np.float64)
    l32 = np.empty((N, E), np.float32)
    idx = np.empty((N, k), np.int32)
    gate = np.empty((N, k), np.float64)
    load = np.empty((E,), np.int32)
    offsets = np.empty((E + 1,), np.int32)
    pos = np.empty((N, k), np.int32)
    dropped = np.empty((N, k), np.uint8)
    colsum = np.empty((E,), np.float64)
    rc = lib().oracle_forward_w8(N, D, F, E, k, float(cf), int(min_capacity), order, drop_policy,
                                 renorm, act, dtype, _p(X), _p(W_r), _p(b), _p(W1q), _p(S1),
                                 _p(W2q), _p(S2), _p(W3q), _p(S3), _p(out), _p(l32), _p(idx),
                                 _p(gate), _p(load), _p(offsets), _p(pos), _p(dropped),
                                 _p(colsum))
    if rc != 0:
        raise ValueError("oracle_forward_w8: non-finite logits")
    return dict(out=out, logits32=l32, idx=idx, gate=gate, load=load, offsets=offsets,
                pos=pos, dropped=dropped, colsum=colsum)


def torch_to_numpy(t):
    """Host numpy view of a torch tensor for the oracle: bf16 -> uint16 bit patterns."""
    import torch
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
