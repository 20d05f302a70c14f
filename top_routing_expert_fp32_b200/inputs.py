"""Seeded synthetic inputs for the MoE FFN forward layer.

This module only draws random tensors; it holds none of the layer's arithmetic. Both the
CUDA path and the CPU oracle consume the exact tensors it returns (the oracle gets host copies
of the same values), so the two sides never disagree about their inputs.

Recipe (every config; seed 0 unless a test says otherwise):

* every tensor has its own ``torch.Generator`` seeded with ``seed * 1000 + tensor_id``
  (X=1, W_r=2, W1=3, W2=4, W3=5, bias=6, logits=7, routing noise=8);
* values are drawn in fp32 with ``torch.randn``, scaled by the standard deviation, then
  cast to the config dtype (bf16 or fp32); W_r and the bias always stay fp32;
* X ~ N(0, 1); W_r, W1, W2 ~ N(0, 1/D); W3 ~ N(0, 1/F) (variance = 1/fan_in);
* optional per-expert router bias ~ N(0, router_bias_var) (variance).

The weight layout is the stacked one of the Grok-1 book (ch.5, sec 5.3.2): a leading
expert dimension, experts contiguous in order 0..E-1: W1 (activated branch), W2 (linear
branch) [E, D, F], W3 (down projection) [E, F, D].
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch

from .configs import DTYPE_BF16, DTYPE_F32, MoEConfig

TID_X, TID_WR, TID_W1, TID_W2, TID_W3, TID_BIAS, TID_LOGITS, TID_NOISE = 1, 2, 3, 4, 5, 6, 7, 8


def torch_dtype(code: int) -> torch.dtype:
    if code == DTYPE_BF16:
        return torch.bfloat16
    if code == DTYPE_F32:
        return torch.float32
    raise ValueError(f"unknown dtype code {code}")


def _gen(device: torch.device, seed: int, tid: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + tid)
    return g


def randn(shape, std: float, dtype: torch.dtype, device, seed: int, tid: int,
          chunks: int = 1) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and cast to ``dtype``. With ``chunks`` > 1 the leading
    dimension is drawn slice by slice (same generator, fixed order) to bound the fp32
    temporary; the result depends on ``chunks``, which every caller fixes per tensor."""
    device = torch.device(device)
    g = _gen(device, seed, tid)
    out = torch.empty(shape, dtype=dtype, device=device)
    if chunks <= 1:
        tmp = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        out.copy_(tmp.mul_(std))
        return out
    for i in range(shape[0]):
        tmp = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
        out[i].copy_(tmp.mul_(std))
    return out


@dataclass
class MoEInputs:
    X: torch.Tensor                 # [N, D] dtype
    W_r: torch.Tensor               # [D, E] fp32
    bias: Optional[torch.Tensor]    # [E] fp32 or None
    W1: torch.Tensor                # [E, D, F] dtype (activated branch)
    W2: torch.Tensor                # [E, D, F] dtype (linear branch)
    W3: torch.Tensor                # [E, F, D] dtype (down projection)


def make_inputs(cfg: MoEConfig, device="cpu", seed: Optional[int] = None,
                weights: bool = True) -> MoEInputs:
    """Draw the inputs of ``cfg`` on ``device``. Expert weights are drawn one expert at a
    time (``chunks`` = E). With ``weights=False`` W1..W3 are empty placeholders."""
    s = cfg.seed if seed is None else seed
    dt = torch_dtype(cfg.dtype)
    X = randn((cfg.N, cfg.D), 1.0, dt, device, s, TID_X)
    W_r = randn((cfg.D, cfg.E), 1.0 / math.sqrt(cfg.D), torch.float32, device, s, TID_WR)
    bias = None
    if cfg.router_bias_var > 0:
        bias = randn((cfg.E,), math.sqrt(cfg.router_bias_var), torch.float32, device, s,
                     TID_BIAS)
    if weights:
        W1 = randn((cfg.E, cfg.D, cfg.F), 1.0 / math.sqrt(cfg.D), dt, device, s, TID_W1,
                   chunks=cfg.E)
        W2 = randn((cfg.E, cfg.D, cfg.F), 1.0 / math.sqrt(cfg.D), dt, device, s, TID_W2,
                   chunks=cfg.E)
        W3 = randn((cfg.E, cfg.F, cfg.D), 1.0 / math.sqrt(cfg.F), dt, device, s, TID_W3,
                   chunks=cfg.E)
    else:
        W1 = W2 = W3 = torch.empty(0, dtype=dt, device=device)
    return MoEInputs(X, W_r, bias, W1, W2, W3)


@dataclass
class MoEWeights8:
    W1q: torch.Tensor   # [E, D, F] int8 (activated branch)
    S1: torch.Tensor    # [E, F] fp32, one scale per expert and output column
    W2q: torch.Tensor   # [E, D, F] int8 (linear branch)
    S2: torch.Tensor    # [E, F] fp32
    W3q: torch.Tensor   # [E, F, D] int8 (down projection)
    S3: torch.Tensor    # [E, D] fp32


def _quantize_columns(w: torch.Tensor):
    """Synthetic 8-bit weights: per output column, scale = max |w| / 127 and q = round(w /
    scale) in [-127, 127]. Input synthesis only (the layer itself only dequantizes)."""
    amax = w.abs().amax(dim=0)
    scale = torch.where(amax > 0, amax / 127.0, torch.ones_like(amax))
    q = torch.clamp(torch.round(w / scale), -127, 127).to(torch.int8)
    return q, scale.to(torch.float32)


def make_w8_weights(cfg: MoEConfig, device="cpu", seed: Optional[int] = None) -> MoEWeights8:
    """8-bit expert weights of the same N(0, 1/fan_in) draws as make_inputs (same generators
    and per-expert chunking), quantized per expert and output column."""
    s = cfg.seed if seed is None else seed
    device = torch.device(device)
    out = []
    for tid, (rows, cols, fan_in) in ((TID_W1, (cfg.D, cfg.F, cfg.D)), (TID_W2, (cfg.D, cfg.F, cfg.D)),
                                      (TID_W3, (cfg.F, cfg.D, cfg.F))):
        g = _gen(device, s, tid)
        q = torch.empty((cfg.E, rows, cols), dtype=torch.int8, device=device)
        sc = torch.empty((cfg.E, cols), dtype=torch.float32, device=device)
        for e in range(cfg.E):
            w = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
            q[e], sc[e] = _quantize_columns(w.mul_(1.0 / math.sqrt(fan_in)))
        out += [q, sc]
    return MoEWeights8(*out)


def make_noise(N: int, E: int, std: float, device="cpu", seed: int = 0) -> torch.Tensor:
    """The random draws of the training-time routing variants, N(0, std^2) fp32 [N, E]: the
    layer takes them as an input so that every consumer sees the same numbers."""
    return randn((N, E), std, torch.float32, device, seed, TID_NOISE)


def make_logits(N: int, E: int, device="cpu", seed: int = 0, std: float = 1.0) -> torch.Tensor:
    """Router logits drawn directly (fp32), for routing tests that start from logits."""
    return randn((N, E), std, torch.float32, device, seed, TID_LOGITS)
