"""Helpers shared by the GPU parity tests: tolerance metrics and oracle plumbing."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from top_routing_expert_fp32_b200 import configs

# Tolerances (the spec parity bar): row-normwise max relative error of the layer output
# vs the oracle's fp64 value before rounding.
TOL_BF16 = 2e-2
TOL_F32 = 1e-5
NEAR_TIE = 1e-4


def tol(cfg) -> float:
    return TOL_BF16 if cfg.dtype == configs.DTYPE_BF16 else TOL_F32


def normwise_rel_err(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per row: max_d |got - ref| / max_d |ref| (rows with ref == 0 use the absolute error)."""
    got = got.astype(np.float64)
    num = np.abs(got - ref).max(axis=1)
    den = np.abs(ref).max(axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def np_host(t: torch.Tensor) -> np.ndarray:
    return oracle.torch_to_numpy(t)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def oracle_dtype(cfg) -> int:
    return oracle.BF16 if cfg.dtype == configs.DTYPE_BF16 else oracle.F32


def alloc_route_out(N, E, k, device="cuda"):
    return dict(logits=torch.empty((N, E), dtype=torch.float32, device=device),
                idx=torch.empty((N, k), dtype=torch.int32, device=device),
                gate=torch.empty((N, k), dtype=torch.float32, device=device),
                colsum=torch.empty((E,), dtype=torch.float32, device=device))


def alloc_dispatch_out(N, E, k, device="cuda"):
    return dict(load=torch.empty((E,), dtype=torch.int32, device=device),
                offsets=torch.empty((E + 1,), dtype=torch.int32, device=device),
                pos=torch.empty((N, k), dtype=torch.int32, device=device),
                dropped=torch.empty((N, k), dtype=torch.uint8, device=device),
                row_token=torch.full((max(N * k, 1),), -7, dtype=torch.int32, device=device))
