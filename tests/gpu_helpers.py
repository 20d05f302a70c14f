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


def check_routing(cfg, inp, ex):
    """Routing parity of a layer run. Returns (the oracle's dispatch of the GPU routing, the
    GPU routing's fp64 gates, the near-tie flip count against the fp64 logits).

    1. The GPU's exported fp32 logits lie within the fp32 accumulation bound of the oracle's
       fp64 logits (the router's arithmetic).
    2. Selection, order and gates taken by the oracle on those same fp32 logits equal the
       GPU's: indices bit-exact (descending, lower expert index on ties), gates to fp32
       rounding.
    3. Load, offsets, positions and drop flags from the oracle's dispatch of those indices
       equal the GPU's bit for bit, on every token (no exemption for flipped tokens).
    4. Against the routing of the oracle's own fp64 logits, a token may differ only when its
       top-k is decided by a gap below the near-tie margin; such tokens are counted."""
    od = oracle_dtype(cfg)
    Xn = np_host(inp.X)
    Wr = inp.W_r.cpu().numpy()
    bias = None if inp.bias is None else inp.bias.cpu().numpy()
    l64, l32 = oracle.router_logits(Xn, od, Wr, bias)
    scale = np.abs(to_f64(inp.X)) @ np.abs(Wr.astype(np.float64))
    got_l = ex["logits"].astype(np.float64)
    assert (np.abs(got_l - l64) <= 1e-5 * scale + 1e-6).all(), "router logits off their bound"
    rg = oracle.route(ex["logits"], k=cfg.k, renorm=cfg.renormalize)
    assert np.array_equal(ex["idx"], rg["idx"]), "selection differs on the GPU's own logits"
    np.testing.assert_allclose(ex["gate"], rg["gate"], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(ex["colsum"], rg["colsum"], rtol=1e-5, atol=1e-4)
    C = oracle.capacity(cfg.N, cfg.k, cfg.E, cfg.capacity_factor, cfg.min_capacity)
    dg = oracle.dispatch(ex["idx"], cfg.E, C, order=cfg.capacity_order)
    for key in ("load", "offsets", "pos", "dropped"):
        assert np.array_equal(ex[key], dg[key]), key
    ro = oracle.route(l32, k=cfg.k, renorm=cfg.renormalize)
    margin = oracle.topk_margin(l64, cfg.k)
    flips = (ex["idx"] != ro["idx"]).any(1)
    assert (margin[flips] < NEAR_TIE).all(), "routing differs on a token that is not near-tied"
    return dg, rg["gate"], int(flips.sum())


def tile_sample(cfg, ex, block=128, n_even=12):
    """Tokens whose records put a checked row in every 128-row block of every expert's segment
    of X_perm (the row tiles of the grouped GEMMs, and each CTA's half of a 256-row CTA-pair
    tile), in each expert's first and last row (its tail tile, M=64 or not), plus evenly
    spaced tokens and, under a capacity, tokens that lost one or all of their slots. The row
    inside a block varies from block to block. Rows map to tokens through the oracle's
    dispatch of the GPU's own routing (equal to the GPU's, checked by check_routing)."""
    C = oracle.capacity(cfg.N, cfg.k, cfg.E, cfg.capacity_factor, cfg.min_capacity)
    dg = oracle.dispatch(ex["idx"], cfg.E, C, order=cfg.capacity_order)
    off, row_token = dg["offsets"], dg["row_token"]
    rows = set()
    for e in range(cfg.E):
        o0, o1 = int(off[e]), int(off[e + 1])
        if o1 <= o0:
            continue
        rows.update((o0, o1 - 1))
        for b in range((o1 - o0 + block - 1) // block):
            rows.add(min(o1 - 1, o0 + b * block + (b * 53 + e * 17) % block))
    toks = {int(row_token[r]) for r in rows}
    toks.update(np.linspace(0, cfg.N - 1, n_even).astype(int).tolist())
    if cfg.capacity_factor > 0:
        d = dg["dropped"]
        toks.update(int(t) for t in np.where(d.all(1))[0][:2])
        toks.update(int(t) for t in np.where(d.any(1) & ~d.all(1))[0][:2])
    return sorted(toks)
