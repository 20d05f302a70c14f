"""GPU parity of the training-time routing variants and the z-loss (moe_route_ex,
moe_forward_ex) against the oracle: noisy top-k (Grok-1 book 5.2.2), GShard random routing of
the later experts (MoE series 3), z-loss = mean (log Z)^2 (Grok-1 book 5.2.2)."""
import numpy as np
import pytest
import torch

import oracle
from top_routing_expert_fp32_b200 import configs, inputs
from gpu_helpers import NEAR_TIE, np_host, oracle_dtype

pytestmark = pytest.mark.gpu

MODES = [configs.ROUTE_NOISY_TOPK, configs.ROUTE_GSHARD_RANDOM]


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


def _cfg(N, D, E, k, dtype=configs.DTYPE_BF16, renorm=1, mode=0, bias_var=0.0, **kw):
    return configs.MoEConfig("rv", N=N, D=D, F=64, E=E, k=k, dtype=dtype, activation=0,
                             renormalize=renorm, router_bias_var=bias_var, routing_mode=mode, **kw)


def _outs(N, E, k):
    return dict(logits=torch.empty((N, E), dtype=torch.float32, device="cuda"),
                idx=torch.full((N, k), -1, dtype=torch.int32, device="cuda"),
                gate=torch.full((N, k), float("nan"), dtype=torch.float32, device="cuda"),
                colsum=torch.empty((E,), dtype=torch.float32, device="cuda"),
                zloss=torch.empty((1,), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("N,E,k,renorm", [(1000, 8, 2, 1), (333, 13, 3, 0), (2050, 64, 8, 1),
                                          (65, 16, 1, 0)])
def test_route_ex_from_logits_bitexact(abi, mode, N, E, k, renorm):
    l32 = inputs.make_logits(N, E, seed=N + E).numpy()
    noise = inputs.make_noise(N, E, 1.0, seed=N)
    cfg = _cfg(N, 64, E, k, renorm=renorm, mode=mode)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    o = _outs(N, E, k)
    o["logits"].copy_(torch.from_numpy(l32))
    abi.route_ex(p, None, None, None, noise.cuda(), o["logits"], o["idx"], o["gate"], o["colsum"],
                 o["zloss"], ws)
    torch.cuda.synchronize()
    ref = oracle.route_ex(l32, k=k, renorm=renorm, mode=mode, noise=noise.numpy())
    assert np.array_equal(o["idx"].cpu().numpy(), ref["idx"])
    np.testing.assert_allclose(o["gate"].cpu().numpy(), ref["gate"], rtol=2e-6, atol=1e-7)
    np.testing.assert_allclose(o["colsum"].cpu().numpy(), ref["colsum"], rtol=1e-4, atol=1e-4)
    assert o["zloss"].item() == pytest.approx(ref["zloss"], rel=1e-5)
    assert abi.device_error(ws) == 0


@pytest.mark.parametrize("mode", [configs.ROUTE_TOPK] + MODES)
@pytest.mark.parametrize("dtype,N,D,E,k", [(configs.DTYPE_BF16, 515, 256, 8, 2),
                                           (configs.DTYPE_BF16, 1000, 2048, 64, 2),
                                           (configs.DTYPE_F32, 300, 200, 24, 2),
                                           (configs.DTYPE_BF16, 20000, 136, 64, 2)])
def test_route_ex_from_x(abi, mode, dtype, N, D, E, k):
    cfg = _cfg(N, D, E, k, dtype=dtype, mode=mode, bias_var=1.0)
    inp = inputs.make_inputs(cfg, "cuda", seed=5, weights=False)
    noise = inputs.make_noise(N, E, 0.5, seed=6)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    o = _outs(N, E, k)
    abi.route_ex(p, inp.X, inp.W_r, inp.bias, noise.cuda(), o["logits"], o["idx"], o["gate"],
                 o["colsum"], o["zloss"], ws)
    torch.cuda.synchronize()
    l64, l32 = oracle.router_logits(np_host(inp.X), oracle_dtype(cfg), inp.W_r.cpu().numpy(),
                                    inp.bias.cpu().numpy())
    ref = oracle.route_ex(l32, k=k, renorm=1, mode=mode, noise=noise.numpy())
    # decisions are taken on z (first pick of GSHARD, all of TOPK) and z + noise: a token may
    # differ only if one of those is near-tied
    margin = oracle.topk_margin(l64, k)
    if mode != configs.ROUTE_TOPK:
        margin = np.minimum(margin, oracle.topk_margin(l64 + noise.numpy().astype(np.float64), k))
    diff = (o["idx"].cpu().numpy() != ref["idx"]).any(1)
    assert (margin[diff] < NEAR_TIE).all()
    same = ~diff
    np.testing.assert_allclose(o["gate"].cpu().numpy()[same], ref["gate"][same], rtol=2e-5,
                               atol=1e-6)
    assert o["zloss"].item() == pytest.approx(ref["zloss"], rel=1e-4)


def test_forward_ex_gshard_with_capacity(abi):
    cfg = configs.MoEConfig("fex", N=500, D=128, F=256, E=16, k=2, dtype=configs.DTYPE_BF16,
                            activation=configs.ACT_SILU, renormalize=1, capacity_factor=1.0,
                            router_bias_var=2.0, routing_mode=configs.ROUTE_GSHARD_RANDOM)
    inp = inputs.make_inputs(cfg, "cuda")
    noise = inputs.make_noise(cfg.N, cfg.E, 1.0, seed=9).cuda()
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    idx = torch.empty((cfg.N, cfg.k), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.N, cfg.k), dtype=torch.float32, device="cuda")
    dropped = torch.empty((cfg.N, cfg.k), dtype=torch.uint8, device="cuda")
    zl = torch.empty((1,), dtype=torch.float32, device="cuda")
    out = torch.empty((cfg.N, cfg.D), dtype=torch.bfloat16, device="cuda")
    abi.forward_ex(p, inp.X, inp.W_r, inp.bias, noise, inp.W1, inp.W2, inp.W3, out, ws,
                   topk_idx=idx, topk_gate=gate, dropped=dropped, z_loss=zl)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    Xn = np_host(inp.X)
    l64, l32 = oracle.router_logits(Xn, oracle.BF16, inp.W_r.cpu().numpy(), inp.bias.cpu().numpy())
    ro = oracle.route_ex(l32, k=2, renorm=1, mode=cfg.routing_mode, noise=noise.cpu().numpy())
    flips = (idx.cpu().numpy() != ro["idx"]).any(1)
    margin = np.minimum(oracle.topk_margin(l64, 2),
                        oracle.topk_margin(l64 + noise.cpu().numpy().astype(np.float64), 2))
    assert (margin[flips] < NEAR_TIE).all()
    assert zl.item() == pytest.approx(ro["zloss"], rel=1e-4)
    if not flips.any():
        C = oracle.capacity(cfg.N, cfg.k, cfg.E, cfg.capacity_factor)
        do = oracle.dispatch(ro["idx"], cfg.E, C)
        assert np.array_equal(dropped.cpu().numpy(), do["dropped"])
        # layer output for a sample of tokens
        toks = np.arange(0, cfg.N, 25)
        rt, re_, sl = [], [], []
        for t in toks:
            for j in range(cfg.k):
                if not do["dropped"][t, j]:
                    rt.append(t); re_.append(ro["idx"][t, j]); sl.append((t, j))
        Y = oracle.expert_ffn(np.array(rt, np.int32), np.array(re_, np.int32), Xn,
                              np_host(inp.W1), np_host(inp.W2), np_host(inp.W3), oracle.BF16,
                              cfg.activation)
        ref = np.zeros((len(toks), cfg.D))
        row = {t: i for i, t in enumerate(toks)}
        for (t, j), y in zip(sl, Y):
            ref[row[t]] += ro["gate"][t, j] * y
        got = out.float().cpu().numpy().astype(np.float64)[toks]
        err = np.abs(got - ref).max(1) / np.maximum(np.abs(ref).max(1), 1e-30)
        assert err.max() <= 2e-2
