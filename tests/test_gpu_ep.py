"""GPU checks of the expert-parallel pieces: moe_gather_rows (the local reorders) and
ep.forward on this library's kernels over an NCCL group of one rank (the exchanges run as
NCCL all-to-alls on one GPU; the multi-rank bookkeeping is covered on CPU with gloo)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from top_routing_expert_fp32_b200 import configs, ep, inputs
from gpu_helpers import NEAR_TIE, TOL_BF16, normwise_rel_err, np_host, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


@pytest.mark.parametrize("n_src,n,shape,dtype", [
    (1000, 2500, (4096,), torch.bfloat16),    # 8 KB rows, repeated indices
    (37, 37, (6,), torch.bfloat16),           # 12-byte rows: 4-byte words
    (513, 1, (3, 8), torch.float32),          # 96-byte rows
    (64, 0, (8,), torch.bfloat16),            # nothing to gather
])
def test_gather_rows_matches_indexing(abi, n_src, n, shape, dtype):
    g = torch.Generator(device="cuda").manual_seed(n_src + n)
    src = torch.randn((n_src,) + shape, generator=g, device="cuda").to(dtype)
    index = torch.randint(0, n_src, (n,), generator=g, device="cuda", dtype=torch.int32)
    dst = torch.full((max(n, 1),) + shape, float("nan"), device="cuda", dtype=dtype)[:n]
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    abi.gather_rows(src, index, dst, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    ref = src[index.long()]
    assert torch.equal(dst.view(torch.uint8), ref.view(torch.uint8))


def test_gather_rows_bad_index_is_reported_and_zero_filled(abi):
    # The kernel's own bounds check turns an out-of-range index into MOE_DEVERR_BAD_INDEX and
    # a zero row; nothing outside src is read.
    src = torch.randn((16, 64), device="cuda").to(torch.bfloat16)
    index = torch.tensor([3, -1, 16, 15, 2**31 - 1], dtype=torch.int32, device="cuda")
    dst = torch.full((5, 64), 7.0, device="cuda", dtype=torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    abi.gather_rows(src, index, dst, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == abi.DEVERR_BAD_INDEX
    assert torch.equal(dst[0], src[3]) and torch.equal(dst[3], src[15])
    assert (dst[[1, 2, 4]].float() == 0).all()
    assert abi.device_error(ws) == 0          # reading the error word clears it


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def nccl_group():
    from datetime import timedelta
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60))
    yield None
    dist.destroy_process_group()


def _cfg(N, D, F, E, k, **kw):
    return configs.MoEConfig("ep", N=N, D=D, F=F, E=E, k=k, dtype=configs.DTYPE_BF16,
                             activation=configs.ACT_SILU, renormalize=1, **kw)


@pytest.mark.parametrize("cfg", [
    _cfg(300, 256, 512, 8, 2),
    _cfg(500, 128, 384, 16, 2, capacity_factor=1.0, router_bias_var=2.0),
    _cfg(257, 384, 640, 8, 1),
], ids=["e8k2", "capacity_e16", "k1"])
def test_ep_forward_one_rank_matches_oracle_and_forward(abi, nccl_group, cfg):
    inp = inputs.make_inputs(cfg, "cuda")
    comp = ep.CudaCompute(cfg, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3)
    out, info = ep.forward(comp, inp.X, cfg.E)
    torch.cuda.synchronize()
    assert comp.device_error() == 0
    # same layer through moe_forward
    layer_out = torch.empty_like(out)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    idx = torch.empty((cfg.N, cfg.k), dtype=torch.int32, device="cuda")
    abi.forward(p, inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, layer_out, ws, topk_idx=idx)
    torch.cuda.synchronize()
    assert normwise_rel_err(to_f64(out), to_f64(layer_out)).max() <= 1e-2
    # and the oracle, on every token whose selection is not a near tie
    Xn = np_host(inp.X)
    ref = oracle.forward(Xn, inp.W_r.cpu().numpy(), None if inp.bias is None else
                         inp.bias.cpu().numpy(), np_host(inp.W1), np_host(inp.W2),
                         np_host(inp.W3), k=cfg.k, cf=cfg.capacity_factor, renorm=1,
                         act=cfg.activation, dtype=oracle.BF16)
    l64, _ = oracle.router_logits(Xn, oracle.BF16, inp.W_r.cpu().numpy(),
                                  None if inp.bias is None else inp.bias.cpu().numpy())
    flips = (idx.cpu().numpy() != ref["idx"]).any(1)
    assert (oracle.topk_margin(l64, cfg.k)[flips] < NEAR_TIE).all()
    if cfg.capacity_factor > 0 and flips.any():
        pytest.skip("near-tie flip under capacity changes other tokens' slots")
    err = normwise_rel_err(to_f64(out)[~flips], ref["out"][~flips])
    assert err.max() <= TOL_BF16, f"max normwise rel err {err.max():.3g}"
    plan = info["plan"]
    assert plan.send_rows == plan.recv_rows
    if not flips.any():
        assert plan.send_rows == [int(ref["offsets"][cfg.E])]
        assert plan.local_offsets.tolist() == ref["offsets"].tolist()


def test_ep_forward_one_rank_full_size_mixtral(abi, nccl_group):
    # The benchmark's layer (N=4096, D=4096, F=14336, E=8, k=2) through ep.forward against
    # moe_forward on the same inputs (the oracle checks moe_forward at this size).
    cfg = configs.CONFIGS["mixtral"]
    inp = inputs.make_inputs(cfg, "cuda")
    comp = ep.CudaCompute(cfg, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3)
    out, info = ep.forward(comp, inp.X, cfg.E)
    ref = torch.empty_like(out)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    abi.forward(p, inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, ref, ws)
    torch.cuda.synchronize()
    assert comp.device_error() == 0 and abi.device_error(ws) == 0
    assert info["plan"].send_rows == [cfg.N * cfg.k]
    assert normwise_rel_err(to_f64(out), to_f64(ref)).max() <= 1e-2
    del inp, comp, out, ref, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg,world", [
    (_cfg(300, 256, 512, 8, 2), 2),
    (_cfg(400, 128, 384, 5, 2, capacity_factor=1.0, router_bias_var=2.0), 2),   # 3 + 2 experts
    (_cfg(257, 384, 640, 8, 1), 3),                                             # 3 + 3 + 2
], ids=["e8k2_world2", "capacity_e5_world2", "k1_world3"])
def test_ep_ranks_with_expert_subsets_on_one_gpu(abi, cfg, world):
    # The compute of every rank of an expert-parallel layer, run here on one GPU: each rank
    # routes and dispatches its own tokens over all E experts, runs the grouped FFN of its own
    # expert block on the rows it receives (sliced weights, rows in the planned expert-major
    # order), reorders the outputs back and combines what comes back to it. The exchanges
    # themselves are replayed by indexing (the NCCL path is ep.forward; the multi-rank
    # bookkeeping is tested on gloo). Every rank's output must equal the oracle's experts on
    # its own routing.
    ranges = ep.expert_ranges(cfg.E, world)
    full = inputs.make_inputs(cfg, "cuda")
    Xs = [full.X] + [inputs.randn((cfg.N, cfg.D), 1.0, full.X.dtype, "cuda", cfg.seed + 1 + r,
                                  inputs.TID_X) for r in range(1, world)]
    comps = [ep.CudaCompute(cfg, full.W_r, full.bias,
                            *(w[e0:e1].contiguous() for w in (full.W1, full.W2, full.W3)))
             for (e0, e1) in ranges]
    routed = [comps[s].route_dispatch(Xs[s]) for s in range(world)]
    offs = [r["offsets"].cpu().numpy().astype(np.int64) for r in routed]
    back = [[None] * world for _ in range(world)]   # back[source][owner]
    for r, (e0, e1) in enumerate(ranges):
        recv_counts = np.array([[offs[s][e + 1] - offs[s][e] for e in range(e0, e1)]
                                for s in range(world)], dtype=np.int64)
        plan = ep.plan_exchange(offs[r], recv_counts, ranges)
        assert plan.send_rows == [int(offs[r][b] - offs[r][a]) for a, b in ranges]
        X_recv = torch.cat([routed[s]["X_perm"][offs[s][e0]:offs[s][e1]] for s in range(world)])
        assert X_recv.shape[0] == sum(plan.recv_rows)
        X_loc = comps[r].gather_rows(X_recv, plan.to_expert_major)
        Y_loc = comps[r].expert_ffn(X_loc, plan.local_offsets, (e0, e1))
        Y_recv = comps[r].gather_rows(Y_loc, plan.to_source_major)
        base = np.concatenate([[0], np.cumsum(plan.recv_rows)])
        for s in range(world):
            back[s][r] = Y_recv[base[s]:base[s + 1]]
    for s in range(world):
        Y_back = torch.cat(back[s])       # owners in expert order = the source's X_perm order
        out = comps[s].combine(Y_back, routed[s])
        torch.cuda.synchronize()
        assert comps[s].device_error() == 0
        idx = routed[s]["idx"].cpu().numpy()
        gate = routed[s]["gate"].cpu().numpy().astype(np.float64)
        dropped = routed[s]["dropped"].cpu().numpy()
        C = oracle.capacity(cfg.N, cfg.k, cfg.E, cfg.capacity_factor)
        do = oracle.dispatch(idx, cfg.E, C)
        assert np.array_equal(do["offsets"], offs[s]) and np.array_equal(do["dropped"], dropped)
        kept = np.argwhere(dropped == 0)
        Xn = np_host(Xs[s])
        Y = oracle.expert_ffn(kept[:, 0].astype(np.int32), idx[dropped == 0].astype(np.int32),
                              Xn, np_host(full.W1), np_host(full.W2), np_host(full.W3),
                              oracle.BF16, cfg.activation)
        ref = np.zeros((cfg.N, cfg.D))
        for (t, j), y in zip(kept, Y):
            ref[t] += gate[t, j] * y
        err = normwise_rel_err(to_f64(out), ref)
        assert err.max() <= TOL_BF16, f"rank {s}: max normwise rel err {err.max():.3g}"
    del comps, routed, full
    torch.cuda.empty_cache()
