"""GPU parity of each kernel behind the C ABI against the CPU oracle, at sizes the oracle
finishes in seconds that span several tiles and ragged tails, plus edge cases.
Integer outputs bit-exact; floating point within the stated tolerances."""
import math

import numpy as np
import pytest
import torch

import oracle
from top_routing_expert_fp32_b200 import configs, inputs
from gpu_helpers import (NEAR_TIE, TOL_BF16, alloc_dispatch_out, alloc_route_out, np_host,
                         normwise_rel_err, oracle_dtype, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


def _cfg(N, D, F, E, k, dtype=configs.DTYPE_BF16, act=0, renorm=1, cf=0.0, bias_var=0.0,
         order=configs.ORDER_SLOT_MAJOR, drop_policy=configs.DROP_ZERO, min_capacity=0):
    return configs.MoEConfig("t", N=N, D=D, F=F, E=E, k=k, dtype=dtype, activation=act,
                             renormalize=renorm, capacity_factor=cf, router_bias_var=bias_var,
                             capacity_order=order, drop_policy=drop_policy,
                             min_capacity=min_capacity)


# ------------------------------------------------------------------ routing from given logits

@pytest.mark.parametrize("N,E,k,renorm,ties", [
    (1, 1, 1, 1, False), (7, 3, 2, 0, False), (64, 4, 2, 1, True), (1000, 8, 2, 1, False),
    (1000, 8, 2, 0, True), (4097, 8, 1, 1, False), (333, 13, 5, 0, True), (2048, 64, 2, 1, False),
    (2050, 64, 8, 0, True), (100, 64, 1, 1, True), (65, 16, 8, 0, False)])
def test_route_from_logits_bitexact(abi, oracle_lib, N, E, k, renorm, ties):
    if ties:
        rng = np.random.default_rng(N + E)
        l32 = rng.integers(-2, 3, size=(N, E)).astype(np.float32)
    else:
        l32 = inputs.make_logits(N, E, seed=N * 7 + E).numpy()
    cfg = _cfg(N, 64, 64, E, k, renorm=renorm)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    o = alloc_route_out(N, E, k)
    o["logits"].copy_(torch.from_numpy(l32))
    abi.route(p, None, None, None, o["logits"], o["idx"], o["gate"], o["colsum"], ws)
    torch.cuda.synchronize()
    ref = oracle_lib.route(l32, k=k, renorm=renorm)
    assert np.array_equal(o["idx"].cpu().numpy(), ref["idx"])
    np.testing.assert_allclose(o["gate"].cpu().numpy(), ref["gate"], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(o["colsum"].cpu().numpy(), ref["colsum"], rtol=1e-5, atol=1e-5)
    assert abi.device_error(ws) == 0


@pytest.mark.parametrize("dtype,N,D,E,k,renorm,bias_var", [
    (configs.DTYPE_BF16, 515, 256, 8, 2, 1, 0.0), (configs.DTYPE_BF16, 1000, 2048, 64, 2, 1, 2.0),
    (configs.DTYPE_F32, 64, 64, 4, 2, 1, 0.0), (configs.DTYPE_BF16, 77, 72, 6, 3, 0, 0.0),
    (configs.DTYPE_F32, 130, 100, 13, 1, 1, 1.0), (configs.DTYPE_BF16, 257, 6144, 8, 2, 0, 0.0),
    (configs.DTYPE_BF16, 600, 520, 33, 3, 1, 1.0), (configs.DTYPE_F32, 300, 200, 24, 2, 0, 0.0),
    (configs.DTYPE_BF16, 64, 4096, 8, 2, 1, 0.0), (configs.DTYPE_BF16, 129, 1000, 64, 8, 0, 2.0),
    (configs.DTYPE_BF16, 20000, 136, 64, 2, 1, 2.0), (configs.DTYPE_BF16, 300, 64, 1, 1, 1, 0.0),
    (configs.DTYPE_BF16, 1111, 328, 13, 4, 0, 1.0)])
def test_route_from_x(abi, oracle_lib, dtype, N, D, E, k, renorm, bias_var):
    cfg = _cfg(N, D, 64, E, k, dtype=dtype, renorm=renorm, bias_var=bias_var)
    inp = inputs.make_inputs(cfg, "cuda", seed=3, weights=False)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    o = alloc_route_out(N, E, k)
    abi.route(p, inp.X, inp.W_r, inp.bias, o["logits"], o["idx"], o["gate"], o["colsum"], ws)
    torch.cuda.synchronize()
    Xn = np_host(inp.X)
    l64, l32 = oracle_lib.router_logits(Xn, oracle_dtype(cfg), inp.W_r.cpu().numpy(),
                                        None if inp.bias is None else inp.bias.cpu().numpy())
    # fp32 accumulation error bound: relative to sum_d |x_d w_de|.
    scale = np.abs(to_f64(inp.X)) @ np.abs(inp.W_r.cpu().double().numpy())
    got_l = o["logits"].cpu().numpy().astype(np.float64)
    assert (np.abs(got_l - l64) <= 1e-5 * scale + 1e-6).all()
    ref = oracle_lib.route(l32, k=k, renorm=renorm)
    margin = oracle_lib.topk_margin(l64, k)
    got_idx = o["idx"].cpu().numpy()
    diff = (got_idx != ref["idx"]).any(1)
    assert (margin[diff] < NEAR_TIE).all(), "top-k mismatch on a token that is not near-tied"
    same = ~diff
    np.testing.assert_allclose(o["gate"].cpu().numpy()[same], ref["gate"][same], rtol=2e-5,
                               atol=1e-6)
    np.testing.assert_allclose(o["colsum"].cpu().numpy(), ref["colsum"], rtol=1e-4, atol=1e-4)


# Routing from X, checked on the GPU's own logits: the kernels that compute the logits take the
# routing decision in registers (bf16 X: the tensor-core router at every cluster size; fp32 X:
# the narrow and wide SIMT routers). Duplicate columns of W_r (and of the bias) make the
# logits of those experts bit-identical, so exact ties reach the in-kernel selection.
ROUTE_X_TIES = [
    # dtype, N, D, E, k, renorm, bias_var, cluster (MOE_ROUTE_CLUSTER; None = automatic)
    (configs.DTYPE_BF16, 515, 1024, 8, 2, 1, 0.0, 1),
    (configs.DTYPE_BF16, 515, 1024, 8, 2, 0, 1.0, 2),
    (configs.DTYPE_BF16, 515, 1024, 8, 3, 1, 0.0, 4),
    (configs.DTYPE_BF16, 515, 1024, 8, 2, 0, 0.0, 8),
    (configs.DTYPE_BF16, 130, 4096, 8, 2, 1, 0.0, None),
    (configs.DTYPE_BF16, 1000, 2048, 64, 2, 1, 2.0, 1),
    (configs.DTYPE_BF16, 300, 2048, 64, 8, 0, 2.0, 8),
    (configs.DTYPE_BF16, 777, 512, 13, 5, 0, 1.0, 2),
    (configs.DTYPE_BF16, 64, 6144, 8, 2, 0, 0.0, None),
    (configs.DTYPE_BF16, 257, 640, 33, 3, 1, 0.0, 4),
    (configs.DTYPE_F32, 300, 200, 8, 2, 1, 0.0, None),     # narrow
    (configs.DTYPE_F32, 130, 100, 16, 4, 0, 1.0, None),    # narrow, 16 experts
    (configs.DTYPE_F32, 300, 200, 24, 2, 0, 0.0, None),    # wide
    (configs.DTYPE_F32, 129, 64, 64, 8, 1, 2.0, None),     # wide, 64 experts
]


@pytest.mark.parametrize("dtype,N,D,E,k,renorm,bias_var,cluster", ROUTE_X_TIES)
def test_route_from_x_bitexact_on_own_logits_with_ties(abi, oracle_lib, monkeypatch, dtype, N,
                                                       D, E, k, renorm, bias_var, cluster):
    if cluster is None:
        monkeypatch.delenv("MOE_ROUTE_CLUSTER", raising=False)
    else:
        monkeypatch.setenv("MOE_ROUTE_CLUSTER", str(cluster))
    cfg = _cfg(N, D, 64, E, k, dtype=dtype, renorm=renorm, bias_var=bias_var)
    inp = inputs.make_inputs(cfg, "cuda", seed=5, weights=False)
    # expert e + E/2 (and e + 1 for a few odd E) repeats expert e's column and bias
    W_r = inp.W_r.clone()
    bias = None if inp.bias is None else inp.bias.clone()
    pairs = [(e, e + E // 2) for e in range(0, E // 2, 2)] or [(0, 0)]
    for src, dst in pairs:
        W_r[:, dst] = W_r[:, src]
        if bias is not None:
            bias[dst] = bias[src]
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    o = alloc_route_out(N, E, k)
    abi.route(p, inp.X, W_r, bias, o["logits"], o["idx"], o["gate"], o["colsum"], ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    lg = o["logits"].cpu().numpy()
    for src, dst in pairs:   # the ties are real: equal columns give bit-identical logits
        assert np.array_equal(lg[:, src].view(np.int32), lg[:, dst].view(np.int32))
    # router arithmetic: within the fp32 accumulation bound of the fp64 logits
    Wn = W_r.cpu().numpy()
    l64, _ = oracle_lib.router_logits(np_host(inp.X), oracle_dtype(cfg), Wn,
                                      None if bias is None else bias.cpu().numpy())
    scale = np.abs(to_f64(inp.X)) @ np.abs(Wn.astype(np.float64))
    assert (np.abs(lg.astype(np.float64) - l64) <= 1e-5 * scale + 1e-6).all()
    # selection, order (lower index first on ties) and gates: bit-exact on the same logits
    ref = oracle_lib.route(lg, k=k, renorm=renorm)
    idx = o["idx"].cpu().numpy()
    assert np.array_equal(idx, ref["idx"])
    np.testing.assert_allclose(o["gate"].cpu().numpy(), ref["gate"], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(o["colsum"].cpu().numpy(), ref["colsum"], rtol=1e-5, atol=1e-5)
    # some selections were decided by the tie rule: both copies of a tied expert selected,
    # the lower index first
    tie_decided = 0
    for src, dst in pairs:
        if src == dst:
            continue
        both = (idx == src).any(1) & (idx == dst).any(1)
        first_src = np.argmax(idx == src, axis=1) < np.argmax(idx == dst, axis=1)
        assert first_src[both].all()
        tie_decided += int(both.sum())
    if E >= 4 and k >= 2:
        assert tie_decided > 0


# ------------------------------------------------------------------ dispatch (bit-exact)

def _dispatch_case(abi, oracle_lib, N, E, k, cf, seed, skew=0.0, all_one=False, X=None,
                   order=configs.ORDER_SLOT_MAJOR, min_capacity=0):
    l32 = inputs.make_logits(N, E, seed=seed).numpy()
    if skew:
        l32 = l32 + (np.arange(E, dtype=np.float32)[::-1] * skew)
    idx = oracle_lib.route(l32, k=k, renorm=1)["idx"]
    if all_one:
        idx = np.tile(np.arange(k, dtype=np.int32), (N, 1))
    dtype = configs.DTYPE_F32 if (X is not None and X.dtype == torch.float32) else configs.DTYPE_BF16
    cfg = _cfg(N, X.shape[1] if X is not None else 64, 64, E, k, dtype=dtype, cf=cf,
               order=order, min_capacity=min_capacity)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    d = alloc_dispatch_out(N, E, k)
    idx_d = torch.from_numpy(idx).cuda()
    X_perm = None
    if X is not None:
        X_perm = torch.full((N * k, X.shape[1]), float("nan"), dtype=X.dtype, device="cuda")
    abi.dispatch(p, X, idx_d, d["load"], d["offsets"], d["pos"], d["dropped"], d["row_token"],
                 X_perm, ws)
    torch.cuda.synchronize()
    C = abi.capacity(p)
    assert C == oracle_lib.capacity(N, k, E, cf, min_capacity)
    ref = oracle_lib.dispatch(idx, E, C, order=order)
    assert np.array_equal(d["load"].cpu().numpy(), ref["load"])
    assert np.array_equal(d["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(d["pos"].cpu().numpy(), ref["pos"])
    assert np.array_equal(d["dropped"].cpu().numpy(), ref["dropped"])
    nk = int(ref["offsets"][E])
    assert np.array_equal(d["row_token"].cpu().numpy()[:nk], ref["row_token"])
    assert abi.device_error(ws) == 0
    # the one-launch dispatch's grid-barrier counters (workspace header ints 20, 21) are back
    # at zero for the next call
    hdr = ws[:256].view(torch.int32).cpu()
    assert hdr[20].item() == 0 and hdr[21].item() == 0
    return d, ref, X_perm


@pytest.mark.parametrize("N,E,k,cf,skew", [
    (1, 1, 1, 0.0, 0), (5, 3, 2, 0.3, 0), (64, 4, 2, 0.0, 0), (1000, 8, 2, 0.0, 0),
    (1000, 8, 2, 1.0, 0.5), (5000, 8, 2, 1.25, 0.3), (16384, 64, 2, 1.25, 0.05),
    (16384, 64, 1, 1.25, 0.05), (3001, 13, 3, 0.7, 0.2), (2049, 64, 8, 1.0, 0.0),
    (1025, 2, 1, 0.5, 0)])
def test_dispatch_bitexact(abi, oracle_lib, N, E, k, cf, skew):
    _dispatch_case(abi, oracle_lib, N, E, k, cf, seed=N + E + k, skew=skew)


def test_dispatch_more_chunks_than_resident_blocks(abi, oracle_lib):
    # 700,000 records = 684 chunks of 1024: more than the blocks that fit on the device at once,
    # so the one-launch dispatch's blocks loop over chunks; twice in a row on one workspace.
    for cf in (1.25, 0.0):
        _dispatch_case(abi, oracle_lib, 350000, 8, 2, cf, seed=77, skew=0.2)


@pytest.mark.parametrize("N,E,k,cf,skew,minc", [
    (5, 3, 2, 0.3, 0, 0), (1000, 8, 2, 1.0, 0.5, 0), (5000, 8, 2, 1.25, 0.3, 700),
    (16384, 64, 2, 1.0, 0.05, 256), (3001, 13, 3, 0.7, 0.2, 0), (2049, 64, 8, 1.0, 0.0, 40),
    (1025, 2, 1, 0.5, 0, 0), (700, 16, 4, 0.25, 0.1, 1000)])
def test_dispatch_token_major_bitexact(abi, oracle_lib, N, E, k, cf, skew, minc):
    # The walkthrough's dispatch loop order (3.2), with GShard's min_capacity floor (2.1).
    _dispatch_case(abi, oracle_lib, N, E, k, cf, seed=N + E + k + 1, skew=skew,
                   order=configs.ORDER_TOKEN_MAJOR, min_capacity=minc)


def test_dispatch_min_capacity_slot_major(abi, oracle_lib):
    d, ref, _ = _dispatch_case(abi, oracle_lib, 3000, 8, 2, 0.25, seed=5, skew=0.2,
                               min_capacity=500)
    assert ref["offsets"][-1] <= 8 * 500 and ref["dropped"].any()


def test_dispatch_all_records_to_one_expert_set(abi, oracle_lib):
    d, ref, _ = _dispatch_case(abi, oracle_lib, 3000, 8, 2, 1.25, seed=1, all_one=True)
    assert ref["dropped"].any()


def test_dispatch_zero_tokens(abi):
    cfg = _cfg(0, 64, 64, 8, 2)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    d = alloc_dispatch_out(1, 8, 2)
    d["load"].fill_(5)
    d["offsets"].fill_(5)
    idx = torch.zeros((1, 2), dtype=torch.int32, device="cuda")
    abi.dispatch(p, None, idx, d["load"], d["offsets"], d["pos"], d["dropped"], d["row_token"],
                 None, ws)
    torch.cuda.synchronize()
    assert (d["load"] == 0).all() and (d["offsets"] == 0).all()


def test_dispatch_bad_index_reported(abi, oracle_lib):
    N, E, k = 300, 8, 2
    idx = oracle_lib.route(inputs.make_logits(N, E, seed=4).numpy(), k=k, renorm=1)["idx"].copy()
    idx[17, 1] = E          # out of range
    idx[200, 0] = -3        # out of range
    cfg = _cfg(N, 64, 64, E, k)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    d = alloc_dispatch_out(N, E, k)
    abi.dispatch(p, None, torch.from_numpy(idx).cuda(), d["load"], d["offsets"], d["pos"],
                 d["dropped"], d["row_token"], None, ws)
    assert abi.device_error(ws) == abi.DEVERR_BAD_INDEX
    dr = d["dropped"].cpu().numpy()
    assert dr[17, 1] == 1 and dr[200, 0] == 1
    assert d["load"].cpu().numpy().sum() == N * k - 2
    assert abi.device_error(ws) == 0  # cleared


@pytest.mark.parametrize("N,D,E,k,cf,dtype", [
    (1000, 4096, 8, 2, 0.0, configs.DTYPE_BF16), (777, 8, 4, 2, 0.5, configs.DTYPE_BF16),
    (300, 16384, 8, 2, 1.0, configs.DTYPE_BF16), (64, 64, 4, 2, 0.0, configs.DTYPE_F32),
    (2500, 2048, 64, 2, 1.25, configs.DTYPE_BF16), (129, 6144, 8, 1, 0.0, configs.DTYPE_BF16)])
def test_gather_exact(abi, oracle_lib, N, D, E, k, cf, dtype):
    X = inputs.randn((N, D), 1.0, inputs.torch_dtype(dtype), "cuda", seed=5, tid=1)
    d, ref, X_perm = _dispatch_case(abi, oracle_lib, N, E, k, cf, seed=9, X=X)
    nk = int(ref["offsets"][E])
    rt = torch.from_numpy(ref["row_token"]).long().cuda()
    assert torch.equal(X_perm[:nk].view(torch.int16 if X.dtype == torch.bfloat16 else torch.int32),
                       X[rt].view(torch.int16 if X.dtype == torch.bfloat16 else torch.int32))
    if nk < N * k:   # rows past the kept records are left untouched
        assert torch.isnan(X_perm[nk:].float()).all()


# ------------------------------------------------------------------ grouped expert FFN

def _tile_env(monkeypatch, tile_rows):
    # "128": one CTA per 128-row tile; "256": CTA pairs (tcgen05 cta_group::2) sharing a
    # 256-row tile; "256w": CTA pairs with two MMAs per k-step into one 512-column accumulator,
    # the tiles of a short last round split into half tiles (one MMA each; with fewer tiles
    # than half the pairs, as in most cases here, every tile); "256wf": the same with whole
    # tiles only.
    monkeypatch.setenv("MOE_GEMM_TILE_ROWS", tile_rows[:3])
    monkeypatch.setenv("MOE_GEMM_WIDE", "1" if "w" in tile_rows else "0")
    monkeypatch.setenv("MOE_GEMM_HALVES", "0" if tile_rows.endswith("wf") else "1")


def _ffn_case(abi, oracle_lib, counts, D, F, act, dtype=configs.DTYPE_BF16, seed=0):
    E = len(counts)
    R = int(sum(counts))
    cfg = _cfg(max(R, 1), D, F, E, 1, dtype=dtype, act=act)
    tdt = inputs.torch_dtype(dtype)
    Xp = inputs.randn((max(R, 1), D), 1.0, tdt, "cuda", seed, 1)
    W1 = inputs.randn((E, D, F), 1 / math.sqrt(D), tdt, "cuda", seed, 3)
    W2 = inputs.randn((E, D, F), 1 / math.sqrt(D), tdt, "cuda", seed, 4)
    W3 = inputs.randn((E, F, D), 1 / math.sqrt(F), tdt, "cuda", seed, 5)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    H = torch.full((max(R, 1), F), float("nan"), dtype=tdt, device="cuda")
    Y = torch.full((max(R, 1), D), float("nan"), dtype=tdt, device="cuda")
    abi.expert_ffn(p, Xp, offsets, W1, W2, W3, H, Y, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    if R == 0:
        return
    rec_e = np.repeat(np.arange(E, dtype=np.int32), counts)
    ref = oracle_lib.expert_ffn(np.arange(R, dtype=np.int32), rec_e, np_host(Xp), np_host(W1),
                                np_host(W2), np_host(W3), oracle_dtype(cfg), act)
    err = normwise_rel_err(to_f64(Y[:R]), ref)
    tol = TOL_BF16 if dtype == configs.DTYPE_BF16 else 1e-5
    assert err.max() <= tol, f"max normwise rel err {err.max():.3g}"
    return err


@pytest.mark.parametrize("counts,D,F,act", [
    ([128], 64, 256, configs.ACT_SILU),
    ([128], 128, 128, configs.ACT_SILU),
    ([0, 1, 300], 128, 256, configs.ACT_SILU),
    ([129, 127, 128, 0, 5, 256, 1, 64], 256, 384, configs.ACT_GELU_ERF),
    ([70, 0, 33], 72, 200, configs.ACT_GELU_TANH),
    ([513, 400], 1024, 512, configs.ACT_SILU),
    ([16, 17, 15, 16, 16, 16, 16, 16], 4096, 1024, configs.ACT_SILU),
    ([700, 0, 257, 1100], 512, 768, configs.ACT_GELU_ERF),
])
@pytest.mark.parametrize("tile_rows", ["128", "256", "256w", "256wf"])
def test_expert_ffn_bf16_tcgen05(abi, oracle_lib, monkeypatch, counts, D, F, act, tile_rows):
    _tile_env(monkeypatch, tile_rows)
    _ffn_case(abi, oracle_lib, counts, D, F, act)


@pytest.mark.parametrize("counts,D,F", [
    ([129, 127, 128, 0, 5, 256, 1, 64], 256, 384),
    ([700, 0, 257, 1100], 512, 768),
    ([3, 0, 200, 1, 64, 65, 0, 128, 7], 128, 1280),
])
@pytest.mark.parametrize("tile_rows,ngroup", [("128", "2"), ("128", "4"), ("256", "3"),
                                              ("256w", "2"), ("256wf", "2")])
def test_expert_ffn_tile_groups(abi, oracle_lib, monkeypatch, counts, D, F, tile_rows, ngroup):
    # Tiles visited in groups of column blocks (a shorter last group included).
    _tile_env(monkeypatch, tile_rows)
    monkeypatch.setenv("MOE_GEMM_NGROUP", ngroup)
    _ffn_case(abi, oracle_lib, counts, D, F, configs.ACT_SILU, seed=3)


@pytest.mark.parametrize("counts,D,F", [
    ([5], 64, 128),                                   # 1 tile: surplus CTAs take none
    ([129, 127, 128, 0, 5, 256, 1, 64], 256, 384),
    ([2000, 1500, 0, 2600], 256, 2048),               # many tiles per CTA
])
@pytest.mark.parametrize("tile_rows", ["128", "256", "256w", "256wf"])
@pytest.mark.parametrize("order", ["dynamic", "static"])
def test_expert_ffn_tile_counter_returns_to_zero(abi, oracle_lib, monkeypatch, counts, D, F,
                                                 tile_rows, order):
    # Tiles are handed out in order by a counter in the workspace header (ints 16 and 17);
    # every launch returns it to zero, so back-to-back launches on one workspace give the same
    # bits and see every tile. The static round-robin order (MOE_GEMM_SCHED=static) gives the
    # same results.
    _tile_env(monkeypatch, tile_rows)
    monkeypatch.setenv("MOE_GEMM_SCHED", order)
    E = len(counts)
    R = int(sum(counts))
    cfg = _cfg(R, D, F, E, 1)
    Xp = inputs.randn((R, D), 1.0, torch.bfloat16, "cuda", 7, 1)
    W1 = inputs.randn((E, D, F), 1 / math.sqrt(D), torch.bfloat16, "cuda", 7, 3)
    W2 = inputs.randn((E, D, F), 1 / math.sqrt(D), torch.bfloat16, "cuda", 7, 4)
    W3 = inputs.randn((E, F, D), 1 / math.sqrt(F), torch.bfloat16, "cuda", 7, 5)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    outs = []
    for _ in range(3):
        H = torch.full((R, F), float("nan"), dtype=torch.bfloat16, device="cuda")
        Y = torch.full((R, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        abi.expert_ffn(p, Xp, offsets, W1, W2, W3, H, Y, ws)
        torch.cuda.synchronize()
        hdr = ws[:256].view(torch.int32).cpu()
        assert hdr[16].item() == 0 and hdr[17].item() == 0
        outs.append((H, Y))
    assert abi.device_error(ws) == 0
    for H, Y in outs[1:]:
        assert torch.equal(H.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(Y.view(torch.int16), outs[0][1].view(torch.int16))
    sel = np.unique(np.concatenate([np.arange(0, R, max(1, R // 50)), [R - 1]]))
    rec_e = np.repeat(np.arange(E, dtype=np.int32), counts)[sel]
    ref = oracle_lib.expert_ffn(sel.astype(np.int32), rec_e, np_host(Xp), np_host(W1),
                                np_host(W2), np_host(W3), oracle.BF16, configs.ACT_SILU)
    err = normwise_rel_err(to_f64(outs[0][1][sel]), ref)
    assert err.max() <= TOL_BF16, f"max normwise rel err {err.max():.3g}"


@pytest.mark.parametrize("halves", ["0", "1", "all"])
@pytest.mark.parametrize("counts,D,F", [
    # up: 25 row blocks x 7 column blocks = 175 tiles; down: 25 x 3 = 75. On 74 pairs both
    # leave a last round of 27 and 1 tiles, which the default splits (whole and half tiles in
    # one launch).
    ([2000, 1500, 0, 2600], 1536, 1792),
    ([300, 0, 513, 40, 1], 1024, 1280),
])
def test_expert_ffn_half_tiles(abi, oracle_lib, monkeypatch, halves, counts, D, F):
    # Wide tiles split into two half-width tiles (one N=256 MMA, half the output columns):
    # never, for a short last round (default), or all of them. Same bits in every mode (the
    # MMAs of an output column are the same), and the oracle on sampled rows.
    _tile_env(monkeypatch, "256w")
    monkeypatch.setenv("MOE_GEMM_HALVES", halves)
    E = len(counts)
    R = int(sum(counts))
    cfg = _cfg(R, D, F, E, 1, act=configs.ACT_GELU_ERF)
    Xp = inputs.randn((R, D), 1.0, torch.bfloat16, "cuda", 11, 1)
    W1 = inputs.randn((E, D, F), 1 / math.sqrt(D), torch.bfloat16, "cuda", 11, 3)
    W2 = inputs.randn((E, D, F), 1 / math.sqrt(D), torch.bfloat16, "cuda", 11, 4)
    W3 = inputs.randn((E, F, D), 1 / math.sqrt(F), torch.bfloat16, "cuda", 11, 5)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    H = torch.full((R, F), float("nan"), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((R, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    abi.expert_ffn(p, Xp, offsets, W1, W2, W3, H, Y, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    assert not torch.isnan(H.float()).any() and not torch.isnan(Y.float()).any()
    monkeypatch.setenv("MOE_GEMM_HALVES", "0")
    H0 = torch.empty_like(H)
    Y0 = torch.empty_like(Y)
    abi.expert_ffn(p, Xp, offsets, W1, W2, W3, H0, Y0, ws)
    torch.cuda.synchronize()
    assert torch.equal(H.view(torch.int16), H0.view(torch.int16))
    assert torch.equal(Y.view(torch.int16), Y0.view(torch.int16))
    sel = np.unique(np.concatenate([np.arange(0, R, max(1, R // 40)), np.cumsum(counts) - 1,
                                    [R - 1]]))
    rec_e = np.repeat(np.arange(E, dtype=np.int32), counts)[sel]
    ref = oracle_lib.expert_ffn(sel.astype(np.int32), rec_e, np_host(Xp), np_host(W1),
                                np_host(W2), np_host(W3), oracle.BF16, configs.ACT_GELU_ERF)
    err = normwise_rel_err(to_f64(Y[sel]), ref)
    assert err.max() <= TOL_BF16, f"max normwise rel err {err.max():.3g}"


def test_expert_ffn_f32(abi, oracle_lib):
    err = _ffn_case(abi, oracle_lib, [40, 0, 57, 31], 64, 128, configs.ACT_SILU,
                    dtype=configs.DTYPE_F32)
    assert err.max() <= 1e-5


def _act64(x, act):
    """The activations in float64 (LLMs-from-scratch 12.1; Grok-1 book 5.3.5)."""
    if act == configs.ACT_SILU:
        return x / (1.0 + np.exp(-x))
    if act == configs.ACT_GELU_ERF:
        return x * 0.5 * np.array([math.erfc(-v / math.sqrt(2.0)) for v in x])
    u = math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)
    return x / (1.0 + np.exp(-2.0 * u))      # = x (1 + tanh u) / 2, which cancels in float64 too


def _bf16_grid(limit):
    # every finite bf16 value with 2^-20 <= |v| <= limit, and zero
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    bits = bits[(bits & 0x7F80) != 0x7F80]          # no inf / NaN patterns
    v = (bits << 16).view(np.float32).astype(np.float64)
    v = v[(np.abs(v) <= limit) & ((np.abs(v) >= 2.0 ** -20) | (v == 0))]
    return np.unique(v)


@pytest.mark.parametrize("dtype", [configs.DTYPE_F32, configs.DTYPE_BF16])
@pytest.mark.parametrize("act", [configs.ACT_SILU, configs.ACT_GELU_ERF, configs.ACT_GELU_TANH])
def test_activation_values_through_the_up_projection(abi, dtype, act):
    # H = act(x W1) (.) (x W2) with x_r = e_r, W1[r, f] = the value to test and W2 = 1: every
    # pre-activation reaches the epilogue exactly (one exact product, the rest zeros), so H is
    # the kernel's activation of a chosen value, checked against float64 over [-14, 14] on
    # every value of magnitude >= 1e-30: relative error within 1e-6 (4 + x^2) (the activations'
    # relative condition number grows like x^2 in the negative tail, so each fp32 rounding
    # inside, of x^2 or of the tanh argument, costs up to about x^2 2^-24 there), plus half a
    # bf16 ulp on the bf16 tensor-core path. The negative tails included: there the forms
    # 1 + erf(x / sqrt 2) and 1 + tanh(u) cancel to zero in fp32.
    D = 64
    if dtype == configs.DTYPE_F32:
        vals = np.unique(np.concatenate([np.linspace(-14.0, 14.0, 64 * 4096 - 200),
                                         -np.logspace(-20, 1, 100), np.logspace(-20, 1, 100)])
                         .astype(np.float32)).astype(np.float64)
    else:
        vals = _bf16_grid(14.0)
    F = -(-len(vals) // (D * 64)) * 64
    grid = np.zeros(D * F)
    grid[:len(vals)] = vals
    grid = grid.reshape(D, F)
    cfg = _cfg(D, D, F, 1, 1, dtype=dtype, act=act)
    tdt = inputs.torch_dtype(dtype)
    Xp = torch.eye(D, dtype=torch.float32, device="cuda").to(tdt)
    W1 = torch.tensor(grid, dtype=torch.float32, device="cuda").to(tdt).reshape(1, D, F)
    W2 = torch.ones((1, D, F), dtype=tdt, device="cuda")
    assert np.array_equal(W1.float().cpu().numpy().reshape(D, F), grid)   # exactly representable
    offsets = torch.tensor([0, D], dtype=torch.int32, device="cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    H = torch.full((D, F), float("nan"), dtype=tdt, device="cuda")
    abi.expert_up(p, Xp, offsets, W1, W2, H, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    x = grid.ravel()
    got = H.double().cpu().numpy().ravel()
    ref = _act64(x, act)
    assert np.isfinite(got).all()
    sel = np.abs(ref) >= 1e-30
    rel = 1e-6 * (4.0 + x * x)
    if dtype == configs.DTYPE_F32:
        bound = rel * np.abs(ref)
    else:
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-300))) - 7)
        bound = 0.5 * ulp + rel * np.abs(ref)
    bad = sel & (np.abs(got - ref) > bound)
    assert not bad.any(), (f"{bad.sum()} values off, first x={x[bad][:5]} "
                           f"got={got[bad][:5]} ref={ref[bad][:5]}")
    assert (np.abs(got[~sel] - ref[~sel]) <= 1e-6 * np.maximum(1.0, np.abs(x[~sel]))).all()


def test_expert_ffn_empty(abi, oracle_lib):
    _ffn_case(abi, oracle_lib, [0, 0, 0], 64, 128, configs.ACT_SILU)


# ------------------------------------------------------------------ combine

@pytest.mark.parametrize("N,D,E,k,cf,dtype", [
    (1000, 4096, 8, 2, 0.0, configs.DTYPE_BF16), (500, 2048, 64, 2, 1.0, configs.DTYPE_BF16),
    (64, 64, 4, 2, 0.0, configs.DTYPE_F32), (300, 72, 5, 3, 0.4, configs.DTYPE_BF16),
    (257, 1024, 8, 1, 0.5, configs.DTYPE_F32),
    # a warp per token (N >= 16 per SM) and a block per token, with up to 8 records per token
    (3000, 264, 8, 2, 0.0, configs.DTYPE_BF16), (2500, 136, 64, 8, 1.0, configs.DTYPE_BF16),
    (200, 264, 64, 8, 1.0, configs.DTYPE_BF16), (100, 96, 13, 5, 0.0, configs.DTYPE_F32),
    (2400, 100, 16, 6, 0.6, configs.DTYPE_F32)])
def test_combine(abi, oracle_lib, N, D, E, k, cf, dtype):
    tdt = inputs.torch_dtype(dtype)
    d, ref, _ = _dispatch_case(abi, oracle_lib, N, E, k, cf, seed=11)
    R = N * k
    Y = inputs.randn((R, D), 1.0, tdt, "cuda", 12, 1)
    rng = np.random.default_rng(3)
    gate = torch.from_numpy(rng.random((N, k)).astype(np.float32)).cuda()
    idx = oracle_lib.route(inputs.make_logits(N, E, seed=11).numpy(), k=k, renorm=1)["idx"]
    cfg = _cfg(N, D, 64, E, k, dtype=dtype, cf=cf)
    p = abi.problem(cfg)
    out = torch.empty((N, D), dtype=tdt, device="cuda")
    abi.combine(p, Y, torch.from_numpy(idx).cuda(), gate, d["offsets"], d["pos"], d["dropped"],
                out)
    torch.cuda.synchronize()
    rows = ref["offsets"][idx] + ref["pos"]
    Yrec = to_f64(Y)[np.where(ref["dropped"] == 1, 0, rows)]
    oref = oracle_lib.combine(gate.cpu().double().numpy(), ref["dropped"], Yrec)
    err = normwise_rel_err(to_f64(out), oref)
    assert err.max() <= (8e-3 if dtype == configs.DTYPE_BF16 else 1e-6)
    allgone = ref["dropped"].all(1)
    assert (to_f64(out)[allgone] == 0).all()


@pytest.mark.parametrize("N,D,E,k,cf,dtype", [
    (2500, 136, 64, 8, 0.7, configs.DTYPE_BF16), (200, 96, 13, 5, 0.5, configs.DTYPE_F32),
    (500, 2048, 64, 2, 1.0, configs.DTYPE_BF16), (300, 72, 5, 3, 0.4, configs.DTYPE_BF16),
    (257, 1024, 8, 4, 0.5, configs.DTYPE_F32), (1000, 4096, 8, 2, 0.6, configs.DTYPE_BF16)])
def test_combine_case_a_reweight(abi, oracle_lib, N, D, E, k, cf, dtype):
    # MoE series 2.2 case A: a token that lost some slots gives the whole weight to the kept ones.
    tdt = inputs.torch_dtype(dtype)
    d, ref, _ = _dispatch_case(abi, oracle_lib, N, E, k, cf, seed=13, skew=0.2)
    partial = ref["dropped"].any(1) & ~ref["dropped"].all(1)
    assert partial.any()
    R = N * k
    Y = inputs.randn((R, D), 1.0, tdt, "cuda", 14, 1)
    rng = np.random.default_rng(5)
    gate = torch.from_numpy(rng.random((N, k)).astype(np.float32)).cuda()
    idx = oracle_lib.route(inputs.make_logits(N, E, seed=13).numpy() +
                           (np.arange(E, dtype=np.float32)[::-1] * 0.2), k=k, renorm=1)["idx"]
    cfg = _cfg(N, D, 64, E, k, dtype=dtype, cf=cf, drop_policy=configs.DROP_RENORM_KEPT)
    p = abi.problem(cfg)
    out = torch.empty((N, D), dtype=tdt, device="cuda")
    abi.combine(p, Y, torch.from_numpy(idx).cuda(), gate, d["offsets"], d["pos"], d["dropped"],
                out)
    torch.cuda.synchronize()
    rows = ref["offsets"][idx] + ref["pos"]
    Yrec = to_f64(Y)[np.where(ref["dropped"] == 1, 0, rows)]
    oref = oracle_lib.combine(gate.cpu().double().numpy(), ref["dropped"], Yrec,
                              policy=oracle_lib.DROP_RENORM_KEPT)
    err = normwise_rel_err(to_f64(out), oref)
    assert err.max() <= (8e-3 if dtype == configs.DTYPE_BF16 else 1e-6)
    assert (to_f64(out)[ref["dropped"].all(1)] == 0).all()
