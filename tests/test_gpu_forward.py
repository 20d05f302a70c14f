"""End-to-end GPU parity of moe_forward (the path the benchmark times) against the oracle.

Small layers are compared on every token. The five named workloads run at their full sizes,
in the same launch configuration the benchmark uses. For every token the oracle checks the
router's fp32 logits against its fp64 ones, and its own selection and dispatch of the GPU's
exported logits bit for bit against the GPU's (near-tie flips against the fp64 routing are
counted). The layer output is then checked from the GPU's routing on a sample of tokens that
puts a checked row in every row tile of the grouped GEMMs."""
import numpy as np
import pytest
import torch

import oracle
from top_routing_expert_fp32_b200 import configs, inputs
from gpu_helpers import (alloc_dispatch_out, alloc_route_out, check_routing, np_host,
                         normwise_rel_err, oracle_dtype, tile_sample, to_f64, tol)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


def run_forward(abi, cfg, inp):
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    r = alloc_route_out(cfg.N, cfg.E, cfg.k)
    d = alloc_dispatch_out(cfg.N, cfg.E, cfg.k)
    out = torch.empty((cfg.N, cfg.D), dtype=inp.X.dtype, device="cuda")
    abi.forward(p, inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, out, ws,
                logits=r["logits"], topk_idx=r["idx"], topk_gate=r["gate"], load=d["load"],
                offsets=d["offsets"], pos=d["pos"], dropped=d["dropped"],
                prob_colsum=r["colsum"])
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    ex = {k: v.cpu().numpy() for k, v in {**r, **d}.items()}
    return out, ex


def check_layer(cfg, inp, out, ex, sample=None):
    """Routing checks (check_routing), then the layer output on the sampled tokens (all tokens
    when sample is None) against the oracle's fp64 experts and combine, taken from the GPU's
    routing (the oracle's dispatch of the GPU's indices and the oracle's gates of the GPU's
    logits): every sampled token is compared, flipped or not. Returns a summary dict."""
    od = oracle_dtype(cfg)
    Xn = np_host(inp.X)
    dg, gate, flips = check_routing(cfg, inp, ex)
    toks = np.arange(cfg.N) if sample is None else np.asarray(sample)
    rec_t, rec_e, slot = [], [], []
    for t in toks:
        for j in range(cfg.k):
            if not dg["dropped"][t, j]:
                rec_t.append(t)
                rec_e.append(ex["idx"][t, j])
                slot.append((t, j))
    Y = oracle.expert_ffn(np.array(rec_t, np.int32), np.array(rec_e, np.int32), Xn,
                          np_host(inp.W1), np_host(inp.W2), np_host(inp.W3), od, cfg.activation)
    ref = np.zeros((len(toks), cfg.D))
    row_of = {t: i for i, t in enumerate(toks)}
    # Gates as the combine applies them (MoE series 2.2 case A under DROP_RENORM_KEPT).
    g_eff = gate.copy()
    if cfg.drop_policy == configs.DROP_RENORM_KEPT:
        kept = dg["dropped"] == 0
        partial = kept.any(1) & ~kept.all(1)
        ksum = (gate * kept).sum(1)
        g_eff[partial] = gate[partial] / ksum[partial, None]
    for (t, j), y in zip(slot, Y):
        ref[row_of[t]] += g_eff[t, j] * y
    got = to_f64(out)[toks]
    err = normwise_rel_err(got, ref)
    assert err.max() <= tol(cfg), f"max normwise rel err {err.max():.3g} > {tol(cfg)}"
    all_dropped = dg["dropped"][toks].all(1)
    assert (got[all_dropped] == 0).all()
    return dict(flips=flips, max_err=float(err.max()), tokens=len(toks),
                records=len(rec_t), drop_rate=oracle.drop_rate(dg["dropped"]))


SMALL = [
    configs.CONFIGS["tiny_f32"],
    configs.MoEConfig("small_silu", N=300, D=256, F=512, E=8, k=2, dtype=configs.DTYPE_BF16,
                      activation=configs.ACT_SILU, renormalize=1),
    configs.MoEConfig("small_gelu_norenorm", N=257, D=384, F=640, E=8, k=2,
                      dtype=configs.DTYPE_BF16, activation=configs.ACT_GELU_ERF, renormalize=0),
    configs.MoEConfig("small_capacity", N=500, D=128, F=256, E=16, k=2, dtype=configs.DTYPE_BF16,
                      activation=configs.ACT_SILU, renormalize=1, capacity_factor=1.0,
                      router_bias_var=2.0),
    configs.MoEConfig("small_capacity_k1", N=500, D=128, F=256, E=16, k=1,
                      dtype=configs.DTYPE_BF16, activation=configs.ACT_SILU, renormalize=1,
                      capacity_factor=0.8, router_bias_var=2.0),
    configs.MoEConfig("small_f32_gelu_tanh", N=96, D=64, F=96, E=5, k=3, dtype=configs.DTYPE_F32,
                      activation=configs.ACT_GELU_TANH, renormalize=0, capacity_factor=0.9),
    # capacity policies: token-major positions, GShard case-A reweight, min_capacity floor
    configs.MoEConfig("small_token_major", N=500, D=128, F=256, E=16, k=2,
                      dtype=configs.DTYPE_BF16, activation=configs.ACT_SILU, renormalize=1,
                      capacity_factor=1.0, router_bias_var=2.0,
                      capacity_order=configs.ORDER_TOKEN_MAJOR),
    configs.MoEConfig("small_gshard", N=500, D=128, F=256, E=16, k=2,
                      dtype=configs.DTYPE_BF16, activation=configs.ACT_SILU, renormalize=1,
                      capacity_factor=0.5, router_bias_var=2.0,
                      capacity_order=configs.ORDER_TOKEN_MAJOR,
                      drop_policy=configs.DROP_RENORM_KEPT, min_capacity=40),
    configs.MoEConfig("small_case_a_k3_norenorm", N=300, D=128, F=192, E=8, k=3,
                      dtype=configs.DTYPE_BF16, activation=configs.ACT_GELU_ERF, renormalize=0,
                      capacity_factor=0.6, router_bias_var=1.0,
                      drop_policy=configs.DROP_RENORM_KEPT),
    configs.MoEConfig("small_f32_token_major_case_a", N=96, D=64, F=96, E=5, k=3,
                      dtype=configs.DTYPE_F32, activation=configs.ACT_SILU, renormalize=1,
                      capacity_factor=0.7, capacity_order=configs.ORDER_TOKEN_MAJOR,
                      drop_policy=configs.DROP_RENORM_KEPT),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_forward_small_all_tokens(abi, cfg):
    inp = inputs.make_inputs(cfg, "cuda")
    out, ex = run_forward(abi, cfg, inp)
    s = check_layer(cfg, inp, out, ex)
    assert s["tokens"] == cfg.N


def test_forward_deterministic_and_host_entry(abi):
    cfg = SMALL[3]
    inp = inputs.make_inputs(cfg, "cuda")
    out1, _ = run_forward(abi, cfg, inp)
    out2, _ = run_forward(abi, cfg, inp)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    p = abi.problem(cfg)
    ws = abi.workspace(p, host=True)
    xh = inp.X.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    abi.forward_host(p, xh, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, oh, ws)
    assert torch.equal(oh.view(torch.int16), out1.cpu().view(torch.int16))


def test_forward_zero_tokens(abi):
    cfg = SMALL[1].with_(N=0)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    inp = inputs.make_inputs(SMALL[1].with_(N=1), "cuda")
    out = torch.empty((1, cfg.D), dtype=torch.bfloat16, device="cuda")
    abi.forward(p, inp.X, inp.W_r, None, inp.W1, inp.W2, inp.W3, out, ws)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["tiny_f32", "decode", "mixtral", "capacity", "capacity_k1",
                                  "capacity_gshard", "grok1"])
def test_forward_named_workload_full_size(abi, name):
    cfg = configs.CONFIGS[name]
    inp = inputs.make_inputs(cfg, "cuda")
    out, ex = run_forward(abi, cfg, inp)
    sample = None if cfg.N <= 64 else tile_sample(cfg, ex)
    s = check_layer(cfg, inp, out, ex, sample)
    print(f"\n{name}: {s}")
    del inp
    torch.cuda.empty_cache()


def test_forward_host_two_halves_equal_forward_on_each_half(abi):
    # Without capacity moe_forward_host runs the batch as two pipelined halves; each half's
    # output must be exactly moe_forward on that half alone.
    cfg = configs.MoEConfig("split", N=1501, D=256, F=512, E=8, k=2, dtype=configs.DTYPE_BF16,
                            activation=configs.ACT_SILU, renormalize=1)
    inp = inputs.make_inputs(cfg, "cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p, host=True)
    xh = inp.X.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    abi.forward_host(p, xh, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, oh, ws)
    n0 = cfg.N // 2
    for lo, hi in ((0, n0), (n0, cfg.N)):
        ph = abi.problem(cfg, N=hi - lo)
        wsh = abi.workspace(ph)
        o = torch.empty((hi - lo, cfg.D), dtype=torch.bfloat16, device="cuda")
        abi.forward(ph, inp.X[lo:hi].contiguous(), inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, o, wsh)
        torch.cuda.synchronize()
        assert torch.equal(o.cpu().view(torch.int16), oh[lo:hi].view(torch.int16))


@pytest.mark.parametrize("cfg,nb", [
    (configs.MoEConfig("many", N=700, D=256, F=512, E=8, k=2, dtype=configs.DTYPE_BF16,
                       activation=configs.ACT_SILU, renormalize=1), 5),
    (configs.MoEConfig("many_cap", N=500, D=128, F=256, E=16, k=2, dtype=configs.DTYPE_BF16,
                       activation=configs.ACT_SILU, renormalize=1, capacity_factor=1.0), 3),
    (configs.MoEConfig("many_one", N=64, D=256, F=512, E=8, k=2, dtype=configs.DTYPE_BF16,
                       activation=configs.ACT_GELU_ERF, renormalize=0), 1),
], ids=["e8_5batches", "capacity_3batches", "one_batch"])
def test_forward_host_many_equals_forward_per_batch(abi, cfg, nb):
    # Each batch of the streamed call is a complete layer call on its own tokens (capacity per
    # batch): its output must be moe_forward's on that batch, bit for bit, whatever the overlap.
    inp = inputs.make_inputs(cfg, "cuda")
    Xb = torch.stack([inputs.randn((cfg.N, cfg.D), 1.0, torch.bfloat16, "cuda", 40 + b,
                                   inputs.TID_X) for b in range(nb)])
    p = abi.problem(cfg)
    ws = abi.workspace(p, host=True)
    xh = Xb.cpu().pin_memory()
    oh = torch.full_like(xh, float("nan")).pin_memory()
    abi.forward_host_many(p, xh, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, oh, ws)
    assert abi.device_error(ws) == 0
    wsd = abi.workspace(p)
    for b in range(nb):
        o = torch.empty((cfg.N, cfg.D), dtype=torch.bfloat16, device="cuda")
        abi.forward(p, Xb[b], inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, o, wsd)
        torch.cuda.synchronize()
        assert torch.equal(o.cpu().view(torch.int16), oh[b].view(torch.int16)), f"batch {b}"


def test_forward_host_many_zero_batches_is_a_no_op(abi):
    cfg = SMALL[1]
    inp = inputs.make_inputs(cfg, "cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p, host=True)
    xh = torch.empty((0, cfg.N, cfg.D), dtype=torch.bfloat16).pin_memory()
    oh = torch.empty_like(xh)
    abi.forward_host_many(p, xh, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, oh, ws)


def test_concurrent_layers_on_two_streams_equal_sequential(abi):
    # Calls on different streams with their own workspaces share no state: run two layers
    # (different sizes and policies) concurrently and compare with sequential runs, bit for bit.
    cfgs = [configs.MoEConfig("s0", N=1500, D=256, F=512, E=8, k=2, dtype=configs.DTYPE_BF16,
                              activation=configs.ACT_SILU, renormalize=1),
            configs.MoEConfig("s1", N=900, D=128, F=256, E=16, k=2, dtype=configs.DTYPE_BF16,
                              activation=configs.ACT_GELU_ERF, renormalize=0,
                              capacity_factor=1.0)]
    inps = [inputs.make_inputs(c, "cuda", seed=20 + i) for i, c in enumerate(cfgs)]
    ps = [abi.problem(c) for c in cfgs]
    wss = [abi.workspace(p) for p in ps]
    seq = []
    for c, inp, p, ws in zip(cfgs, inps, ps, wss):
        o = torch.empty((c.N, c.D), dtype=torch.bfloat16, device="cuda")
        abi.forward(p, inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, o, ws)
        seq.append(o)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(o) for o in seq]
    for _ in range(3):
        for c, inp, p, ws, st, o in zip(cfgs, inps, ps, wss, streams, outs):
            abi.forward(p, inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, o, ws,
                        stream=st)
    torch.cuda.synchronize()
    for ws in wss:
        assert abi.device_error(ws) == 0
    for a, b in zip(seq, outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["capacity", "mixtral"])
def test_diagnostics_from_the_layer_match_the_oracle(abi, name):
    # Balance loss and drop rate (moe_balance_loss / moe_drop_rate) from the GPU layer's own
    # load, prob_colsum and dropped, against the oracle's routing of the same inputs.
    cfg = configs.CONFIGS[name]
    inp = inputs.make_inputs(cfg, "cuda", weights=False)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    r = alloc_route_out(cfg.N, cfg.E, cfg.k)
    d = alloc_dispatch_out(cfg.N, cfg.E, cfg.k)
    X_perm = torch.empty((cfg.N * cfg.k, cfg.D), dtype=inp.X.dtype, device="cuda")
    abi.route(p, inp.X, inp.W_r, inp.bias, r["logits"], r["idx"], r["gate"], r["colsum"], ws)
    abi.dispatch(p, inp.X, r["idx"], d["load"], d["offsets"], d["pos"], d["dropped"],
                 d["row_token"], X_perm, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    loss = abi.balance_loss(p, d["load"], r["colsum"])
    rate = abi.drop_rate(p, d["dropped"])
    Xn = np_host(inp.X)
    bias = None if inp.bias is None else inp.bias.cpu().numpy()
    l64, l32 = oracle.router_logits(Xn, oracle_dtype(cfg), inp.W_r.cpu().numpy(), bias)
    ro = oracle.route(l32, k=cfg.k, renorm=cfg.renormalize)
    flips = int((r["idx"].cpu().numpy() != ro["idx"]).any(1).sum())
    do = oracle.dispatch(ro["idx"], cfg.E, oracle.capacity(cfg.N, cfg.k, cfg.E,
                                                           cfg.capacity_factor))
    ref_loss = oracle.balance_loss(cfg.N, cfg.k, do["load"], ro["colsum"])
    ref_rate = oracle.drop_rate(do["dropped"])
    # a near-tie flip moves one record between experts: 1 / (N k) in f, a few in the drops
    assert loss == pytest.approx(ref_loss, rel=1e-4 + 4 * flips / (cfg.N * cfg.k))
    assert abs(rate - ref_rate) <= 2 * flips / (cfg.N * cfg.k) + 1e-12
    if name == "capacity":
        assert rate > 0.0
    del X_perm
    torch.cuda.empty_cache()
