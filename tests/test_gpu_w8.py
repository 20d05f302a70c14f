"""GPU parity of the 8-bit expert-weight path (moe_expert_up_w8 / moe_expert_down_w8 /
moe_forward_w8, and their K-contiguous variants after moe_pack_w8) against the oracle's fp64
dequantized experts (W = q * s per expert and output column; Grok-1 book 5.3.3, 5.3.5)."""
import math

import numpy as np
import pytest
import torch

import oracle
from top_routing_expert_fp32_b200 import configs, inputs
from gpu_helpers import (TOL_BF16, alloc_dispatch_out, alloc_route_out, check_routing,
                         normwise_rel_err, np_host, tile_sample, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


def _cfg(N, D, F, E, k=1, act=configs.ACT_SILU, **kw):
    return configs.MoEConfig("w8", N=N, D=D, F=F, E=E, k=k, dtype=configs.DTYPE_BF16,
                             activation=act, renormalize=1, **kw)


def _packed(abi, p, w):
    """The K-contiguous copies of w's 8-bit matrices (moe_pack_w8), scales shared."""
    W1p = torch.empty(w.W1q.shape[0], w.W1q.shape[2], w.W1q.shape[1], dtype=torch.int8,
                      device="cuda")
    W2p = torch.empty_like(W1p)
    W3p = torch.empty(w.W3q.shape[0], w.W3q.shape[2], w.W3q.shape[1], dtype=torch.int8,
                      device="cuda")
    abi.pack_w8(p, w.W1q, w.W2q, w.W3q, W1p, W2p, W3p)
    return inputs.MoEWeights8(W1p, w.S1, W2p, w.S2, W3p, w.S3)


def _ffn_w8(abi, counts, D, F, act, seed=0, packed=False):
    E = len(counts)
    R = int(sum(counts))
    cfg = _cfg(max(R, 1), D, F, E, act=act)
    Xp = inputs.randn((max(R, 1), D), 1.0, torch.bfloat16, "cuda", seed, 1)
    w = inputs.make_w8_weights(cfg, "cuda", seed)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    H = torch.full((max(R, 1), F), float("nan"), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((max(R, 1), D), float("nan"), dtype=torch.bfloat16, device="cuda")
    if packed:
        wp = _packed(abi, p, w)
        abi.expert_up_w8p(p, Xp, offsets, wp.W1q, wp.S1, wp.W2q, wp.S2, H, ws)
        abi.expert_down_w8p(p, H, offsets, wp.W3q, wp.S3, Y, ws)
    else:
        abi.expert_up_w8(p, Xp, offsets, w.W1q, w.S1, w.W2q, w.S2, H, ws)
        abi.expert_down_w8(p, H, offsets, w.W3q, w.S3, Y, ws)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    return cfg, Xp, w, offsets, H, Y, R


@pytest.mark.parametrize("counts,D,F,act", [
    ([128], 64, 256, configs.ACT_SILU),
    ([0, 1, 300], 128, 256, configs.ACT_SILU),
    ([129, 127, 128, 0, 5, 256, 1, 64], 256, 384, configs.ACT_GELU_ERF),
    ([70, 0, 33], 80, 208, configs.ACT_GELU_TANH),
    ([16, 17, 15, 16, 16, 16, 16, 16], 4096, 1024, configs.ACT_SILU),
    ([700, 0, 257, 1100], 512, 400, configs.ACT_GELU_ERF),
])
@pytest.mark.parametrize("kernel", ["smem", "tmem", "packed", "tmem_a_in_smem",
                                    "packed_a_in_smem"])
def test_expert_ffn_w8_matches_oracle(abi, monkeypatch, counts, D, F, act, kernel):
    # smem: the shared-memory kernel (larger batches); tmem: the transposed kernel for few rows
    # per expert, its converted weights the MMA's A operand in tensor memory (default) or, for
    # the *_a_in_smem cases, in shared memory; packed: the transposed kernel on K-contiguous
    # weights from moe_pack_w8.
    monkeypatch.setenv("MOE_W8_KERNEL", "smem" if kernel == "smem" else "tmem")
    monkeypatch.setenv("MOE_W8T_A", "smem" if kernel.endswith("_a_in_smem") else "tmem")
    kernel = kernel.replace("_a_in_smem", "")
    cfg, Xp, w, offsets, H, Y, R = _ffn_w8(abi, counts, D, F, act, packed=kernel == "packed")
    rec_e = np.repeat(np.arange(len(counts), dtype=np.int32), counts)
    ref = oracle.expert_ffn_w8(np.arange(R, dtype=np.int32), rec_e, np_host(Xp), oracle.BF16,
                               w.W1q.cpu().numpy(), w.S1.cpu().numpy(), w.W2q.cpu().numpy(),
                               w.S2.cpu().numpy(), w.W3q.cpu().numpy(), w.S3.cpu().numpy(), act)
    err = normwise_rel_err(to_f64(Y[:R]), ref)
    assert err.max() <= TOL_BF16, f"max normwise rel err {err.max():.3g}"


def test_unit_scales_reproduce_bf16_kernel_bit_for_bit(abi, monkeypatch):
    # int8 -> bf16 is exact and a unit scale is exact, so with the same 128-row tiles the 8-bit
    # path must give the bf16 path's bits on W = q.
    monkeypatch.setenv("MOE_GEMM_TILE_ROWS", "128")
    monkeypatch.setenv("MOE_W8_KERNEL", "smem")
    counts, D, F = [129, 3, 200, 64], 256, 384
    cfg, Xp, w, offsets, H8, Y8, R = _ffn_w8(abi, counts, D, F, configs.ACT_SILU, seed=4)
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    one = lambda s: torch.ones_like(s)
    H1 = torch.empty_like(H8)
    Y1 = torch.empty_like(Y8)
    abi.expert_up_w8(p, Xp, offsets, w.W1q, one(w.S1), w.W2q, one(w.S2), H1, ws)
    abi.expert_down_w8(p, H1, offsets, w.W3q, one(w.S3), Y1, ws)
    W1, W2, W3 = (q.to(torch.bfloat16) for q in (w.W1q, w.W2q, w.W3q))
    Hb = torch.empty_like(H8)
    Yb = torch.empty_like(Y8)
    abi.expert_up(p, Xp, offsets, W1, W2, Hb, ws)
    abi.expert_down(p, Hb, offsets, W3, Yb, ws)
    torch.cuda.synchronize()
    assert torch.equal(H1[:R].view(torch.int16), Hb[:R].view(torch.int16))
    assert torch.equal(Y1[:R].view(torch.int16), Yb[:R].view(torch.int16))


@pytest.mark.parametrize("E,k,n", [(1, 16, 16), (3, 80, 208), (2, 4096, 48), (5, 1040, 336)])
def test_pack_w8_is_exact_transpose(abi, E, k, n):
    # W1q/W2q are [E, D, F] (k = D rows), W3q is [E, F, D]: moe_pack_w8 transposes each
    # expert's matrix, ragged 32 x 32 tiles included, byte for byte.
    cfg = _cfg(16, k, n, E)
    p = abi.problem(cfg)
    g = torch.Generator(device="cuda").manual_seed(E * 7 + k + n)
    rnd = lambda *sh: torch.randint(-128, 128, sh, generator=g, device="cuda",
                                    dtype=torch.int32).to(torch.int8)
    w = inputs.MoEWeights8(rnd(E, k, n), None, rnd(E, k, n), None, rnd(E, n, k), None)
    wp = _packed(abi, p, w)
    torch.cuda.synchronize()
    assert torch.equal(wp.W1q, w.W1q.transpose(1, 2))
    assert torch.equal(wp.W2q, w.W2q.transpose(1, 2))
    assert torch.equal(wp.W3q, w.W3q.transpose(1, 2))


@pytest.mark.parametrize("a_loc", ["smem", "tmem"])
def test_packed_reproduces_tmem_kernel_bit_for_bit(abi, monkeypatch, a_loc):
    # The same bf16 values of q enter the same MMAs in the same order, only the staging layout
    # differs, so H and Y match the unpacked transposed kernel bit for bit.
    monkeypatch.setenv("MOE_W8_KERNEL", "tmem")
    monkeypatch.setenv("MOE_W8T_A", a_loc)
    counts, D, F = [0, 65, 3, 130, 64, 1], 336, 208
    _, _, _, _, Hu, Yu, R = _ffn_w8(abi, counts, D, F, configs.ACT_GELU_TANH, seed=9)
    _, _, _, _, Hp, Yp, _ = _ffn_w8(abi, counts, D, F, configs.ACT_GELU_TANH, seed=9,
                                    packed=True)
    assert torch.equal(Hu[:R].view(torch.int16), Hp[:R].view(torch.int16))
    assert torch.equal(Yu[:R].view(torch.int16), Yp[:R].view(torch.int16))


def test_w8_rejected_without_bf16_or_16_multiples(abi):
    from top_routing_expert_fp32_b200.abi import MoEError
    cfg = _cfg(64, 24, 64, 4)           # D % 16 != 0
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    t = torch.zeros(16, dtype=torch.int8, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(MoEError):
        abi.expert_up_w8(p, f, t, t, f, t, f, f, ws)


def _forward_w8_check(abi, cfg, sample=None, packed=False):
    """The 8-bit layer against the oracle's fp64 dequantized experts, from the GPU's routing
    (check_routing: logits within their bound, selection and dispatch of the GPU's own logits
    bit-exact, near-tie flips counted). sample="tiles": a checked row in every row tile."""
    inp = inputs.make_inputs(cfg, "cuda", weights=False)
    w = inputs.make_w8_weights(cfg, "cuda")
    p = abi.problem(cfg)
    ws = abi.workspace(p)
    wk = _packed(abi, p, w) if packed else w
    N, E, k = cfg.N, cfg.E, cfg.k
    r = alloc_route_out(N, E, k)
    d = alloc_dispatch_out(N, E, k)
    out = torch.empty((N, cfg.D), dtype=torch.bfloat16, device="cuda")
    abi.forward_w8(p, inp.X, inp.W_r, inp.bias, wk, out, ws, logits=r["logits"],
                   topk_idx=r["idx"], topk_gate=r["gate"], load=d["load"], offsets=d["offsets"],
                   pos=d["pos"], dropped=d["dropped"], prob_colsum=r["colsum"], packed=packed)
    torch.cuda.synchronize()
    assert abi.device_error(ws) == 0
    ex = {key: v.cpu().numpy() for key, v in {**r, **d}.items()}
    dg, gate, flips = check_routing(cfg, inp, ex)
    Xn = np_host(inp.X)
    if isinstance(sample, str):
        sample = tile_sample(cfg, ex)
    toks = np.arange(N) if sample is None else np.asarray(sample)
    rec_t, rec_e, slot = [], [], []
    for t in toks:
        for j in range(k):
            if not dg["dropped"][t, j]:
                rec_t.append(t)
                rec_e.append(ex["idx"][t, j])
                slot.append((t, j))
    Y = oracle.expert_ffn_w8(np.array(rec_t, np.int32), np.array(rec_e, np.int32), Xn,
                             oracle.BF16, w.W1q.cpu().numpy(), w.S1.cpu().numpy(),
                             w.W2q.cpu().numpy(), w.S2.cpu().numpy(), w.W3q.cpu().numpy(),
                             w.S3.cpu().numpy(), cfg.activation)
    ref = np.zeros((len(toks), cfg.D))
    row = {t: i for i, t in enumerate(toks)}
    for (t, j), y in zip(slot, Y):
        ref[row[t]] += gate[t, j] * y
    err = normwise_rel_err(to_f64(out)[toks], ref)
    assert err.max() <= TOL_BF16, f"max normwise rel err {err.max():.3g}"
    return len(toks), flips


@pytest.mark.parametrize("cfg", [
    _cfg(300, 256, 512, 8, k=2),
    _cfg(500, 128, 256, 16, k=2, capacity_factor=1.0, router_bias_var=2.0),
    _cfg(257, 384, 640, 8, k=2, act=configs.ACT_GELU_ERF).with_(renormalize=0),
], ids=["silu_e8", "capacity_e16", "gelu_norenorm"])
@pytest.mark.parametrize("packed", [False, True], ids=["kn", "packed"])
def test_forward_w8_small_all_tokens(abi, cfg, packed):
    n, flips = _forward_w8_check(abi, cfg, packed=packed)
    assert n == cfg.N


@pytest.mark.parametrize("name,packed", [("decode", False), ("mixtral", False),
                                         ("decode", True)])
def test_forward_w8_full_size_sampled(abi, name, packed):
    cfg = configs.CONFIGS[name]
    _forward_w8_check(abi, cfg, "tiles", packed=packed)
    torch.cuda.empty_cache()
