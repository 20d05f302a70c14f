"""Out-of-bounds write checks without a sanitizer: every output, intermediate and workspace
buffer handed to the library sits between guard bands filled with a byte pattern, and after
the calls every guard byte must be unchanged. Ragged shapes (tails of every tile size),
capacity drops, 8-bit weights and the row gather are covered."""
import numpy as np
import pytest
import torch

from top_routing_expert_fp32_b200 import configs, inputs

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps the interior 256-byte aligned)
PATTERN = 0xA5


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


class Guarded:
    """A tensor of `shape` and `dtype` inside a byte buffer with pattern-filled guard bands."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + ((n + 255) // 256) * 256 + GUARD,), PATTERN,
                              dtype=torch.uint8, device="cuda")
        self.n = n
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self):
        torch.cuda.synchronize()
        pre = self.raw[:GUARD]
        post = self.raw[GUARD + self.n:]
        return bool((pre == PATTERN).all()) and bool((post == PATTERN).all())


def _workspace(abi, p, host=False):
    n = abi.workspace_size(p, host)
    g = Guarded((max(n, 256),), torch.uint8)
    abi.lib.moe_workspace_init(g.t.data_ptr(), g.t.numel(), None)
    return g


CASES = [
    configs.MoEConfig("g_ragged", N=333, D=200, F=328, E=8, k=2, dtype=configs.DTYPE_BF16,
                      activation=configs.ACT_SILU, renormalize=1),
    configs.MoEConfig("g_capacity", N=517, D=128, F=256, E=16, k=2, dtype=configs.DTYPE_BF16,
                      activation=configs.ACT_GELU_ERF, renormalize=0, capacity_factor=1.0,
                      router_bias_var=2.0),
    configs.MoEConfig("g_pairs", N=1600, D=256, F=384, E=4, k=1, dtype=configs.DTYPE_BF16,
                      activation=configs.ACT_SILU, renormalize=1),
    configs.MoEConfig("g_f32", N=70, D=64, F=96, E=4, k=2, dtype=configs.DTYPE_F32,
                      activation=configs.ACT_GELU_TANH, renormalize=1),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_step_entry_points_write_only_their_buffers(abi, cfg):
    inp = inputs.make_inputs(cfg, "cuda")
    p = abi.problem(cfg)
    N, D, F, E, k = cfg.N, cfg.D, cfg.F, cfg.E, cfg.k
    R = N * k
    dt = inp.X.dtype
    ws = _workspace(abi, p)
    b = {name: Guarded(shape, t) for name, shape, t in [
        ("logits", (N, E), torch.float32), ("idx", (N, k), torch.int32),
        ("gate", (N, k), torch.float32), ("colsum", (E,), torch.float32),
        ("load", (E,), torch.int32), ("offsets", (E + 1,), torch.int32),
        ("pos", (N, k), torch.int32), ("dropped", (N, k), torch.uint8),
        ("row_token", (R,), torch.int32), ("X_perm", (R, D), dt), ("H", (R, F), dt),
        ("Y", (R, D), dt), ("out", (N, D), dt), ("out2", (N, D), dt)]}
    t = {n: g.t for n, g in b.items()}
    abi.route(p, inp.X, inp.W_r, inp.bias, t["logits"], t["idx"], t["gate"], t["colsum"], ws.t)
    abi.dispatch(p, inp.X, t["idx"], t["load"], t["offsets"], t["pos"], t["dropped"],
                 t["row_token"], t["X_perm"], ws.t)
    abi.expert_up(p, t["X_perm"], t["offsets"], inp.W1, inp.W2, t["H"], ws.t)
    abi.expert_down(p, t["H"], t["offsets"], inp.W3, t["Y"], ws.t)
    abi.combine(p, t["Y"], t["idx"], t["gate"], t["offsets"], t["pos"], t["dropped"], t["out"])
    abi.forward(p, inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, t["out2"], ws.t)
    torch.cuda.synchronize()
    assert abi.device_error(ws.t) == 0
    bad = [n for n, g in b.items() if not g.intact()]
    assert not bad, f"guard bands overwritten around {bad}"
    assert ws.intact(), "workspace guard overwritten"
    assert torch.equal(t["out"].view(torch.uint8), t["out2"].view(torch.uint8))


def test_w8_and_gather_write_only_their_buffers(abi):
    cfg = configs.MoEConfig("g_w8", N=90, D=208, F=336, E=6, k=2, dtype=configs.DTYPE_BF16,
                            activation=configs.ACT_SILU, renormalize=1)
    p = abi.problem(cfg)
    R = cfg.N * cfg.k
    counts = np.array([0, 40, 1, 77, 0, 62])
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    Xp = inputs.randn((R, cfg.D), 1.0, torch.bfloat16, "cuda", 3, 1)
    w = inputs.make_w8_weights(cfg, "cuda", 3)
    ws = _workspace(abi, p)
    H = Guarded((R, cfg.F), torch.bfloat16)
    Y = Guarded((R, cfg.D), torch.bfloat16)
    for kernel in ("smem", "tmem"):
        import os
        os.environ["MOE_W8_KERNEL"] = kernel
        try:
            abi.expert_up_w8(p, Xp, offsets, w.W1q, w.S1, w.W2q, w.S2, H.t, ws.t)
            abi.expert_down_w8(p, H.t, offsets, w.W3q, w.S3, Y.t, ws.t)
        finally:
            del os.environ["MOE_W8_KERNEL"]
        torch.cuda.synchronize()
        assert abi.device_error(ws.t) == 0
        assert H.intact() and Y.intact() and ws.intact(), kernel
    src = torch.randn((50, 24), device="cuda").to(torch.bfloat16)
    index = torch.randint(0, 50, (77,), device="cuda", dtype=torch.int32)
    dst = Guarded((77, 24), torch.bfloat16)
    abi.gather_rows(src, index, dst.t, ws.t)
    assert dst.intact() and ws.intact()
    assert torch.equal(dst.t, src[index.long()])
