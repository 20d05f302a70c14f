"""Failure detection on the GPU without a fault: a bounded device wait that runs out is
reported through the workspace's error word, and the context stays usable (no trap, no
unbounded spin)."""
import pytest
import torch

from top_routing_expert_fp32_b200 import configs, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import abi as a
    return a


def _forward(abi, cfg, inp, ws):
    out = torch.empty((cfg.N, cfg.D), dtype=torch.bfloat16, device="cuda")
    abi.forward(abi.problem(cfg), inp.X, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, out, ws)
    torch.cuda.synchronize()
    return out


def test_wait_timeout_is_reported_and_the_context_stays_usable(abi):
    cfg = configs.MoEConfig("fd", N=300, D=256, F=512, E=8, k=2, dtype=configs.DTYPE_BF16,
                            activation=configs.ACT_SILU, renormalize=1)
    inp = inputs.make_inputs(cfg, "cuda")
    ws = abi.workspace(abi.problem(cfg))
    before = _forward(abi, cfg, inp, ws)
    assert abi.device_error(ws) == 0
    # A wait on a barrier nothing completes, bounded at 50 ms of wall time.
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    abi.selftest_wait_timeout(ws, 50_000)
    e1.record()
    e1.synchronize()
    assert e0.elapsed_time(e1) >= 40.0          # the wait ran until its bound
    assert abi.device_error(ws) == abi.DEVERR_WAIT_TIMEOUT
    assert abi.device_error(ws) == 0            # reading the word cleared it
    after = _forward(abi, cfg, inp, ws)         # same stream, same context
    assert abi.device_error(ws) == 0
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
