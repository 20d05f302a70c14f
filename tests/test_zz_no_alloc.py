"""moe_dispatch_noalloc: the dispatch step for callers that cannot give the library device
memory (no cudaMalloc once they run, or all device memory owned by their own pool). Its
results must equal moe_dispatch's, call after call, with the counters kept in the library's
fixed array instead of a workspace, and a call after the first must leave the device's free
memory unchanged.

The file name sorts last so that pytest collects it after every other test file: a run that
stops at the first failure (-x) has then already run the rest of the suite when this one
fails. It also passes when run alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from top_routing_expert_fp32_b200 import configs, inputs


def _abi():
    from top_routing_expert_fp32_b200 import build
    build.build()
    from top_routing_expert_fp32_b200 import abi
    return abi


def _cfg(N, E, k, cf, D=64):
    return configs.MoEConfig("noalloc", N=N, D=D, F=64, E=E, k=k, dtype=configs.DTYPE_BF16,
                             activation=0, renormalize=1, capacity_factor=cf)


def test_noalloc_rejects_oversized_problems_on_host():
    abi = _abi()
    p = abi.problem(_cfg(300000, 64, 2, 1.25))   # ceil(600000/1024)*64 = 37504 > 16384
    st = abi.lib.moe_dispatch_noalloc(ctypes.byref(p), None, 8, 8, 8, 8, 8, 8, None, None)
    assert st == abi.MOE_ERR_UNSUPPORTED
    assert b"exceeds the fixed scratch" in abi.lib.moe_last_error()
    p = abi.problem(_cfg(64, 8, 2, 0.0))
    st = abi.lib.moe_dispatch_noalloc(ctypes.byref(p), None, 8, 8, 8, 8, 8, None, None, None)
    assert st == abi.MOE_ERR_INVALID_ARG   # row_token is required


def _run_both(abi, cfg, idx_np, X=None, check_free=False):
    N, E, k = cfg.N, cfg.E, cfg.k
    p = abi.problem(cfg)
    idx = torch.from_numpy(idx_np).cuda()

    def outputs():
        return dict(load=torch.full((E,), -1, dtype=torch.int32, device="cuda"),
                    offsets=torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
                    pos=torch.full((N, k), -1, dtype=torch.int32, device="cuda"),
                    dropped=torch.full((N, k), 7, dtype=torch.uint8, device="cuda"),
                    row_token=torch.full((N * k,), -1, dtype=torch.int32, device="cuda"),
                    X_perm=None if X is None else torch.zeros((N * k, X.shape[1]),
                                                              dtype=X.dtype, device="cuda"))

    ref, got = outputs(), outputs()
    ws = abi.workspace(p)
    abi.dispatch(p, X, idx, ref["load"], ref["offsets"], ref["pos"], ref["dropped"],
                 ref["row_token"], ref["X_perm"], ws)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    abi.dispatch_noalloc(p, X, idx, got["load"], got["offsets"], got["pos"], got["dropped"],
                         got["row_token"], got["X_perm"])
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    if check_free:  # the device's free memory (cudaMemGetInfo) is what an allocation would take
        assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    kept = int(ref["offsets"][E].item())
    for key in ("load", "offsets", "pos", "dropped"):
        assert torch.equal(ref[key], got[key]), key
    assert torch.equal(ref["row_token"][:kept], got["row_token"][:kept])
    if X is not None:
        assert torch.equal(ref["X_perm"][:kept].view(torch.int16),
                           got["X_perm"][:kept].view(torch.int16))
    return kept


@pytest.mark.gpu
def test_noalloc_dispatch_matches_workspace_dispatch_twice_in_a_row():
    abi = _abi()
    import oracle
    # First call: capacity stress shape with drops and the gather.
    cfg1 = _cfg(16384, 64, 2, 1.25, D=256)
    l1 = inputs.make_logits(cfg1.N, cfg1.E, seed=21).numpy() + \
        np.linspace(1.5, -1.5, cfg1.E, dtype=np.float32)
    idx1 = oracle.route(l1, k=cfg1.k, renorm=1)["idx"]
    X1 = inputs.randn((cfg1.N, cfg1.D), 1.0, torch.bfloat16, "cuda", 21, 1)
    kept1 = _run_both(abi, cfg1, idx1, X1)
    assert kept1 < cfg1.N * cfg1.k      # some records were dropped
    # Second call reuses the same fixed counters with a different, smaller problem.
    cfg2 = _cfg(3001, 8, 2, 0.0)
    idx2 = oracle.route(inputs.make_logits(cfg2.N, cfg2.E, seed=22).numpy(), k=2,
                        renorm=1)["idx"]
    kept2 = _run_both(abi, cfg2, idx2, check_free=True)
    assert kept2 == cfg2.N * cfg2.k
