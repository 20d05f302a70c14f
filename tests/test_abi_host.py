"""CPU tests of the C ABI: the library builds and loads without a GPU, exports every symbol
include/moe.h declares, and its host-side logic (capacity, workspace sizing, argument checks)
behaves as documented. No compute call is made here."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    from top_routing_expert_fp32_b200 import build
    build.build()
    from top_routing_expert_fp32_b200 import abi as a
    return a


def _header_functions():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported(abi):
    declared = _header_functions()
    assert set(declared) == set(abi.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s(moe_[a-z0-9_]+)$", out, flags=re.M))
    missing = set(declared) - exported
    assert not missing, f"declared but not exported: {missing}"
    for name in declared:
        assert hasattr(abi.lib, name)


def test_library_built_for_sm100a(abi):
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", abi.LIB_PATH],
                         capture_output=True, text=True)
    assert out.returncode == 0 and "sm_100a" in out.stdout


def test_version_and_status_strings(abi):
    assert abi.lib.moe_version() >= 110
    assert abi.lib.moe_status_string(0) == b"ok"
    assert abi.lib.moe_status_string(3) == b"CUDA error"


@pytest.mark.parametrize("N,k,E,cf", [(16384, 2, 64, 1.25), (16384, 1, 64, 1.25), (8, 2, 4, 1.0),
                                      (10, 2, 3, 1.0), (100, 2, 8, 0.0), (0, 2, 8, 1.25),
                                      (7, 3, 5, 0.3), (4096, 2, 8, -1.0)])
def test_capacity_matches_oracle(abi, oracle_lib, N, k, E, cf):
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("c", N=N, D=64, F=64, E=E, k=k, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1, capacity_factor=cf)
    assert abi.capacity(abi.problem(cfg)) == oracle_lib.capacity(N, k, E, cf)


@pytest.mark.parametrize("N,k,E,cf,minc", [(8, 2, 4, 0.5, 3), (8, 2, 4, 1.0, 3), (16384, 2, 64, 1.0, 256),
                                           (100, 2, 8, 0.0, 1000), (5, 2, 3, 0.3, 2)])
def test_capacity_with_floor_matches_oracle(abi, oracle_lib, N, k, E, cf, minc):
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("c", N=N, D=64, F=64, E=E, k=k, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1, capacity_factor=cf, min_capacity=minc)
    assert abi.capacity(abi.problem(cfg)) == oracle_lib.capacity(N, k, E, cf, minc)


def test_problem_struct_matches_header_layout(abi, tmp_path):
    # The ctypes mirror must have the C header's size and field offsets (gcc, host only).
    import subprocess
    fields = [f for f, _ in abi.moe_problem._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe.h"\nint main(void) {\n'
                   '  printf("%zu", sizeof(moe_problem));\n' +
                   "".join(f'  printf(" %zu", offsetof(moe_problem, {f}));\n' for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    assert got[0] == ctypes.sizeof(abi.moe_problem)
    assert got[1:] == [getattr(abi.moe_problem, f).offset for f in fields]


def test_workspace_size_covers_intermediates(abi):
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.CONFIGS["mixtral"]
    p = abi.problem(cfg)
    n = abi.workspace_size(p)
    R = cfg.N * cfg.k
    assert n >= 2 * R * (2 * cfg.D + cfg.F)  # X_perm, H, Y in bf16
    assert abi.workspace_size(p, host=True) >= n + 2 * 2 * cfg.N * cfg.D
    p0 = abi.problem(cfg, N=0)
    assert abi.workspace_size(p0) >= 256


def test_workspace_size_covers_the_router_operand(abi):
    # bf16 X with more than 16 experts: the router writes the three bf16 terms of W_r, rows
    # 3 Ep rounded up to 16 by D, into the workspace once per call; 16 experts or fewer (and
    # fp32 X) need no such region.
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.CONFIGS["capacity"]
    D, E = cfg.D, cfg.E
    nb = -(-3 * (-(-E // 8) * 8) // 16) * 16
    with64 = abi.workspace_size(abi.problem(cfg))
    def variant(name, E_, dtype):
        return configs.MoEConfig(name, N=cfg.N, D=D, F=cfg.F, E=E_, k=cfg.k, dtype=dtype,
                                 activation=cfg.activation, renormalize=cfg.renormalize,
                                 capacity_factor=cfg.capacity_factor)
    cfg16 = variant("e16", 16, configs.DTYPE_BF16)
    cfg17 = variant("e17", 17, configs.DTYPE_BF16)
    n16 = abi.workspace_size(abi.problem(cfg16))
    n17 = abi.workspace_size(abi.problem(cfg17))
    assert n17 - n16 >= (-(-3 * 24 // 16) * 16) * D * 2      # E = 17: Ep = 24, 80 rows
    assert with64 >= nb * D * 2 + 2 * cfg.N * cfg.k * (2 * D + cfg.F)
    n32 = abi.workspace_size(abi.problem(variant("f32", 64, configs.DTYPE_F32)))
    assert n32 >= 4 * cfg.N * cfg.k * (2 * D + cfg.F)   # fp32 intermediates, no operand


def _call_route(abi, p, ws=None, ws_bytes=0, X=None, W_r=None, logits=None, idx=8, gate=8):
    return abi.lib.moe_route(ctypes.byref(p), X, W_r, None, logits, idx, gate, None, ws,
                             ws_bytes, None)


@pytest.mark.parametrize("field,value,status", [
    ("k", 0, 1), ("k", 9, 1), ("E", 65, 2), ("N", -1, 1), ("D", 0, 1), ("dtype", 7, 1),
    ("activation", 3, 1), ("renormalize", 2, 1), ("reserved", 1, 1), ("D", 12, 2),
    ("capacity_factor", float("nan"), 1), ("capacity_order", 2, 1), ("drop_policy", -1, 1),
    ("min_capacity", -5, 1)])
def test_invalid_problems_rejected_on_host(abi, field, value, status):
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("c", N=64, D=64, F=64, E=8, k=2, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1)
    p = abi.problem(cfg)
    setattr(p, field, value)
    b = ctypes.c_size_t()
    assert abi.lib.moe_workspace_size(ctypes.byref(p), ctypes.byref(b)) == status
    assert len(abi.lib.moe_last_error()) > 0


def test_k9_with_large_E_is_unsupported(abi):
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("c", N=64, D=64, F=64, E=16, k=9, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1)
    b = ctypes.c_size_t()
    assert abi.lib.moe_workspace_size(ctypes.byref(abi.problem(cfg)), ctypes.byref(b)) == 2


def test_null_and_misaligned_pointers_rejected(abi):
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("c", N=64, D=64, F=64, E=8, k=2, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1)
    p = abi.problem(cfg)
    need = abi.workspace_size(p)
    # No workspace.
    assert _call_route(abi, p, X=4096, W_r=4096) == abi.MOE_ERR_INVALID_ARG
    # Workspace too small.
    assert _call_route(abi, p, ws=4096, ws_bytes=need - 1, X=4096, W_r=4096) == \
        abi.MOE_ERR_INVALID_ARG
    assert b"too small" in abi.lib.moe_last_error()
    # Misaligned X.
    assert _call_route(abi, p, ws=4096, ws_bytes=need, X=4100, W_r=4096) == \
        abi.MOE_ERR_INVALID_ARG
    assert b"aligned" in abi.lib.moe_last_error()
    # Routing from logits needs the logits pointer.
    assert _call_route(abi, p, ws=4096, ws_bytes=need) == abi.MOE_ERR_INVALID_ARG
    # Dispatch: X without X_perm.
    st = abi.lib.moe_dispatch(ctypes.byref(p), 4096, 4096, 4096, 4096, 4096, 4096, None, None,
                              4096, need, None)
    assert st == abi.MOE_ERR_INVALID_ARG
    # Forward: missing weights.
    st = abi.lib.moe_forward(ctypes.byref(p), 4096, 4096, None, None, 4096, 4096, 4096,
                             *([None] * 8), 4096, need, None)
    assert st == abi.MOE_ERR_INVALID_ARG and b"W1" in abi.lib.moe_last_error()


def test_w8_entry_points_reject_unsupported_shapes_on_host(abi):
    # 8-bit expert weights need bf16 activations and D, F multiples of 16; the check runs on
    # the host before anything is enqueued.
    from top_routing_expert_fp32_b200 import configs
    for dtype, D in ((configs.DTYPE_F32, 64), (configs.DTYPE_BF16, 24)):
        cfg = configs.MoEConfig("w8", N=8, D=D, F=64, E=4, k=1, dtype=dtype, activation=0,
                                renormalize=1)
        p = abi.problem(cfg)
        st = abi.lib.moe_expert_up_w8(ctypes.byref(p), 16, 16, 16, 16, 16, 16, 16, 256, 1 << 20,
                                      None)
        assert st == 2, abi.lib.moe_last_error()
        st = abi.lib.moe_forward_w8(ctypes.byref(p), *([16] * 10), *([None] * 8), 256, 1 << 20,
                                    None)
        assert st == 2


def test_routing_mode_checks_on_host(abi):
    # Unknown modes are invalid; the entry points without a noise argument take plain top-k
    # only; moe_route_ex needs the noise for the noisy modes.
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("r", N=8, D=64, F=64, E=4, k=2, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1)
    p = abi.problem(cfg)
    b = ctypes.c_size_t()
    p.routing_mode = 3
    assert abi.lib.moe_workspace_size(ctypes.byref(p), ctypes.byref(b)) == 1
    p.routing_mode = configs.ROUTE_GSHARD_RANDOM
    assert abi.lib.moe_workspace_size(ctypes.byref(p), ctypes.byref(b)) == 0
    ws_bytes = b.value
    st = abi.lib.moe_route(ctypes.byref(p), 16, 16, None, None, 16, 16, None, 256, ws_bytes, None)
    assert st == 1 and b"noise" in abi.lib.moe_last_error()
    st = abi.lib.moe_route_ex(ctypes.byref(p), 16, 16, None, None, None, 16, 16, None, None, 256,
                              ws_bytes, None)
    assert st == 1 and b"noise" in abi.lib.moe_last_error()


def test_streamed_host_entry_and_gather_reject_bad_arguments_on_host(abi):
    # Checked before anything is enqueued (no GPU needed).
    from top_routing_expert_fp32_b200 import configs
    cfg = configs.MoEConfig("h", N=64, D=64, F=64, E=8, k=2, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1)
    p = abi.problem(cfg)
    b = ctypes.c_size_t()
    assert abi.lib.moe_workspace_size_host(ctypes.byref(p), ctypes.byref(b)) == 0
    need_h = b.value
    # the host workspace holds the layer's plus four N x D activation buffers
    assert need_h >= abi.workspace_size(p) + 4 * 64 * 64 * 2
    fwd = lambda nb, ws_bytes, x=4096: abi.lib.moe_forward_host_many(
        ctypes.byref(p), nb, x, 4096, None, 4096, 4096, 4096, 4096, 4096, ws_bytes, None)
    assert fwd(-1, need_h) == abi.MOE_ERR_INVALID_ARG
    assert fwd(2, need_h - 1) == abi.MOE_ERR_INVALID_ARG          # workspace too small
    assert fwd(2, need_h, x=None) == abi.MOE_ERR_INVALID_ARG      # no host X
    assert b"X_host" in abi.lib.moe_last_error()
    g = abi.lib.moe_gather_rows
    assert g(4096, 10, 4096, 5, 6, 4096, 4096, 256, None) == abi.MOE_ERR_INVALID_ARG  # 6 % 4
    assert g(4096, 10, 4096, -1, 8, 4096, 4096, 256, None) == abi.MOE_ERR_INVALID_ARG
    assert g(4096, 10, 4096, 5, 8, 4096, 4096, 128, None) == abi.MOE_ERR_INVALID_ARG  # small ws
    assert g(4096, 10, None, 5, 8, 4096, 4096, 256, None) == abi.MOE_ERR_INVALID_ARG  # no index
    assert g(4096, 10, 4096, 5, 8, 4100, 4096, 256, None) == abi.MOE_ERR_INVALID_ARG  # dst align


def test_selftest_wait_timeout_rejects_bad_arguments_on_host(abi):
    st = abi.lib.moe_selftest_wait_timeout
    assert st(None, 256, 1000, None) == abi.MOE_ERR_INVALID_ARG
    assert st(4096, 128, 1000, None) == abi.MOE_ERR_INVALID_ARG      # workspace too small
    assert st(4096, 256, 0, None) == abi.MOE_ERR_INVALID_ARG         # timeout out of range
    assert st(4096, 256, 10**8, None) == abi.MOE_ERR_INVALID_ARG


def test_diagnostics_host_functions_match_the_oracle(abi, oracle_lib):
    # Host-only entry points (no device work): balance loss E * sum f_e P_e and drop rate.
    from top_routing_expert_fp32_b200 import configs
    rng = np.random.default_rng(7)
    for N, E, k in ((64, 4, 2), (1000, 64, 2), (333, 13, 5), (5, 8, 1)):
        cfg = configs.MoEConfig("d", N=N, D=64, F=64, E=E, k=k, dtype=configs.DTYPE_BF16,
                                activation=0, renormalize=1)
        p = abi.problem(cfg)
        load = rng.multinomial(N * k, rng.dirichlet(np.ones(E))).astype(np.int32)
        colsum = (rng.dirichlet(np.ones(E)) * N).astype(np.float32)
        got = abi.balance_loss(p, torch.from_numpy(load), torch.from_numpy(colsum))
        want = oracle_lib.balance_loss(N, k, load, colsum.astype(np.float64))
        assert got == pytest.approx(want, rel=1e-12, abs=0)
        # uniform routing: exactly 1 whatever k ([W] 2.2)
        if (N * k) % E == 0 and N % E == 0:
            u = abi.balance_loss(p, torch.full((E,), N * k // E, dtype=torch.int32),
                                 torch.full((E,), N / E, dtype=torch.float32))
            assert u == pytest.approx(1.0, rel=1e-12)
        dropped = (rng.random((N, k)) < 0.3).astype(np.uint8)
        assert abi.drop_rate(p, torch.from_numpy(dropped)) == pytest.approx(
            oracle_lib.drop_rate(dropped), rel=0, abs=0)
    cfg0 = configs.MoEConfig("d0", N=0, D=64, F=64, E=4, k=2, dtype=configs.DTYPE_BF16,
                             activation=0, renormalize=1)
    p0 = abi.problem(cfg0)
    z = torch.zeros(4, dtype=torch.int32)
    assert abi.balance_loss(p0, z, z.float()) == 0.0
    assert abi.drop_rate(p0, torch.zeros((0, 2), dtype=torch.uint8)) == 0.0
    out = ctypes.c_double()
    assert abi.lib.moe_balance_loss(ctypes.byref(p0), None, 16, ctypes.byref(out)) == \
        abi.MOE_ERR_INVALID_ARG


def test_combine_needs_the_drop_flags_under_a_capacity(abi):
    # With a capacity some records are dropped and only `dropped` says which; without it the
    # kernel would take every position as a row of Y. Rejected on the host; accepted (still
    # nothing enqueued here: N = 0) without a capacity.
    from top_routing_expert_fp32_b200 import configs
    for cf, want in ((1.25, abi.MOE_ERR_INVALID_ARG), (0.0, abi.MOE_OK)):
        cfg = configs.MoEConfig("c", N=0, D=64, F=64, E=8, k=2, dtype=configs.DTYPE_BF16,
                                activation=0, renormalize=1, capacity_factor=cf)
        p = abi.problem(cfg)
        st = abi.lib.moe_combine(ctypes.byref(p), 4096, 4096, 4096, 4096, 4096, None, 4096, None)
        assert st == want, abi.lib.moe_last_error()
        if want != abi.MOE_OK:
            assert b"dropped" in abi.lib.moe_last_error()
