"""Expert parallelism (experts split over ranks, rows exchanged by all-to-all; Grok-1 book 5.6,
MoE series 4.1) on CPU with gloo: the exchange plan and the two all-to-alls of ep.forward,
with the oracle as each rank's compute. Every rank must get exactly the oracle's single-device
layer on its own tokens (capacity per rank), whatever the world size and expert split."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from top_routing_expert_fp32_b200 import ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


# ---------------------------------------------------------------- plan (no process group)

def test_expert_ranges_cover_experts_in_order():
    for E in (1, 2, 7, 8, 64):
        for world in (1, 2, 3, 8):
            r = ep.expert_ranges(E, world)
            assert r[0][0] == 0 and r[-1][1] == E and len(r) == world
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [e1 - e0 for e0, e1 in r]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_plan_reorders_source_major_to_expert_major():
    # Rank 1 of 2 owns experts 2..3. Source 0 sends 2 rows of expert 2 and 1 of expert 3,
    # source 1 sends 0 of expert 2 and 3 of expert 3. Received buffer (source-major):
    #   [s0e2 s0e2 s0e3 | s1e3 s1e3 s1e3]; expert-major: [s0e2 s0e2 | s0e3 s1e3 s1e3 s1e3].
    ranges = ep.expert_ranges(4, 2)
    offsets = np.array([0, 5, 9, 9, 12])          # this rank's own dispatch
    plan = ep.plan_exchange(offsets, np.array([[2, 1], [0, 3]]), ranges)
    assert plan.send_rows == [9, 3]
    assert plan.recv_rows == [3, 3]
    assert plan.local_offsets.tolist() == [0, 2, 6]
    assert plan.to_expert_major.tolist() == [0, 1, 2, 3, 4, 5]
    plan = ep.plan_exchange(offsets, np.array([[1, 2], [3, 1]]), ranges)
    # received [s0e2 | s0e3 s0e3 | s1e2 s1e2 s1e2 | s1e3] -> [s0e2 s1e2*3 | s0e3*2 s1e3]
    assert plan.to_expert_major.tolist() == [0, 3, 4, 5, 1, 2, 6]
    inv = plan.to_source_major
    assert (inv[plan.to_expert_major] == np.arange(7)).all()


def test_a2a_bytes_formula():
    # 2 exchanges x N tokens x k slots x d_model x bytes per element (MoE series 4.1).
    assert ep.a2a_bytes(4096, 4096, 2, 2) == 2 * 4096 * 2 * 4096 * 2
    assert ep.a2a_bytes(0, 4096, 2, 2) == 0
    with pytest.raises(ValueError):
        ep.a2a_bytes(-1, 8, 1, 2)


# ---------------------------------------------------------------- layer over gloo ranks

class OracleCompute(ep.LocalCompute):
    """Each step of a rank's layer by the oracle (fp32 inputs, fp64 arithmetic)."""

    def __init__(self, W_r, bias, W1, W2, W3, k, cf, renorm, act, order=0, policy=0):
        import oracle
        self.o = oracle
        self.W_r, self.bias, self.W1, self.W2, self.W3 = W_r, bias, W1, W2, W3
        self.k, self.cf, self.renorm, self.act = k, cf, renorm, act
        self.order, self.policy = order, policy

    def route_dispatch(self, X):
        o = self.o
        N = X.shape[0]
        E = self.W_r.shape[1]
        _, l32 = o.router_logits(X, o.F32, self.W_r, self.bias)
        ro = o.route(l32, k=self.k, renorm=self.renorm)
        do = o.dispatch(ro["idx"], E, o.capacity(N, self.k, E, self.cf), order=self.order)
        X_perm = torch.from_numpy(np.ascontiguousarray(X[do["row_token"]], dtype=np.float32))
        return dict(offsets=torch.from_numpy(do["offsets"].astype(np.int32)), X_perm=X_perm,
                    idx=ro["idx"], gate=ro["gate"], pos=do["pos"], dropped=do["dropped"])

    def expert_ffn(self, X_loc, local_offsets, expert_range):
        e0, e1 = expert_range
        R = X_loc.shape[0]
        if R == 0:
            return torch.zeros((0, X_loc.shape[1]), dtype=torch.float64)
        rec_e = np.repeat(np.arange(e1 - e0, dtype=np.int32), np.diff(local_offsets))
        Y = self.o.expert_ffn(np.arange(R, dtype=np.int32), rec_e, X_loc.numpy(),
                              self.W1[e0:e1], self.W2[e0:e1], self.W3[e0:e1], self.o.F32,
                              self.act)
        return torch.from_numpy(Y)

    def gather_rows(self, src, index):
        return src[torch.from_numpy(index.astype(np.int64))].contiguous()

    def combine(self, Y_perm, r):
        N, k = r["idx"].shape
        Y = Y_perm.numpy()
        Yrec = np.zeros((N, k, Y.shape[1] if Y.ndim == 2 else 0))
        off = r["offsets"].numpy()
        for t in range(N):
            for j in range(k):
                if not r["dropped"][t, j]:
                    Yrec[t, j] = Y[off[r["idx"][t, j]] + r["pos"][t, j]]
        return torch.from_numpy(self.o.combine(r["gate"], r["dropped"], Yrec, self.policy))


def _weights(E, D, F, seed=5):
    g = np.random.default_rng(seed)
    return (g.standard_normal((D, E)).astype(np.float32) / np.sqrt(D),
            g.standard_normal(E).astype(np.float32),
            (g.standard_normal((E, D, F)) / np.sqrt(D)).astype(np.float32),
            (g.standard_normal((E, D, F)) / np.sqrt(D)).astype(np.float32),
            (g.standard_normal((E, F, D)) / np.sqrt(F)).astype(np.float32))


def _worker(rank, world, port, case, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        E, D, F, k, cf = case["E"], case["D"], case["F"], case["k"], case["cf"]
        W_r, bias, W1, W2, W3 = _weights(E, D, F)
        N = case["N"] + 7 * rank                        # ragged batches across ranks
        X = np.random.default_rng(100 + rank).standard_normal((N, D)).astype(np.float32)
        order, policy = case.get("order", 0), case.get("policy", 0)
        comp = OracleCompute(W_r, bias, W1, W2, W3, k, cf, 1, 0, order, policy)
        out, info = ep.forward(comp, X, E)
        ref = oracle.forward(X, W_r, bias, W1, W2, W3, k=k, cf=cf, renorm=1, act=0,
                             dtype=oracle.F32, order=order, drop_policy=policy)
        results[rank] = (float(np.abs(out.numpy() - ref["out"]).max()),
                         int(ref["dropped"].sum()), info["plan"].send_rows,
                         info["plan"].recv_rows)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, dict(E=8, D=32, F=48, k=2, N=40, cf=0.0)),
    (2, dict(E=8, D=32, F=48, k=2, N=40, cf=1.0)),
    (3, dict(E=8, D=16, F=32, k=2, N=33, cf=0.0)),     # expert blocks of 3, 3, 2
    (3, dict(E=4, D=16, F=32, k=1, N=25, cf=1.25)),    # blocks of 2, 1, 1
    (3, dict(E=2, D=16, F=32, k=2, N=20, cf=0.0)),     # rank 2 owns no expert
    # token-major capacity order and the case-A reweight of kept gates (MoE series 2.2)
    (2, dict(E=6, D=16, F=32, k=3, N=45, cf=0.8, order=1, policy=1)),
], ids=["w2", "w2_capacity", "w3_uneven", "w3_k1_capacity", "w3_more_ranks_than_experts",
        "w2_token_major_case_a"])
def test_ep_forward_equals_single_device_layer_gloo(world, case):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, case, results), nprocs=world, join=True,
                       start_method="spawn")
    assert len(results) == world
    for rank in range(world):
        err, ndrop, send, recv = results[rank]
        assert err == 0.0, f"rank {rank}: max abs diff {err}"
    # what rank a sends to rank b is what b receives from a
    for a in range(world):
        for b in range(world):
            assert results[a][2][b] == results[b][3][a]
    if case["cf"] > 0:
        assert sum(results[r][1] for r in range(world)) > 0   # the capacity case drops
