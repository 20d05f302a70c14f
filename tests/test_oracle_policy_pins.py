"""Pins for the oracle's capacity policies (CPU only): token-major slot order (the dispatch
loop of the MoE formula-to-code walkthrough, 3.2), GShard's case-A reweight of a token's kept
slots and the min_capacity floor (MoE series, 2.1-2.2). Each is checked against values worked
out by hand on the pages' 8-token example, closed forms, or brute force on tiny inputs."""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _example():
    with open(os.path.join(GOLDEN, "gshard_top2_example.json")) as f:
        return json.load(f)


def _idx(ex):
    return np.array([t["top2"] for t in ex["tokens"]], np.int32)


def test_worked_example_token_major_dispatch(oracle_lib):
    ex = _example()
    d = oracle_lib.dispatch(_idx(ex), ex["E"], ex["expected_capacity"],
                            order=oracle_lib.TOKEN_MAJOR)
    exp = ex["token_major_capacity_4"]
    assert d["load"].tolist() == exp["load"]
    assert d["offsets"].tolist() == exp["offsets"]
    assert d["pos"].tolist() == exp["pos"]
    assert d["dropped"].tolist() == exp["dropped"]
    assert d["dropped"].tolist() == ex["token_major_capacity_4_dropped_for_contrast"]
    assert d["row_token"].tolist() == exp["row_token"]
    assert oracle_lib.drop_rate(d["dropped"]) == pytest.approx(exp["drop_rate"], abs=0)


@pytest.mark.parametrize("order", ["slot_major", "token_major"])
def test_worked_example_case_a_reweight(oracle_lib, order):
    # Effective combine weights = combine of one-hot expert outputs: Y[t, j] = e_j.
    ex = _example()
    l32 = np.log(np.array([t["probs"] for t in ex["tokens"]], np.float64)).astype(np.float32)
    r = oracle_lib.route(l32, k=2, renorm=1)
    o = oracle_lib.TOKEN_MAJOR if order == "token_major" else oracle_lib.SLOT_MAJOR
    d = oracle_lib.dispatch(r["idx"], ex["E"], ex["expected_capacity"], order=o)
    Y = np.zeros((8, 2, 2))
    Y[:, 0, 0] = 1.0
    Y[:, 1, 1] = 1.0
    w_zero = oracle_lib.combine(r["gate"], d["dropped"], Y, policy=oracle_lib.DROP_ZERO)
    w_case_a = oracle_lib.combine(r["gate"], d["dropped"], Y, policy=oracle_lib.DROP_RENORM_KEPT)
    changed = {int(t): v for t, v in ex["case_a_reweight"][order + "_weights_changed"].items()}
    for t in range(8):
        if t in changed:
            assert w_case_a[t].tolist() == changed[t]
        else:   # no slot dropped: both policies keep the gates as they are
            assert (d["dropped"][t] == 0).all()
            assert w_case_a[t].tolist() == r["gate"][t].tolist() == w_zero[t].tolist()
    # Case B (every slot dropped) contributes nothing under both policies.
    assert w_zero[7].tolist() == [0.0, 0.0]


def test_min_capacity_values(oracle_lib):
    for c in _example()["min_capacity"]["cases"]:
        assert oracle_lib.capacity(c["S"], c["K"], c["E"], c["capacity_factor"],
                                   c["min_capacity"]) == c["capacity"]
    # No capacity (CF <= 0) keeps every record whatever the floor.
    assert oracle_lib.capacity(8, 2, 4, 0.0, 100) == 16


def test_single_slot_orders_coincide(oracle_lib):
    # k = 1: slot-major and token-major visit the records in the same order.
    rng = np.random.default_rng(4)
    idx = rng.integers(0, 5, size=(200, 1)).astype(np.int32)
    a = oracle_lib.dispatch(idx, 5, 30, order=oracle_lib.SLOT_MAJOR)
    b = oracle_lib.dispatch(idx, 5, 30, order=oracle_lib.TOKEN_MAJOR)
    for key in ("load", "offsets", "pos", "dropped", "row_token"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_token_major_bruteforce(oracle_lib, seed):
    # Brute force: a record's position is the number of records before it in token-major
    # order (earlier tokens, or the same token's lower slots) that chose the same expert.
    rng = np.random.default_rng(seed)
    N, E, k, C = 23, 5, 3, 6
    idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    d = oracle_lib.dispatch(idx, E, C, order=oracle_lib.TOKEN_MAJOR)
    flat = idx.reshape(-1)
    for r in range(N * k):
        p = int((flat[:r] == flat[r]).sum())
        assert d["pos"].reshape(-1)[r] == p
        assert d["dropped"].reshape(-1)[r] == (p >= C)
    kept = np.minimum(np.bincount(flat, minlength=E), C)
    assert d["offsets"].tolist() == [0] + np.cumsum(kept).tolist()


def test_case_a_bruteforce_forward(oracle_lib):
    # The whole forward under (token-major, case-A reweight, min_capacity) equals a per-token
    # brute force over the kept experts with the kept gates renormalised.
    from scipy.special import expit
    N, D, F, E, k = 30, 6, 5, 4, 2
    rng = np.random.default_rng(9)
    X = rng.standard_normal((N, D)).astype(np.float32)
    W_r = rng.standard_normal((D, E)).astype(np.float32)
    bias = np.array([2.5, 0.5, 0, -2.0], np.float32)
    W1 = rng.standard_normal((E, D, F)).astype(np.float32)
    W2 = rng.standard_normal((E, D, F)).astype(np.float32)
    W3 = rng.standard_normal((E, F, D)).astype(np.float32)
    cf, minc = 0.5, 9
    o = oracle_lib.forward(X, W_r, bias, W1, W2, W3, k=k, cf=cf, renorm=0, act=0,
                           dtype=oracle_lib.F32, min_capacity=minc,
                           order=oracle_lib.TOKEN_MAJOR, drop_policy=oracle_lib.DROP_RENORM_KEPT)
    C = oracle_lib.capacity(N, k, E, cf, minc)
    assert C == 9   # ceil(0.5 * 30 * 2 / 4) = 8 < 9
    d = oracle_lib.dispatch(o["idx"], E, C, order=oracle_lib.TOKEN_MAJOR)
    assert np.array_equal(d["dropped"], o["dropped"])
    partial = (o["dropped"].any(1)) & ~(o["dropped"].all(1))
    assert partial.any()
    Xd = X.astype(np.float64)
    ref = np.zeros((N, D))
    for t in range(N):
        keep = [j for j in range(k) if not o["dropped"][t, j]]
        s = sum(o["gate"][t, j] for j in keep)
        for j in keep:
            e = o["idx"][t, j]
            a = Xd[t] @ W1[e].astype(np.float64)
            b = Xd[t] @ W2[e].astype(np.float64)
            g = o["gate"][t, j] / s if len(keep) < k else o["gate"][t, j]
            ref[t] += g * ((a * expit(a) * b) @ W3[e].astype(np.float64))
    np.testing.assert_allclose(o["out"], ref, rtol=1e-12, atol=1e-12)
