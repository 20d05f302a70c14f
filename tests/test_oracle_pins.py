"""Pins for the CPU oracle: each test checks it against something other than itself -- the
pages' worked example, closed forms, textbook special cases, library routines (numpy, scipy)
and brute force on tiny inputs -- chosen so a dropped term, a wrong sign or index, or a
transposed operand anywhere in the oracle fails at least one of them. CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from top_routing_expert_fp32_b200 import configs, inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _example():
    with open(os.path.join(GOLDEN, "gshard_top2_example.json")) as f:
        return json.load(f)


def _example_logits(ex):
    # Probabilities p are fed as logits ln(p): softmax(ln p) = p because sum(p) = 1.
    p = np.array([t["probs"] for t in ex["tokens"]], np.float64)
    return np.log(p).astype(np.float32)


# ------------------------------------------------------------------ worked example (GShard)

def test_worked_example_top2_and_gates(oracle_lib):
    ex = _example()
    l32 = _example_logits(ex)
    r = oracle_lib.route(l32, k=2, renorm=0)
    assert r["idx"].tolist() == [t["top2"] for t in ex["tokens"]]
    np.testing.assert_allclose(r["gate"][:2], ex["expected_gates_no_renorm_t0_t1"], rtol=1e-6)
    rr = oracle_lib.route(l32, k=2, renorm=1)
    assert rr["idx"].tolist() == [t["top2"] for t in ex["tokens"]]
    np.testing.assert_allclose(rr["gate"][:2], ex["expected_gates_renorm_t0_t1"], rtol=1e-6)
    np.testing.assert_allclose(rr["gate"].sum(1), 1.0, rtol=1e-12)


def test_worked_example_capacity(oracle_lib):
    ex = _example()
    assert oracle_lib.capacity(ex["S"], ex["k"], ex["E"], ex["capacity_factor"]) == \
        ex["expected_capacity"]


def test_worked_example_slot_major_dispatch(oracle_lib):
    ex = _example()
    idx = np.array([t["top2"] for t in ex["tokens"]], np.int32)
    d = oracle_lib.dispatch(idx, ex["E"], ex["expected_capacity"])
    exp = ex["slot_major_capacity_4"]
    assert d["load"].tolist() == exp["load"]
    assert d["offsets"].tolist() == exp["offsets"]
    assert d["pos"].tolist() == exp["pos"]
    assert d["dropped"].tolist() == exp["dropped"]
    assert d["row_token"].tolist() == exp["row_token"]
    assert d["dropped"].tolist() != ex["token_major_capacity_4_dropped_for_contrast"]
    assert oracle_lib.drop_rate(d["dropped"]) == pytest.approx(exp["drop_rate"], abs=0)


def test_worked_example_balance_loss(oracle_lib):
    ex = _example()
    l32 = _example_logits(ex)
    r = oracle_lib.route(l32, k=2, renorm=1)
    d = oracle_lib.dispatch(r["idx"], ex["E"], 10 ** 9)
    np.testing.assert_allclose(r["colsum"] / ex["S"], ex["mean_probs"], rtol=1e-6)
    L = oracle_lib.balance_loss(ex["S"], 2, d["load"], r["colsum"])
    assert L == pytest.approx(ex["balance_loss_nk_denominator"], rel=1e-6)


# ------------------------------------------------------------------ special cases

def test_uniform_logits_gate_sum_is_k_over_E(oracle_lib):
    # Grok-1 ch.5 5.2.3: with near-uniform routing the two gates sum to about 2/8 = 0.25.
    l32 = np.zeros((5, 8), np.float32)
    r = oracle_lib.route(l32, k=2, renorm=0)
    assert (r["idx"] == np.array([0, 1])).all()
    np.testing.assert_allclose(r["gate"], 1.0 / 8, rtol=1e-15)
    np.testing.assert_allclose(r["gate"].sum(1), 0.25, rtol=1e-15)
    rr = oracle_lib.route(l32, k=2, renorm=1)
    np.testing.assert_allclose(rr["gate"], 0.5, rtol=1e-15)


def test_k1_renormalised_gate_is_exactly_one(oracle_lib):
    # LLMs-from-scratch 12.4: a one-element softmax is identically 1.
    l32 = inputs.make_logits(257, 8, seed=3).numpy()
    r = oracle_lib.route(l32, k=1, renorm=1)
    assert (r["gate"] == 1.0).all()


def test_softmax_known_values_and_shift(oracle_lib):
    l32 = np.log(np.array([[1.0, 2.0, 3.0]])).astype(np.float32)
    r = oracle_lib.route(l32, k=3, renorm=0, want_probs=True)
    np.testing.assert_allclose(r["probs"][0], [1 / 6, 2 / 6, 3 / 6], rtol=1e-6)
    # Without subtracting the max, exp(1000) overflows; the stable form gives e/(2e+1).
    big = np.array([[1000.0, 1000.0, 999.0]], np.float32)
    r = oracle_lib.route(big, k=1, renorm=0, want_probs=True)
    e = math.e
    np.testing.assert_allclose(r["probs"][0], [e / (2 * e + 1), e / (2 * e + 1), 1 / (2 * e + 1)],
                               rtol=1e-14)
    assert r["idx"][0, 0] == 0


def test_tie_break_lowest_index(oracle_lib):
    l32 = np.array([[1, 3, 3, 2], [-0.0, 0.0, -1, -1], [5, 5, 5, 5]], np.float32)
    r = oracle_lib.route(l32, k=2, renorm=1)
    assert r["idx"].tolist() == [[1, 2], [0, 1], [0, 1]]
    l32 = np.zeros((1, 8), np.float32)
    assert oracle_lib.route(l32, k=3, renorm=0)["idx"].tolist() == [[0, 1, 2]]


def test_selection_matches_stable_library_sort(oracle_lib):
    # numpy's stable argsort of -logits is an independent order with the same tie rule.
    rng = np.random.default_rng(5)
    l32 = rng.integers(-3, 4, size=(500, 16)).astype(np.float32)  # many exact ties
    for k in (1, 2, 5, 16):
        r = oracle_lib.route(l32, k=k, renorm=1)
        ref = np.argsort(-l32, axis=1, kind="stable")[:, :k]
        assert (r["idx"] == ref).all()


def test_balance_loss_is_one_under_uniform_routing(oracle_lib):
    # Walkthrough 2.2 / Switch 7.3: f_i = P_i = 1/E gives exactly 1. With W_r = 0 every token
    # has P_i = 1/E, so the loss is sum_i f_i = 1 for ANY selection under f = load/(N*k).
    N, E, k = 96, 8, 2
    l32 = np.zeros((N, E), np.float32)
    r = oracle_lib.route(l32, k=k, renorm=0)
    rng = np.random.default_rng(0)
    for trial in range(3):
        idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
        d = oracle_lib.dispatch(idx, E, N * k)
        assert oracle_lib.balance_loss(N, k, d["load"], r["colsum"]) == pytest.approx(1.0, abs=1e-15)
        # The walkthrough's code divides f by N only: the same routing then gives k.
        assert oracle_lib.balance_loss(N, k, d["load"], r["colsum"], nk_denominator=False) == \
            pytest.approx(float(k), abs=1e-14)
    # Round-robin routing with skewed probabilities still gives f_i = 1/E -> loss = E*sum P_i/E = 1.
    l32 = inputs.make_logits(N, E, seed=1).numpy()
    r = oracle_lib.route(l32, k=k, renorm=0)
    idx = np.array([[(2 * t) % E, (2 * t + 1) % E] for t in range(N)], np.int32)
    d = oracle_lib.dispatch(idx, E, N * k)
    assert (d["load"] == N * k // E).all()
    assert oracle_lib.balance_loss(N, k, d["load"], r["colsum"]) == pytest.approx(1.0, abs=1e-12)


# ------------------------------------------------------------------ dispatch invariants

@pytest.mark.parametrize("N,E,k", [(1, 1, 1), (7, 3, 2), (64, 4, 2), (333, 8, 2), (200, 64, 2),
                                   (50, 5, 5), (129, 16, 1)])
def test_records_invariants_no_capacity(oracle_lib, N, E, k):
    # LLMs-from-scratch 12.2: N tokens with k dispatches each -> exactly N*k records;
    # walkthrough 1.3: the load counts every record once.
    l32 = inputs.make_logits(N, E, seed=N + E).numpy()
    r = oracle_lib.route(l32, k=k, renorm=1)
    d = oracle_lib.dispatch(r["idx"], E, oracle_lib.capacity(N, k, E, 0.0))
    assert d["load"].sum() == N * k
    assert d["offsets"][-1] == N * k and len(d["row_token"]) == N * k
    assert not d["dropped"].any()
    assert (np.bincount(d["row_token"], minlength=N) == k).all()
    assert (np.bincount(r["idx"].ravel(), minlength=E) == d["load"]).all()
    # row of each record lands in its expert's segment and holds its token
    rows = d["offsets"][r["idx"]] + d["pos"]
    assert (d["row_token"][rows] == np.arange(N)[:, None]).all()
    for e in range(E):
        seg = slice(d["offsets"][e], d["offsets"][e + 1])
        assert (r["idx"][np.isin(np.arange(N), d["row_token"][seg])] == e).any(1).all()


def test_capacity_formula_values(oracle_lib):
    # ceil(CF*N*K/E) (walkthrough 3.1); the capacity/drop configuration gives 640 and 320.
    assert oracle_lib.capacity(16384, 2, 64, 1.25) == 640
    assert oracle_lib.capacity(16384, 1, 64, 1.25) == 320
    assert oracle_lib.capacity(10, 2, 3, 1.0) == 7          # ceil(20/3)
    assert oracle_lib.capacity(10, 1, 4, 1.0) == 3          # ceil(2.5)
    assert oracle_lib.capacity(8, 2, 4, 1.0) == 4           # the GShard example
    assert oracle_lib.capacity(100, 2, 8, 0.0) == 200       # no capacity: every record fits
    assert oracle_lib.capacity(0, 2, 8, 1.25) == 0


def test_five_tokens_three_experts_capacity_one(oracle_lib):
    # LLMs-from-scratch 12.5: 5 tokens, 3 experts, top-2 -> 10 dispatches; with capacity 1 per
    # expert, 7 are over capacity (whenever all three experts are used).
    hit_all = 0
    for seed in range(40):
        l32 = inputs.make_logits(5, 3, seed=seed).numpy()
        r = oracle_lib.route(l32, k=2, renorm=1)
        d = oracle_lib.dispatch(r["idx"], 3, 1)
        assert d["pos"].size == 10
        used = len(np.unique(r["idx"]))
        assert int(d["dropped"].sum()) == 10 - used
        if used == 3:
            hit_all += 1
            assert int(d["dropped"].sum()) == 7
    assert hit_all > 0


@pytest.mark.parametrize("seed", range(12))
def test_slot_major_structure(oracle_lib, seed):
    """Properties that together determine slot-major-then-token assignment uniquely:
    positions of each expert are 0..load-1 once each; rank-j records of an expert get
    consecutive positions in token order; every rank-j record of an expert precedes (gets a
    smaller position than) every rank-(j+1) record of it. Hence kept rank-j records form a
    token-order prefix, and a rank-j record is kept only if all earlier-rank ones are."""
    rng = np.random.default_rng(seed)
    N, E = int(rng.integers(1, 40)), int(rng.integers(1, 7))
    k = int(rng.integers(1, E + 1))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    C = int(rng.integers(0, N * k // E + 3))
    d = oracle_lib.dispatch(idx, E, C)
    for e in range(E):
        recs = [(j, t) for j in range(k) for t in range(N) if idx[t, j] == e]
        ps = [int(d["pos"][t, j]) for (j, t) in recs]
        assert sorted(ps) == list(range(len(recs)))
        order = sorted(recs, key=lambda jt: d["pos"][jt[1], jt[0]])
        assert order == sorted(recs)           # (j, t) lexicographic: slot-major, then token
        for (j, t) in recs:
            assert d["dropped"][t, j] == (d["pos"][t, j] >= C)
    overflow = sum(max(0, int(l) - C) for l in d["load"])
    assert int(d["dropped"].sum()) == overflow


# ------------------------------------------------------------------ activations and experts

def _tiny_weights(E, D, F, seed):
    rng = np.random.default_rng(seed)
    W1 = (rng.standard_normal((E, D, F)) / np.sqrt(D)).astype(np.float32)
    W2 = (rng.standard_normal((E, D, F)) / np.sqrt(D)).astype(np.float32)
    W3 = (rng.standard_normal((E, F, D)) / np.sqrt(F)).astype(np.float32)
    return W1, W2, W3


def test_activation_tabulated_values(oracle_lib):
    # 1x1 expert: y = act(x*w1) * (x*w2) * w3 with x=1, w1=a, w2=3, w3=1. The activated branch
    # is W1 (Grok "linear", the GELU input) and W2 is the linear branch (Grok "linear_v").
    from scipy.special import expit
    from scipy.stats import norm
    X = np.ones((1, 1), np.float32)
    for a in (1.0, -1.0, 2.0, 0.5):
        W1 = np.full((1, 1, 1), a, np.float32)
        W2 = np.full((1, 1, 1), 3.0, np.float32)
        W3 = np.ones((1, 1, 1), np.float32)
        rec = (np.zeros(1, np.int32), np.zeros(1, np.int32))
        y_silu = oracle_lib.expert_ffn(*rec, X, W1, W2, W3, oracle_lib.F32, oracle_lib.SILU)
        y_gelu = oracle_lib.expert_ffn(*rec, X, W1, W2, W3, oracle_lib.F32, oracle_lib.GELU_ERF)
        y_tanh = oracle_lib.expert_ffn(*rec, X, W1, W2, W3, oracle_lib.F32,
                                       oracle_lib.GELU_TANH)
        assert y_silu[0, 0] == pytest.approx(3.0 * a * expit(a), rel=1e-14)
        assert y_gelu[0, 0] == pytest.approx(3.0 * a * norm.cdf(a), rel=1e-14)
        assert y_tanh[0, 0] == pytest.approx(y_gelu[0, 0], abs=3e-3)   # close approximation
    # Standard normal table: Phi(1) = 0.8413447, so GELU(1) = 0.8413447.
    W1 = np.ones((1, 1, 1), np.float32)
    y = oracle_lib.expert_ffn(np.zeros(1, np.int32), np.zeros(1, np.int32), X, W1,
                              np.ones((1, 1, 1), np.float32), np.ones((1, 1, 1), np.float32),
                              oracle_lib.F32, oracle_lib.GELU_ERF)
    assert y[0, 0] == pytest.approx(0.8413447460685429, abs=1e-12)


def test_single_expert_is_textbook_gated_ffn(oracle_lib):
    # E=1, k=1 reduces to one gated FFN: down(act(x W_gate) * (x W_up)) (Grok-1 ch.5 LlamaMLP),
    # evaluated here with numpy matmuls.
    from scipy.special import expit
    N, D, F = 9, 8, 16
    rng = np.random.default_rng(1)
    X = rng.standard_normal((N, D)).astype(np.float32)
    W1, W2, W3 = _tiny_weights(1, D, F, 2)
    W_r = rng.standard_normal((D, 1)).astype(np.float32)
    o = oracle_lib.forward(X, W_r, None, W1, W2, W3, k=1, cf=0.0, renorm=1,
                           act=oracle_lib.SILU, dtype=oracle_lib.F32)
    Xd = X.astype(np.float64)
    a = Xd @ W1[0].astype(np.float64)
    b = Xd @ W2[0].astype(np.float64)
    ref = (a * expit(a) * b) @ W3[0].astype(np.float64)
    np.testing.assert_allclose(o["out"], ref, rtol=1e-12, atol=1e-12)


def _numpy_dense_onehot_forward(X, W_r, bias, W1, W2, W3, k, renorm, act):
    """Grok-1-style dense evaluation written with numpy: every token through every expert
    (einsum), then a one-hot selection of each token's k experts, then the gate-weighted sum.
    Top-k via numpy's stable argsort of the negated fp32 logits."""
    from scipy.special import expit, erf
    Xd = X.astype(np.float64)
    l64 = Xd @ W_r.astype(np.float64) + (0 if bias is None else bias.astype(np.float64))
    l32 = l64.astype(np.float32)
    z = l32.astype(np.float64)
    p = np.exp(z - z.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    idx = np.argsort(-l32, axis=1, kind="stable")[:, :k]
    g = np.take_along_axis(p, idx, 1)
    if renorm:
        g = g / g.sum(1, keepdims=True)
    A = np.einsum("nd,edf->enf", Xd, W1.astype(np.float64))
    B = np.einsum("nd,edf->enf", Xd, W2.astype(np.float64))
    if act == 0:
        H = A * expit(A) * B
    else:
        H = 0.5 * A * (1 + erf(A / np.sqrt(2))) * B
    Yall = np.einsum("enf,efd->end", H, W3.astype(np.float64))   # [E, N, D]
    E = W_r.shape[1]
    onehot = np.zeros((k, E, X.shape[0]))
    for j in range(k):
        onehot[j, idx[:, j], np.arange(X.shape[0])] = 1.0
    sel = np.einsum("jen,end->jnd", onehot, Yall)                 # [k, N, D]
    return np.einsum("nj,jnd->nd", g, sel), idx, g


@pytest.mark.parametrize("k,renorm,act,bias", [(2, 1, 0, False), (2, 0, 1, False),
                                               (1, 1, 0, True), (3, 0, 0, True),
                                               (5, 1, 1, False)])
def test_forward_equals_dense_onehot(oracle_lib, k, renorm, act, bias):
    N, D, F, E = 23, 16, 24, 5
    rng = np.random.default_rng(10 + k)
    X = rng.standard_normal((N, D)).astype(np.float32)
    W_r = (rng.standard_normal((D, E)) / np.sqrt(D)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32) if bias else None
    W1, W2, W3 = _tiny_weights(E, D, F, 3 + k)
    o = oracle_lib.forward(X, W_r, b, W1, W2, W3, k=k, cf=0.0, renorm=renorm, act=act,
                           dtype=oracle_lib.F32)
    ref, idx, g = _numpy_dense_onehot_forward(X, W_r, b, W1, W2, W3, k, renorm, act)
    assert (o["idx"] == idx).all()
    np.testing.assert_allclose(o["gate"], g, rtol=1e-12)
    np.testing.assert_allclose(o["out"], ref, rtol=1e-10, atol=1e-12)


def test_all_experts_renormalised_is_dense_mixture(oracle_lib):
    # k = E with renormalisation: out = sum_e softmax(l)_e f_e(x), the dense mixture.
    N, D, F, E = 11, 8, 12, 4
    rng = np.random.default_rng(4)
    X = rng.standard_normal((N, D)).astype(np.float32)
    W_r = rng.standard_normal((D, E)).astype(np.float32)
    W1, W2, W3 = _tiny_weights(E, D, F, 9)
    o = oracle_lib.forward(X, W_r, None, W1, W2, W3, k=E, cf=0.0, renorm=1, act=0,
                           dtype=oracle_lib.F32)
    from scipy.special import softmax, expit
    Xd = X.astype(np.float64)
    p = softmax((Xd @ W_r.astype(np.float64)).astype(np.float32).astype(np.float64), axis=1)
    ref = np.zeros((N, D))
    for e in range(E):
        a = Xd @ W1[e].astype(np.float64)
        b = Xd @ W2[e].astype(np.float64)
        ref += p[:, e:e + 1] * ((a * expit(a) * b) @ W3[e].astype(np.float64))
    np.testing.assert_allclose(o["out"], ref, rtol=1e-10, atol=1e-12)


def test_capacity_drops_contribute_zero_bruteforce(oracle_lib):
    # With capacity: per-token brute force over the token's own kept experts (GShard 2.2:
    # a fully dropped token contributes 0) equals the dispatched forward.
    from scipy.special import expit
    N, D, F, E, k = 40, 8, 8, 4, 2
    rng = np.random.default_rng(7)
    X = rng.standard_normal((N, D)).astype(np.float32)
    W_r = rng.standard_normal((D, E)).astype(np.float32)
    bias = np.array([3.0, 0, 0, -3.0], np.float32)   # skew towards expert 0
    W1, W2, W3 = _tiny_weights(E, D, F, 8)
    cf = 0.75
    o = oracle_lib.forward(X, W_r, bias, W1, W2, W3, k=k, cf=cf, renorm=1, act=0,
                           dtype=oracle_lib.F32)
    C = oracle_lib.capacity(N, k, E, cf)
    assert o["dropped"].any() and (o["dropped"].all(1)).any()
    d = oracle_lib.dispatch(o["idx"], E, C)
    assert (d["dropped"] == o["dropped"]).all()
    ref = np.zeros((N, D))
    Xd = X.astype(np.float64)
    for t in range(N):
        for j in range(k):
            if o["dropped"][t, j]:
                continue
            e = o["idx"][t, j]
            a = Xd[t] @ W1[e].astype(np.float64)
            b = Xd[t] @ W2[e].astype(np.float64)
            ref[t] += o["gate"][t, j] * ((a * expit(a) * b) @ W3[e].astype(np.float64))
    np.testing.assert_allclose(o["out"], ref, rtol=1e-12, atol=1e-13)
    assert (o["out"][o["dropped"].all(1)] == 0).all()
    assert oracle_lib.drop_rate(o["dropped"]) == o["dropped"].sum() / (N * k)


def test_router_logits_match_library_matmul_bf16(oracle_lib):
    cfg = configs.MoEConfig("t", N=37, D=96, F=8, E=6, k=2, dtype=configs.DTYPE_BF16,
                            activation=0, renormalize=1, router_bias_var=2.0)
    inp = inputs.make_inputs(cfg, "cpu", seed=2, weights=False)
    Xn = oracle_lib.torch_to_numpy(inp.X)
    l64, l32 = oracle_lib.router_logits(Xn, oracle_lib.BF16, inp.W_r.numpy(), inp.bias.numpy())
    ref = inp.X.double().numpy() @ inp.W_r.double().numpy() + inp.bias.double().numpy()
    np.testing.assert_allclose(l64, ref, rtol=1e-12, atol=1e-12)
    assert (l32 == l64.astype(np.float32)).all()


def test_combine_matches_per_token_loop(oracle_lib):
    # LLMs-from-scratch 12.5: the gathered combine equals the per-token sum exactly.
    rng = np.random.default_rng(3)
    N, k, D = 13, 3, 7
    gate = rng.random((N, k))
    Y = rng.standard_normal((N, k, D))
    dropped = (rng.random((N, k)) < 0.3).astype(np.uint8)
    out = oracle_lib.combine(gate, dropped, Y)
    ref = np.zeros((N, D))
    for t in range(N):
        for j in range(k):
            if not dropped[t, j]:
                ref[t] += gate[t, j] * Y[t, j]
    assert np.array_equal(out, ref)


def test_topk_margin(oracle_lib):
    l = np.array([[3.0, 1.0, 2.0, 0.0], [1.0, 1.0, 1.0, 1.0], [5.0, 4.9, 0.0, 4.0]])
    m = oracle_lib.topk_margin(l, 2)
    np.testing.assert_allclose(m, [1.0, 0.0, 0.1], rtol=1e-12)
    m1 = oracle_lib.topk_margin(l, 1)
    np.testing.assert_allclose(m1, [1.0, 0.0, 0.1], rtol=1e-12)
    assert oracle_lib.topk_margin(np.ones((2, 1)), 1).tolist() == [math.inf, math.inf]


def test_nonfinite_logits_rejected(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.route(np.array([[1.0, np.nan]], np.float32), k=1, renorm=0)


def test_input_generator_recipe():
    """The generator draws N(0,1) X and N(0, 1/fan_in) weights, per-tensor seeded."""
    cfg = configs.CONFIGS["tiny_f32"]
    a = inputs.make_inputs(cfg, "cpu")
    b = inputs.make_inputs(cfg, "cpu")
    for x, y in zip((a.X, a.W_r, a.W1, a.W2, a.W3), (b.X, b.W_r, b.W1, b.W2, b.W3)):
        assert torch.equal(x, y)
    assert a.X.dtype == torch.float32 and a.W1.shape == (4, 64, 128) and a.W3.shape == (4, 128, 64)
    assert abs(a.W1.std().item() * math.sqrt(64) - 1) < 0.05
    assert abs(a.W3.std().item() * math.sqrt(128) - 1) < 0.05
    c = inputs.make_inputs(cfg.with_(dtype=configs.DTYPE_BF16, router_bias_var=2.0), "cpu")
    assert c.X.dtype == torch.bfloat16 and c.W_r.dtype == torch.float32 and c.bias.shape == (4,)
