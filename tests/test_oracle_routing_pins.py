"""Pins for the oracle's training-time routing variants and z-loss (CPU only): noisy top-k
(Grok-1 book ch.5, 5.2.2), GShard random routing of the second expert (MoE series, 3) and the
z-loss (log Z)^2 (Grok-1 book ch.5, 5.2.2). Checked against values worked out by hand on the
pages' example, closed forms and invariants."""
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ex():
    with open(os.path.join(GOLDEN, "gshard_top2_example.json")) as f:
        return json.load(f)


def _tok0_logits(ex):
    return np.log(np.array([ex["tokens"][0]["probs"]], np.float64)).astype(np.float32)


def test_worked_example_gshard_random_second_expert(oracle_lib):
    ex = _ex()
    v = ex["routing_variants_token0"]
    r = oracle_lib.route_ex(_tok0_logits(ex), k=2, renorm=1, mode=oracle_lib.ROUTE_GSHARD_RANDOM,
                            noise=np.array([v["gshard_noise"]], np.float32))
    assert r["idx"][0].tolist() == v["gshard_top2"]
    np.testing.assert_allclose(r["gate"][0], v["gshard_gates_renorm"], rtol=1e-6)


def test_worked_example_noisy_topk(oracle_lib):
    ex = _ex()
    v = ex["routing_variants_token0"]
    r = oracle_lib.route_ex(_tok0_logits(ex), k=2, renorm=1, mode=oracle_lib.ROUTE_NOISY_TOPK,
                            noise=np.array([v["noisy_noise"]], np.float32))
    assert r["idx"][0].tolist() == v["noisy_top2"]
    np.testing.assert_allclose(r["gate"][0], v["noisy_gates_renorm"], rtol=1e-6)


def test_zero_noise_reduces_to_plain_topk(oracle_lib):
    rng = np.random.default_rng(0)
    l = rng.standard_normal((200, 8)).astype(np.float32)
    base = oracle_lib.route(l, k=3, renorm=0)
    for mode in (oracle_lib.ROUTE_NOISY_TOPK, oracle_lib.ROUTE_GSHARD_RANDOM):
        r = oracle_lib.route_ex(l, k=3, renorm=0, mode=mode, noise=np.zeros_like(l))
        assert np.array_equal(r["idx"], base["idx"])
        assert np.array_equal(r["gate"], base["gate"])
        assert np.array_equal(r["colsum"], base["colsum"])


def test_gshard_first_expert_ignores_noise_and_gates_use_clean_probs(oracle_lib):
    rng = np.random.default_rng(1)
    l = rng.standard_normal((300, 16)).astype(np.float32)
    n = (3.0 * rng.standard_normal((300, 16))).astype(np.float32)
    r = oracle_lib.route_ex(l, k=2, renorm=0, mode=oracle_lib.ROUTE_GSHARD_RANDOM, noise=n,
                            want_probs=True)
    assert np.array_equal(r["idx"][:, 0], np.argmax(l, axis=1))
    p = np.exp(l.astype(np.float64) - l.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(r["gate"], np.take_along_axis(p, r["idx"], 1), rtol=1e-12)
    # the second expert is the largest perturbed logit once the first is masked
    zn = (l + n).astype(np.float32)
    np.put_along_axis(zn, r["idx"][:, :1], -np.inf, 1)
    assert np.array_equal(r["idx"][:, 1], np.argmax(zn, axis=1))


def test_noisy_topk_constant_noise_changes_nothing_but_rounding(oracle_lib):
    rng = np.random.default_rng(2)
    l = rng.standard_normal((100, 8)).astype(np.float32)
    base = oracle_lib.route(l, k=2, renorm=1)
    r = oracle_lib.route_ex(l, k=2, renorm=1, mode=oracle_lib.ROUTE_NOISY_TOPK,
                            noise=np.full_like(l, 0.75))
    assert np.array_equal(r["idx"], base["idx"])
    np.testing.assert_allclose(r["gate"], base["gate"], rtol=1e-6)


def test_zloss_closed_forms(oracle_lib):
    ex = _ex()
    l = np.log(np.array([t["probs"] for t in ex["tokens"]], np.float64)).astype(np.float32)
    assert oracle_lib.route_ex(l, k=2, renorm=1)["zloss"] == pytest.approx(0.0, abs=1e-12)
    E, c = 8, 1.3
    u = np.full((5, E), c, np.float32)   # log Z = c + ln E for uniform logits
    assert oracle_lib.route_ex(u, k=2, renorm=1)["zloss"] == pytest.approx(
        (np.float32(c) + math.log(E)) ** 2, rel=1e-12)
    one = np.array([[2.0], [-3.0]], np.float32)   # E = 1: log Z = z
    assert oracle_lib.route_ex(one, k=1, renorm=1)["zloss"] == pytest.approx((4.0 + 9.0) / 2)
