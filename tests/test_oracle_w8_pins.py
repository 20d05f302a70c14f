"""Pins for the oracle's 8-bit expert weights (CPU only). The Grok-1 book (ch.5, 5.3.3 and
5.3.5) dequantizes before each expert matmul, weight = weight * scales; the scales are read as
one value per expert and output column, broadcast over the reduction dimension. Checked against
the (separately pinned) bf16 path, a textbook dense gated FFN written with numpy, and exact
linearity in the scales."""
import numpy as np
import torch
from scipy.special import expit


def _q(rng, shape):
    return rng.integers(-127, 128, size=shape).astype(np.int8)


def _bf16_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def test_unit_scales_equal_bf16_weights(oracle_lib):
    # int8 values are exact in bf16, so q with all scales 1 is the bf16 expert on W = q.
    rng = np.random.default_rng(0)
    E, D, F, n = 3, 24, 40, 17
    W1q, W2q, W3q = _q(rng, (E, D, F)), _q(rng, (E, D, F)), _q(rng, (E, F, D))
    ones_f, ones_d = np.ones((E, F), np.float32), np.ones((E, D), np.float32)
    X = _bf16_bits(rng.standard_normal((n, D)) * 0.05)
    rt = rng.integers(0, n, size=n).astype(np.int32)
    re = rng.integers(0, E, size=n).astype(np.int32)
    y8 = oracle_lib.expert_ffn_w8(rt, re, X, oracle_lib.BF16, W1q, ones_f, W2q, ones_f, W3q,
                                  ones_d, oracle_lib.SILU)
    yb = oracle_lib.expert_ffn(rt, re, X, _bf16_bits(W1q), _bf16_bits(W2q), _bf16_bits(W3q),
                               oracle_lib.BF16, oracle_lib.SILU)
    assert np.array_equal(y8, yb)


def test_single_expert_textbook_gated_ffn_with_column_scales(oracle_lib):
    rng = np.random.default_rng(1)
    N, D, F = 9, 12, 20   # D != F: a scale applied along the wrong axis cannot pass
    X = rng.standard_normal((N, D)).astype(np.float32)
    W1q, W2q, W3q = _q(rng, (1, D, F)), _q(rng, (1, D, F)), _q(rng, (1, F, D))
    S1 = (rng.random((1, F)) * 0.02).astype(np.float32)
    S2 = (rng.random((1, F)) * 0.02).astype(np.float32)
    S3 = (rng.random((1, D)) * 0.02).astype(np.float32)
    W_r = np.zeros((D, 1), np.float32)
    o = oracle_lib.forward_w8(X, W_r, None, W1q, S1, W2q, S2, W3q, S3, k=1, cf=0.0, renorm=1,
                              act=oracle_lib.SILU, dtype=oracle_lib.F32)
    W1 = W1q[0].astype(np.float64) * S1[0].astype(np.float64)[None, :]
    W2 = W2q[0].astype(np.float64) * S2[0].astype(np.float64)[None, :]
    W3 = W3q[0].astype(np.float64) * S3[0].astype(np.float64)[None, :]
    a = X.astype(np.float64) @ W1
    ref = (a * expit(a) * (X.astype(np.float64) @ W2)) @ W3
    np.testing.assert_allclose(o["out"], ref, rtol=1e-11, atol=1e-13)


def test_output_is_linear_in_down_and_linear_branch_scales(oracle_lib):
    rng = np.random.default_rng(2)
    E, D, F, n = 2, 16, 24, 11
    W1q, W2q, W3q = _q(rng, (E, D, F)), _q(rng, (E, D, F)), _q(rng, (E, F, D))
    S1, S2 = (rng.random((E, F)) * 0.01).astype(np.float32), (rng.random((E, F)) * 0.01).astype(np.float32)
    S3 = (rng.random((E, D)) * 0.01).astype(np.float32)
    X = rng.standard_normal((n, D)).astype(np.float32)
    rt = np.arange(n, dtype=np.int32)
    re = (np.arange(n) % E).astype(np.int32)

    def y(s1, s2, s3):
        return oracle_lib.expert_ffn_w8(rt, re, X, oracle_lib.F32, W1q, s1, W2q, s2, W3q, s3,
                                        oracle_lib.GELU_ERF)

    base = y(S1, S2, S3)
    S3b = S3.copy()
    S3b[1, 5] *= 2.0            # expert 1, output column 5
    got = y(S1, S2, S3b)
    exp = base.copy()
    exp[re == 1, 5] *= 2.0
    assert np.array_equal(got, exp)
    assert np.array_equal(y(S1, 2.0 * S2, S3), 2.0 * base)
