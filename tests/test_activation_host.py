"""The activation constants in csrc/common.cuh on the CPU: they are the ones
csrc/activation_coeffs.py fits, and the kernels' formulas evaluated step by step in fp32 (numpy,
exact exponentials in place of the approximate hardware ones) stay within the stated relative
errors of float64 GELU (Grok-1 book 5.3.5: x * Phi(x)) and SiLU (LLMs-from-scratch 12.1)."""
import math
import os
import re
import sys

import numpy as np
from scipy.special import erfc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "top_routing_expert_fp32_b200", "csrc")
sys.path.insert(0, CSRC)
import activation_coeffs  # noqa: E402


def _header_coefficients():
    with open(os.path.join(CSRC, "common.cuh")) as f:
        src = f.read()
    body = re.search(r"constexpr float kP\[10\] = \{([^}]*)\}", src).group(1)
    return np.array([float(v.strip().rstrip("f")) for v in body.split(",")], dtype=np.float32)


def test_header_holds_the_fitted_coefficients():
    assert np.array_equal(_header_coefficients(), activation_coeffs.fit())


def test_fit_matches_erfc_at_the_ends():
    P = activation_coeffs.fit().astype(np.float64)
    # t = 1 (x = 0): q = erfc(0) / 2 = 1/2, so P(1) = -1
    assert abs(P.sum() + 1.0) < 1e-6
    # t -> 0 (x -> inf): erfcx(z) t^-1 -> 1 / (2 sqrt(pi)), so P(0) = log2(1 / (2 sqrt pi)) - 1
    assert abs(P[0] - (math.log2(1.0 / (2.0 * math.sqrt(math.pi))) - 1.0)) < 1e-5


def test_kernel_formula_in_fp32_against_float64():
    f32 = np.float32
    c = _header_coefficients()
    x = np.concatenate([np.linspace(-11.0, 11.0, 400001),
                        -np.logspace(-30, 1, 2001), np.logspace(-30, 1, 2001)]).astype(f32)
    t = (f32(1.0) / (np.abs(x) * f32(0.353553390593273762) + f32(1.0)).astype(f32)).astype(f32)
    P = np.full(t.shape, c[9], dtype=f32)
    for i in range(8, -1, -1):
        P = (P * t + c[i]).astype(f32)
    arg = ((x * x).astype(f32) * f32(-0.721347520444481703) + P).astype(f32)
    q = (t * np.exp2(arg.astype(np.float64)).astype(f32)).astype(f32)
    g = (x * np.where(x < 0, q, (f32(1.0) - q).astype(f32))).astype(f32).astype(np.float64)
    x64 = x.astype(np.float64)
    ref = x64 * 0.5 * erfc(-x64 / math.sqrt(2.0))
    keep = np.abs(ref) >= 1e-30
    rel = np.abs(g[keep] - ref[keep]) / np.abs(ref[keep])
    xs = x64[keep]
    assert rel[np.abs(xs) < 1.0].max() < 6e-7
    assert rel[(xs >= -5.0) & (xs <= -1.0)].max() < 2e-6
    assert rel.max() < 1e-5
    # the form 0.5 x (1 + erf(x / sqrt 2)) in the same precision cancels: zero below -5.7
    from scipy.special import erf
    naive = f32(0.5) * x * (f32(1.0) + erf(x * f32(0.70710678)).astype(f32))
    assert (naive[x < -6.0] == 0).all() and (g[x < -6.0] < 0).all()


def _silu_seed_from_header():
    with open(os.path.join(CSRC, "common.cuh")) as f:
        src = f.read()
    return int(re.search(r"__int_as_float\((0x[0-9A-Fa-f]+) - __float_as_int\(y\)\)", src).group(1),
               16)


def test_silu_seed_is_the_fitted_one_and_the_reciprocal_converges():
    K = _silu_seed_from_header()
    assert K == activation_coeffs.reciprocal_seed()
    assert activation_coeffs.seed_error(K, np.linspace(1.0, 4.0, 20001)) < 0.052
    y = np.concatenate([np.linspace(1.0, 1e6, 200001), np.logspace(0, 37.9, 5001)])
    r = activation_coeffs.newton_reciprocal_f32(K, y).astype(np.float64)
    assert np.max(np.abs(r * y.astype(np.float32) - 1.0)) < 1.2e-7     # about one ulp


def test_silu_formula_in_fp32_against_float64():
    f32 = np.float32
    K = _silu_seed_from_header()
    x = np.concatenate([np.linspace(-14.0, 14.0, 200001),
                        -np.logspace(-20, 1, 1001), np.logspace(-20, 1, 1001)]).astype(f32)
    arg = np.minimum((x * f32(-1.44269504088896341)).astype(f32), f32(126.0))
    y = (f32(1.0) + np.exp2(arg.astype(np.float64)).astype(f32)).astype(f32)
    r = activation_coeffs.newton_reciprocal_f32(K, y)
    got = (x * r).astype(f32).astype(np.float64)
    x64 = x.astype(np.float64)
    ref = x64 / (1.0 + np.exp(-x64))
    keep = np.abs(ref) >= 1e-30
    rel = np.abs(got[keep] - ref[keep]) / np.abs(ref[keep])
    xs = x64[keep]
    assert rel[np.abs(xs) <= 5.0].max() < 4e-7
    assert rel.max() < 1e-6          # the rounding of x log2(e) grows with |x|
