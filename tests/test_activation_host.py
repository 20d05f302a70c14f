"""The exact-GELU coefficients in csrc/common.cuh on the CPU: they are the ones
csrc/gelu_coeffs.py fits, and the kernel's formula evaluated step by step in fp32 (numpy, exact
reciprocal and exponential in place of the approximate hardware ones) stays within the stated
relative error of float64 GELU (Grok-1 book 5.3.5: x * Phi(x))."""
import math
import os
import re
import sys

import numpy as np
from scipy.special import erfc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "top_routing_expert_fp32_b200", "csrc")
sys.path.insert(0, CSRC)
import gelu_coeffs  # noqa: E402


def _header_coefficients():
    with open(os.path.join(CSRC, "common.cuh")) as f:
        src = f.read()
    body = re.search(r"constexpr float kP\[10\] = \{([^}]*)\}", src).group(1)
    return np.array([float(v.strip().rstrip("f")) for v in body.split(",")], dtype=np.float32)


def test_header_holds_the_fitted_coefficients():
    assert np.array_equal(_header_coefficients(), gelu_coeffs.fit())


def test_fit_matches_erfc_at_the_ends():
    P = gelu_coeffs.fit().astype(np.float64)
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
