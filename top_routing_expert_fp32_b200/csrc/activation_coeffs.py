"""Constants of the activations in common.cuh: the exact-GELU polynomial (``gelu_erf``) and
the reciprocal seed of SiLU (``silu``).

Exact GELU.

GELU(x) = x * Phi(x) with Phi(x) = erfc(-x / sqrt 2) / 2. The kernels evaluate the upper tail
q(x) = erfc(|x| / sqrt 2) / 2 and take Phi = q for x < 0 and 1 - q otherwise, so the negative
tail keeps its relative accuracy (1 + erf(x / sqrt 2) cancels there).

For z >= 0 the complementary error function is written as

    erfc(z) = t * exp(-z^2 + p(t)),    t = 1 / (1 + z / 2),

the form used by Press et al., Numerical Recipes, section 6.2 ("erfcc"): z in [0, inf) maps to
t in (0, 1], and p(t) = log(erfcx(z) / t) is smooth there, so one polynomial in t covers the
whole axis. The coefficients here are this script's own least-squares Chebyshev fit (degree 9,
600 Chebyshev nodes in t), converted to the power basis in t and rounded to fp32. They fold in
the base change for the hardware exponential and the halving:

    q = t * 2^(P(t) - x^2 * log2(e) / 2),   P(t) = log2(e) * p(t) - 1.

SiLU. a / (1 + e^-a) takes the reciprocal of y = 1 + e^-a on the FMA pipe: a first
approximation float(K - bits(y)) from y's bit pattern (subtracting the bits from a constant
negates the exponent and roughly inverts the mantissa), then three Newton steps
r <- r + r (1 - y r). K is chosen here to minimise the seed's largest relative error over two
binades (the error pattern repeats every two); the three steps then leave at most about one
ulp.

Run ``python activation_coeffs.py`` to print the constants, the error of the fp32 Horner
evaluation of P against float64 (as a relative error of q), and the seed's and the refined
reciprocal's errors.
"""
import numpy as np
import numpy.polynomial.chebyshev as cheb
from scipy.special import erfcx

DEGREE = 9
NODES = 600
T_SCALE = 2.0  # t = 1 / (1 + z / T_SCALE)


def z_of_t(t):
    return T_SCALE * (1.0 - t) / t


def target(t):
    """P(t) in float64: log2(erfcx(z) / t) - 1."""
    return np.log2(erfcx(z_of_t(t)) / t) - 1.0


def fit():
    k = np.arange(NODES)
    xs = np.cos(np.pi * (k + 0.5) / NODES)          # Chebyshev nodes of [-1, 1]
    t = np.clip((xs + 1.0) / 2.0, 1e-12, 1.0)
    c = cheb.chebfit(xs, target(t), DEGREE)
    power_in_xs = np.polynomial.Polynomial(cheb.cheb2poly(c))
    power_in_t = power_in_xs(np.polynomial.Polynomial([-1.0, 2.0]))   # xs = 2t - 1
    return power_in_t.coef.astype(np.float32)      # c[0] + c[1] t + ... + c[9] t^9


def horner_f32(coef, t):
    acc = np.full(t.shape, coef[-1], dtype=np.float32)
    for a in coef[-2::-1]:
        acc = (acc * t + a).astype(np.float32)
    return acc


def max_rel_error_of_q(coef):
    t = np.linspace(1e-7, 1.0, 1000001).astype(np.float32)
    err = horner_f32(coef, t).astype(np.float64) - target(t.astype(np.float64))
    return float(np.max(np.abs(err)) * np.log(2.0))


def seed_error(K, y):
    bits = y.astype(np.float32).view(np.int32).astype(np.int64)
    r0 = (np.int64(K) - bits).astype(np.int32).view(np.float32).astype(np.float64)
    return float(np.max(np.abs(r0 * y.astype(np.float32).astype(np.float64) - 1.0)))


def reciprocal_seed():
    """K minimising max |float(K - bits(y)) * y - 1| over y in [1, 4), coarse then fine."""
    y = np.linspace(1.0, 4.0, 200001)
    best = min(range(0x7EF00000, 0x7EF80000, 0x400), key=lambda K: seed_error(K, y))
    return min(range(best - 0x400, best + 0x400, 4), key=lambda K: seed_error(K, y))


def newton_reciprocal_f32(K, y):
    """The kernel's reciprocal of fp32 y in fp32: the seed and three Newton steps."""
    y = y.astype(np.float32)
    r = (np.int64(K) - y.view(np.int32).astype(np.int64)).astype(np.int32).view(np.float32)
    for _ in range(3):
        e = (np.float32(1.0) - y.astype(np.float64) * r.astype(np.float64)).astype(np.float32)
        r = (r.astype(np.float64) + r.astype(np.float64) * e.astype(np.float64)).astype(np.float32)
    return r


if __name__ == "__main__":
    coef = fit()
    print(f"// degree {DEGREE}, max relative error of q from P in fp32: "
          f"{max_rel_error_of_q(coef):.2e}")
    print("constexpr float kGeluP[%d] = {" % (DEGREE + 1))
    print("    " + ", ".join(f"{float(a):.9g}f" for a in coef) + "};")
    K = reciprocal_seed()
    y = np.concatenate([np.linspace(1.0, 2.0 ** 20, 400001), np.logspace(0, 37.9, 20001)])
    r = newton_reciprocal_f32(K, y).astype(np.float64)
    print(f"// reciprocal seed K = {K:#x}: seed error {seed_error(K, np.linspace(1, 4, 200001)):.4f}, "
          f"after three Newton steps {np.max(np.abs(r * y.astype(np.float32) - 1.0)):.2e}")
