"""Lloyd-Max codebook for the Lemma-1 coordinate law (fp64, CPU). Test infrastructure.

Follows the TurboQuant review (Jump2Paper, arXiv 2504.19874):
  * Lemma 1: a coordinate of a uniform point on S^{d-1} has density
        f_X(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2),  -1 <= x <= 1.
  * Theorem 1 (MSE) derivation: after the rotation the per-vector MSE splits into d
    copies of a 1-D continuous k-means problem on f_X, D_mse = d * C(f_X, b), and the
    codebook is found by Lloyd-Max iteration (the experiment setup table: codebooks for
    b = 1..8 are precomputed by Max-Lloyd numerical optimisation).
  * Intuition paragraph on the 1-bit case: each centroid is the probability-weighted
    mean of its cell.

Lloyd's two steps, in this order, until the centroids move less than `tol`:
  1. boundaries t_k = midpoints of neighbouring centroids;
  2. centroids c_i = E[X | t_{i-1} < X < t_i] under f_X.

Cell masses come from the Beta CDF (u = (x+1)/2 ~ Beta((d-1)/2, (d-1)/2), a change of
variable of Lemma 1) and the cell first moment from the antiderivative of x f_X(x),
which is -C_d (1-x^2)^((d-1)/2) / (d-1).
"""
from __future__ import annotations

import math

import numpy as np
from scipy import special

__all__ = [
    "norm_const",
    "f_X",
    "cdf",
    "first_moment",
    "second_moment",
    "lloyd_max",
    "cell_mse",
    "d_mse",
    "panter_dite_bound",
    "entropy_bits",
]


def norm_const(d: int) -> float:
    """C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)), the constant of Lemma 1."""
    return math.exp(math.lgamma(d / 2.0) - math.lgamma((d - 1) / 2.0)) / math.sqrt(math.pi)


def f_X(x, d: int):
    """Lemma-1 density of one coordinate of a uniform point on the unit sphere in R^d."""
    x = np.asarray(x, dtype=np.float64)
    return norm_const(d) * np.power(np.clip(1.0 - x * x, 0.0, None), (d - 3) / 2.0)


def cdf(x, d: int):
    """P(X <= x) for the Lemma-1 law: the Beta((d-1)/2,(d-1)/2) CDF at (x+1)/2."""
    a = (d - 1) / 2.0
    u = (np.clip(np.asarray(x, dtype=np.float64), -1.0, 1.0) + 1.0) / 2.0
    return special.betainc(a, a, u)


def first_moment(lo, hi, d: int):
    """Integral of x f_X(x) over [lo, hi] (closed-form antiderivative)."""
    c = norm_const(d)
    p = (d - 1) / 2.0

    def G(x):
        return -c * np.power(np.clip(1.0 - np.asarray(x, np.float64) ** 2, 0.0, None), p) / (d - 1)

    return G(hi) - G(lo)


def second_moment(lo, hi, d: int):
    """Integral of x^2 f_X(x) over [lo, hi].

    Uses x^2 = 1 - (1 - x^2) and C_d (1-x^2)^((d-1)/2) = ((d-1)/d) f_{X,d+2}(x).
    """
    return (cdf(hi, d) - cdf(lo, d)) - (d - 1) / d * (cdf(hi, d + 2) - cdf(lo, d + 2))


def _cells(bounds):
    edges = np.concatenate(([-1.0], np.asarray(bounds, np.float64), [1.0]))
    return edges[:-1], edges[1:]


def lloyd_max(d: int, b: int, tol: float = 1e-14, max_iter: int = 1_000_000):
    """Lloyd-Max quantizer of f_X with 2^b levels.

    Returns (centroids[2^b] ascending, boundaries[2^b - 1], D_mse = d * C(f_X, b), iterations).
    Starts from the conditional means of 2^b equal-probability cells.
    """
    if d < 2 or b < 0:
        raise ValueError("need d >= 2 and b >= 0")
    L = 1 << b
    if L == 1:
        return np.zeros(1), np.zeros(0), d_mse(d, np.zeros(1), np.zeros(0)), 0
    a = (d - 1) / 2.0
    q = special.betaincinv(a, a, np.arange(1, L) / L) * 2.0 - 1.0
    lo, hi = _cells(q)
    c = first_moment(lo, hi, d) / (cdf(hi, d) - cdf(lo, d))
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])                               # step 1: midpoints
        lo, hi = _cells(t)
        c_new = first_moment(lo, hi, d) / (cdf(hi, d) - cdf(lo, d))  # step 2: cell means
        moved = np.max(np.abs(c_new - c))
        c = c_new
        if moved < tol:
            break
    # f_X is even, so the optimal codebook is antisymmetric; rounding noise is removed
    # so that 0 is exactly a boundary (a zero coordinate goes to the upper cell).
    c = 0.5 * (c - c[::-1])
    t = 0.5 * (c[:-1] + c[1:])
    return c, t, d_mse(d, c, t), it


def cell_mse(d: int, centroids, bounds):
    """Per-cell integral of (x - c_i)^2 f_X(x)."""
    lo, hi = _cells(bounds)
    c = np.asarray(centroids, np.float64)
    m0 = cdf(hi, d) - cdf(lo, d)
    m1 = first_moment(lo, hi, d)
    m2 = second_moment(lo, hi, d)
    return m2 - 2.0 * c * m1 + c * c * m0


def d_mse(d: int, centroids, bounds) -> float:
    """D_mse = d * C(f_X, b) for the given codebook (Theorem 1 derivation)."""
    return float(d * np.sum(cell_mse(d, centroids, bounds)))


def panter_dite_bound(d: int, b: int) -> float:
    """d * (1/12) (integral of f_X^{1/3})^3 4^{-b}: the high-resolution bound of Theorem 1."""
    from scipy import integrate
    val, _ = integrate.quad(lambda x: f_X(x, d) ** (1.0 / 3.0), -1.0, 1.0,
                            epsabs=0.0, epsrel=1e-12, limit=500)
    return d * val ** 3 / 12.0 * 4.0 ** (-b)


def entropy_bits(d: int, bounds) -> float:
    """Shannon entropy (bits) of the code index under f_X (limitations paragraph, b = 4)."""
    lo, hi = _cells(bounds)
    p = cdf(hi, d) - cdf(lo, d)
    p = p[p > 0]
    return float(-np.sum(p * np.log2(p)))
