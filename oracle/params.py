"""Offline parameters of a TurboQuant context: rotation Pi, QJL matrix S, codebook.

Order of draws (one SplitMix64/Box-Muller stream per context seed): the d x d
Gaussian G first (row-major), then the m x d Gaussian S (row-major), m = d.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import special

from .rng import gaussian_stream

MODE_PROD = 0   # (b-1)-bit MSE codebook + 1-bit QJL sign sketch of the residual (keys)
MODE_MSE = 1    # b-bit MSE codebook only (values)


def haar_rotation(G: np.ndarray) -> np.ndarray:
    """Pi = Q from the QR factorisation of the Gaussian matrix G.

    [TQN] "生成随机旋转矩阵": ``Pi, _ = np.linalg.qr(G)`` with G ~ N(0,1)^{d x d};
    [ZX] "随机旋转与Beta分布" and [ADM] (PolarQuant paragraph): a random rotation.
    Reading: the pages leave QR's column signs open; we fix R_ii > 0, which makes
    the factorisation unique (so any correct QR gives the same Pi) and the
    distribution of Pi exactly Haar (Mezzadri, "How to generate random matrices
    from the classical compact groups", Notices AMS 2007).
    """
    Q, R = np.linalg.qr(G)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


def _log_cd(d: int) -> float:
    """log of the normalising constant Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return special.gammaln(d / 2.0) - special.gammaln((d - 1) / 2.0) - 0.5 * math.log(math.pi)


def beta_coordinate_density(x, d: int):
    """f_d(x) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2) on [-1, 1].

    [TQN] "PolarQuant：极坐标变换 — 坐标分布公式"; [ZX] "随机旋转与Beta分布";
    [ADM] PolarQuant paragraph (known Beta law, close to Gaussian in high d).
    It is the law of one coordinate of a uniformly random unit vector in R^d.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    inside = np.abs(x) < 1.0
    xi = x[inside]
    out[inside] = np.exp(_log_cd(d) + 0.5 * (d - 3) * np.log1p(-xi * xi))
    return out


def _upper_tail(x, d: int):
    """P(X > x) for x >= 0:  X^2 ~ Beta(1/2, (d-1)/2), so P(X > x) = I_{1-x^2}((d-1)/2, 1/2) / 2."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * special.betainc((d - 1) / 2.0, 0.5, np.clip(1.0 - x * x, 0.0, 1.0))


def beta_coordinate_cdf(x, d: int):
    """F_d(x) = P(X <= x) for the density above."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x <= 0.0, _upper_tail(-x, d), 1.0 - _upper_tail(x, d))


def _beta_mass(a: float, b: float, d: int) -> float:
    """P(a < X <= b), written so that tail intervals do not cancel."""
    if a >= 0.0:
        return float(_upper_tail(a, d) - _upper_tail(b, d))
    if b <= 0.0:
        return float(_upper_tail(-b, d) - _upper_tail(-a, d))
    return float(1.0 - _upper_tail(-a, d) - _upper_tail(b, d))


def _beta_first_moment(a: float, b: float, d: int) -> float:
    """int_a^b x f_d(x) dx in closed form:
    d/dx (1-x^2)^((d-1)/2) = -(d-1) x (1-x^2)^((d-3)/2), so the integral is
    C_d/(d-1) [ (1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2) ]."""
    def g(t):
        t = min(max(t, -1.0), 1.0)
        if abs(t) >= 1.0:
            return 0.0
        return math.exp(0.5 * (d - 1) * math.log1p(-t * t))
    return math.exp(_log_cd(d)) / (d - 1) * (g(a) - g(b))


def lloyd_max(mass, first_moment, levels: int, lo: float, hi: float, init_bounds,
              tol: float = 1e-15, max_iter: int = 200000):
    """Lloyd-Max optimal scalar quantizer (1-D continuous k-means) of a density.

    [TQN] "预计算 Lloyd-Max 质心" (computed once offline, reused); [ADM] PolarQuant
    paragraph (Lloyd-Max solves the continuous 1-D k-means problem per coordinate).
    Alternates the two optimality conditions until the centroids stop moving:
      boundaries t_j = (c_j + c_{j+1}) / 2,
      centroids  c_j = int_{t_{j-1}}^{t_j} x f / int_{t_{j-1}}^{t_j} f,  t_{-1}=lo, t_K=hi.
    Returns (centroids [levels], boundaries [levels-1]).
    """
    t = np.asarray(init_bounds, dtype=np.float64)
    edges = np.concatenate([[lo], t, [hi]])
    c = np.array([first_moment(edges[j], edges[j + 1]) / mass(edges[j], edges[j + 1])
                  for j in range(levels)])
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[lo], t, [hi]])
        c_new = np.array([first_moment(edges[j], edges[j + 1]) / mass(edges[j], edges[j + 1])
                          for j in range(levels)])
        delta = np.max(np.abs(c_new - c))
        c = c_new
        if delta <= tol:
            break
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


def lloyd_max_beta(d: int, levels: int):
    """Lloyd-Max codebook on the coordinate density f_d (d >= 3), started from
    equal-probability boundaries (the fixed point is unique for a log-concave density,
    Fleischer 1964, so the start only affects the iteration count)."""
    if d < 3:
        raise ValueError("the coordinate density needs d >= 3")
    probs = np.arange(1, levels) / levels
    init = np.array([_beta_quantile(p, d) for p in probs])
    c, _ = lloyd_max(lambda a, b: _beta_mass(a, b, d),
                     lambda a, b: _beta_first_moment(a, b, d),
                     levels, -1.0, 1.0, init)
    # f_d is even, so the exact quantizer is odd-symmetric; make the computed one exactly
    # so (the middle boundary is then exactly 0 and y = 0 sits on it, going to the lower cell)
    c = 0.5 * (c - c[::-1])
    return c, 0.5 * (c[:-1] + c[1:])


def _beta_quantile(p: float, d: int) -> float:
    if p == 0.5:
        return 0.0
    if p > 0.5:
        return -_beta_quantile(1.0 - p, d)
    # P(X <= -x) = p  <=>  I_{1-x^2}((d-1)/2, 1/2) = 2p
    w = special.betaincinv((d - 1) / 2.0, 0.5, 2.0 * p)
    return -math.sqrt(max(0.0, 1.0 - w))


def lloyd_max_gaussian(levels: int):
    """The same Lloyd-Max iteration on the standard normal density (the d -> infinity
    limit of sqrt(d) X, [TQN] "坐标分布公式 — 核心优势": near-Gaussian in high d)."""
    def mass(a, b):
        return float(special.ndtr(b) - special.ndtr(a)) if b <= 0 else float(special.ndtr(-a) - special.ndtr(-b))

    def first_moment(a, b):
        phi = lambda z: 0.0 if math.isinf(z) else math.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
        return phi(a) - phi(b)
    init = special.ndtri(np.arange(1, levels) / levels)
    return lloyd_max(mass, first_moment, levels, -math.inf, math.inf, init)


def make_params(d: int, bits: int, seed: int, mode: int = MODE_PROD) -> dict:
    """All offline parameters of a context (d, bits, seed, mode).

    prod (keys): k = bits - 1 MSE bits + 1 QJL bit per coordinate, m = d
    ([ADM] two-stage pipeline: PolarQuant at b-1 bits, then 1-bit QJL on the residual;
    [ZX] "两阶段内积量化").  MSE (values): k = bits.
    Returns Pi [d,d], S [m,d], centroids [2^k], boundaries [2^k - 1], k, m, mode, d.
    """
    if mode == MODE_PROD:
        k = bits - 1
    elif mode == MODE_MSE:
        k = bits
    else:
        raise ValueError("mode must be MODE_PROD or MODE_MSE")
    if k < 1:
        raise ValueError("need at least one MSE bit")
    m = d
    g = gaussian_stream(seed, d * d + m * d)
    G = g[: d * d].reshape(d, d)
    S = g[d * d:].reshape(m, d)
    Pi = haar_rotation(G)
    c, t = lloyd_max_beta(d, 2 ** k)
    return dict(d=d, bits=bits, k=k, m=m, mode=mode, seed=seed, Pi=Pi, S=S,
                centroids=c, boundaries=t)
