"""Pins of the float64 oracle against facts fixed outside it: published test vectors,
textbook tables, closed forms, independent algorithms, brute force and Monte Carlo."""
import math
import os

import numpy as np
import pytest
from scipy import integrate, special, stats

import oracle
from oracle.params import (MODE_MSE, MODE_PROD, beta_coordinate_cdf, beta_coordinate_density,
                           haar_rotation, lloyd_max_beta, lloyd_max_gaussian, make_params)
from oracle.quantize import nearest_index

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- RNG
def test_splitmix64_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "splitmix64_seed0.txt"))
            if l.strip() and not l.startswith("#")]
    got = oracle.splitmix64(0, len(rows))
    for (i, hexval) in rows:
        assert int(got[int(i)]) == int(hexval, 16)


def test_splitmix64_is_counter_based():
    full = oracle.splitmix64(42, 100)
    assert np.array_equal(full[37:61], oracle.splitmix64(42, 24, start=37))


def test_uniform_is_in_half_open_unit_interval():
    u = oracle.uniform01(np.array([0, 2 ** 64 - 1, 2 ** 11 - 1, 2 ** 11], dtype=np.uint64))
    assert u[0] == 2.0 ** -53 and u[1] == 1.0
    assert u[2] == 2.0 ** -53 and u[3] == 2.0 * 2.0 ** -53


def test_gaussian_stream_is_standard_normal():
    g = oracle.gaussian_stream(7, 200001)
    assert len(g) == 200001
    assert abs(g.mean()) < 4.0 / math.sqrt(len(g))
    assert abs(g.var() - 1.0) < 4.0 * math.sqrt(2.0 / len(g))
    assert stats.kstest(g, "norm").pvalue > 1e-4
    # the odd (sine) and even (cosine) draws of Box-Muller are uncorrelated
    assert abs(np.corrcoef(g[0:-1:2], g[1::2])[0, 1]) < 4.0 / math.sqrt(len(g) / 2)


# ------------------------------------------------------------------------ rotation
@pytest.mark.parametrize("d", [16, 64, 128, 200, 1536])
def test_rotation_is_orthogonal(d):
    p = make_params(d, 2, 1000 + d, MODE_MSE) if d != 1536 else None
    if p is None:
        g = oracle.gaussian_stream(5, d * d).reshape(d, d)
        Pi = haar_rotation(g)
    else:
        Pi = p["Pi"]
    err = np.abs(Pi @ Pi.T - np.eye(d)).max()
    assert err <= 1e-12


def _modified_gram_schmidt(G):
    Q = np.array(G, dtype=np.float64, copy=True)
    d = Q.shape[1]
    for j in range(d):
        for i in range(j):
            Q[:, j] -= (Q[:, i] @ Q[:, j]) * Q[:, i]
        Q[:, j] /= np.linalg.norm(Q[:, j])
    return Q


@pytest.mark.parametrize("d", [4, 16, 64])
def test_rotation_equals_gram_schmidt(d):
    """Gram-Schmidt on the columns of G gives the QR factor with R_ii > 0, so it must
    reproduce Pi: pins the sign convention and that Pi = Q (not Q^T)."""
    g = oracle.gaussian_stream(11, d * d).reshape(d, d)
    Pi = haar_rotation(g)
    assert np.abs(Pi - _modified_gram_schmidt(g)).max() < 1e-10
    R = Pi.T @ g
    assert np.abs(np.tril(R, -1)).max() < 1e-10
    assert np.all(np.diag(R) > 0)


def test_params_draw_order():
    """G then S from one stream, both row-major."""
    d = 8
    p = make_params(d, 3, 99, MODE_PROD)
    g = oracle.gaussian_stream(99, 2 * d * d)
    assert np.array_equal(p["S"], g[d * d:].reshape(d, d))
    assert np.abs(p["Pi"] - haar_rotation(g[:d * d].reshape(d, d))).max() == 0.0


# ------------------------------------------------------------------------- density
@pytest.mark.parametrize("d", [3, 4, 16, 128, 1536])
def test_density_integrates_to_one_and_second_moment(d):
    f = lambda x: float(beta_coordinate_density(np.array([x]), d)[0])
    s = 1.0 / math.sqrt(d)
    pts = [-10 * s, -3 * s, 0.0, 3 * s, 10 * s] if d > 50 else None
    total = integrate.quad(f, -1, 1, points=pts, limit=200, epsabs=1e-14, epsrel=1e-13)[0]
    m2 = integrate.quad(lambda x: x * x * f(x), -1, 1, points=pts, limit=200,
                        epsabs=1e-14, epsrel=1e-13)[0]
    assert abs(total - 1.0) < 1e-10
    assert abs(m2 - 1.0 / d) < 1e-10 / d   # E[X^2] = 1/d for a coordinate of a unit vector


def test_density_d3_is_uniform():
    x = np.linspace(-0.99, 0.99, 11)
    assert np.allclose(beta_coordinate_density(x, 3), 0.5, atol=1e-15)


@pytest.mark.parametrize("d", [3, 16, 128])
def test_cdf_is_integral_of_density(d):
    for x in [-0.7, -0.2, -0.01, 0.0, 0.05, 0.3, 0.9]:
        ref = integrate.quad(lambda t: float(beta_coordinate_density(np.array([t]), d)[0]),
                             -1, x, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
        assert abs(float(beta_coordinate_cdf(x, d)) - ref) < 1e-11


@pytest.mark.parametrize("d", [16, 128])
def test_density_matches_rotated_random_unit_vectors(d):
    rng = np.random.Generator(np.random.PCG64(2024))
    g = rng.standard_normal((100000 // d + 1, d))
    Pi = haar_rotation(rng.standard_normal((d, d)))
    u = (g / np.linalg.norm(g, axis=1, keepdims=True)) @ Pi.T
    coords = u.ravel()[:100000]
    assert stats.kstest(coords, lambda x: beta_coordinate_cdf(x, d)).pvalue > 1e-4


# ------------------------------------------------------------------------ codebook
@pytest.mark.parametrize("levels", [2, 4, 8, 16])
def test_codebook_d3_is_uniform_quantizer(levels):
    """f_3 is uniform on [-1, 1]: the Lloyd-Max quantizer is the uniform one."""
    c, t = lloyd_max_beta(3, levels)
    j = np.arange(levels)
    assert np.abs(c - (-1.0 + (2 * j + 1) / levels)).max() < 1e-12
    assert np.abs(t - (-1.0 + 2.0 * np.arange(1, levels) / levels)).max() < 1e-12


@pytest.mark.parametrize("d", [3, 5, 16, 64, 128, 1536])
def test_codebook_one_bit_closed_form(d):
    """K = 2: c = +-E|X| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))."""
    c, t = lloyd_max_beta(d, 2)
    e = math.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    assert abs(c[1] - e) < 1e-13 and abs(c[0] + e) < 1e-13 and abs(t[0]) < 1e-15


@pytest.mark.parametrize("d,levels", [(16, 8), (64, 4), (64, 8), (128, 8), (128, 16), (1536, 8)])
def test_codebook_fixed_point_under_gauss_legendre(d, levels):
    """Each centroid is the conditional mean of its cell, checked with an independent
    Gauss-Legendre rule on the density (not the incomplete-beta route used to fit it)."""
    c, t = lloyd_max_beta(d, levels)
    edges = np.concatenate([[-1.0], t, [1.0]])
    xg, wg = np.polynomial.legendre.leggauss(200)
    s = 12.0 / math.sqrt(d)
    for j in range(levels):
        a, b = max(edges[j], -min(1.0, s)), min(edges[j + 1], min(1.0, s))
        # split the cell into pieces so the rule resolves the density
        cuts = np.linspace(a, b, 9)
        num = den = 0.0
        for lo, hi in zip(cuts[:-1], cuts[1:]):
            x = 0.5 * (hi - lo) * xg + 0.5 * (hi + lo)
            w = 0.5 * (hi - lo) * wg
            f = beta_coordinate_density(x, d)
            num += np.sum(w * x * f)
            den += np.sum(w * f)
        assert abs(num / den - c[j]) < 1e-12
    assert np.abs(t - 0.5 * (c[:-1] + c[1:])).max() == 0.0


@pytest.mark.parametrize("d,levels", [(16, 4), (128, 8), (128, 16), (1536, 8)])
def test_codebook_symmetric_and_sorted(d, levels):
    c, t = lloyd_max_beta(d, levels)
    assert np.all(np.diff(c) > 0)
    assert np.abs(c + c[::-1]).max() == 0.0
    assert t[levels // 2 - 1] == 0.0


def _max1960():
    table = {}
    for line in open(os.path.join(GOLDEN, "max1960_gaussian_lloyd_max.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        parts = line.split()
        vals = np.array([float(v) for v in parts[2:]])
        # 1.5 units in the last printed digit: the 1960 table carries up to about one unit
        # of computational error there (its 2-level output 0.7980 vs sqrt(2/pi) = 0.79788)
        tol = np.array([1.5 * 10.0 ** -len(v.split(".")[1]) for v in parts[2:]])
        table[(int(parts[0]), parts[1])] = (vals, tol)
    return table


@pytest.mark.parametrize("levels", [2, 4, 8, 16])
def test_gaussian_lloyd_max_matches_max_1960(levels):
    tab = _max1960()
    c, t = lloyd_max_gaussian(levels)
    if levels == 2:
        assert abs(c[1] - math.sqrt(2.0 / math.pi)) < 1e-14   # E|Z| in closed form
    vals, tol = tab[(levels, "output")]
    assert np.all(np.abs(c[levels // 2:] - vals) <= tol)
    if levels > 2:
        vals, tol = tab[(levels, "threshold")]
        assert np.all(np.abs(t[levels // 2:] - vals) <= tol)
    # distortion of the fitted quantizer, by quadrature
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    mse = sum(integrate.quad(lambda x: (x - c[j]) ** 2 * math.exp(-x * x / 2) / math.sqrt(2 * math.pi),
                             edges[j], edges[j + 1])[0] for j in range(levels))
    # the distortion column is checked to 0.1 %: at 16 levels the 1960 entry (0.009497)
    # sits 0.04 % below the distortion of its own printed levels (0.0095010)
    vals, _ = tab[(levels, "mse")]
    assert abs(mse - vals[0]) <= 1e-3 * vals[0]


@pytest.mark.parametrize("levels", [4, 8, 16])
def test_codebook_tends_to_gaussian_levels(levels):
    """sqrt(d) X -> N(0,1) as d grows, so sqrt(d) c_d -> the Gaussian levels, O(1/d)."""
    cg, _ = lloyd_max_gaussian(levels)
    errs = []
    for d in (64, 128, 1536):
        c, _ = lloyd_max_beta(d, levels)
        errs.append(np.abs(math.sqrt(d) * c - cg).max())
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 0.01
    assert 1.5 < errs[0] / errs[1] < 2.5     # halving 1/d roughly halves the gap


def test_mse_distortion_monte_carlo():
    """E||u - Pi^T c[idx]||^2 over random unit vectors equals d * int (x - Q(x))^2 f."""
    d, levels = 64, 8
    p = make_params(d, 3, 5, MODE_MSE)
    c, t = p["centroids"], p["boundaries"]
    edges = np.concatenate([[-1.0], t, [1.0]])
    f = lambda x: float(beta_coordinate_density(np.array([x]), d)[0])
    per_coord = sum(integrate.quad(lambda x: (x - c[j]) ** 2 * f(x), edges[j], edges[j + 1],
                                   epsabs=1e-15)[0] for j in range(levels))
    rng = np.random.Generator(np.random.PCG64(3))
    x = rng.standard_normal((20000, d))
    out = oracle.quantize(p, x)
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    err = np.sum((u - c[out["idx"]] @ p["Pi"]) ** 2, axis=1)
    assert abs(err.mean() - d * per_coord) < 3.0 * err.std() / math.sqrt(len(err))


# ---------------------------------------------------------------------- quantizer
def test_nearest_index_equals_brute_force_argmin():
    rng = np.random.Generator(np.random.PCG64(8))
    for d in (4, 8, 16):
        c, t = lloyd_max_beta(d, 8)
        y = np.concatenate([rng.uniform(-1, 1, 2000),
                            t[None, :].repeat(50, 0).ravel() + rng.uniform(-1e-9, 1e-9, 50 * len(t)),
                            c])
        idx = nearest_index(y, t)
        dist = np.abs(y[:, None] - c[None, :])
        best = np.argmin(dist, axis=1)
        assert np.array_equal(idx, best)
        # a value exactly on a boundary goes to the lower of its two neighbours
        assert np.array_equal(nearest_index(t, t), np.arange(len(t)))


def _hand_params():
    """d = 3 with Pi a permutation (cyclic shift) and S small integers: every quantity
    below can be worked out by hand."""
    Pi = np.array([[0.0, 1.0, 0.0], [0.0, 0.0, 1.0], [1.0, 0.0, 0.0]])
    S = np.array([[1.0, 0.0, 0.0], [1.0, 1.0, 0.0], [0.0, -1.0, 2.0]])
    c, t = lloyd_max_beta(3, 4)   # uniform on [-1, 1]: c = -3/4, -1/4, 1/4, 3/4
    return dict(d=3, bits=3, k=2, m=3, mode=MODE_PROD, seed=0, Pi=Pi, S=S, centroids=c, boundaries=t)


def test_quantize_hand_worked_example():
    p = _hand_params()
    x = np.array([[6.0, -2.0, 3.0]])            # ||x|| = 7
    out = oracle.quantize(p, x)
    # u = (6, -2, 3)/7; y = Pi u = (-2, 3, 6)/7 = (-0.2857, 0.4286, 0.8571)
    assert np.array_equal(out["idx"][0], [1, 2, 3])          # -1/4, 1/4, 3/4
    assert out["norm"][0] == 7.0
    # Pi^T c[idx] = (3/4, -1/4, 1/4); r = u - that = (6/7-3/4, -2/7+1/4, 3/7-1/4)
    r = np.array([6 / 7 - 0.75, -2 / 7 + 0.25, 3 / 7 - 0.25])
    assert out["rnorm"][0] == np.float64(np.float16(np.linalg.norm(r)))
    # S r = (r0, r0 + r1, -r1 + 2 r2) = (0.107, 0.071, 0.393) -> all non-negative
    assert np.array_equal(out["signs"][0], [1, 1, 1])
    x2 = np.array([[-6.0, 2.0, -3.0]])
    out2 = oracle.quantize(p, x2)
    assert np.array_equal(out2["idx"][0], [2, 1, 0])
    assert np.array_equal(out2["signs"][0], [0, 0, 0])


def test_quantize_zero_vector():
    p = _hand_params()
    out = oracle.quantize(p, np.zeros((1, 3)))
    assert out["norm"][0] == 0.0 and out["rnorm"][0] == 0.0
    assert np.array_equal(out["idx"][0], [1, 1, 1])   # y = 0 sits on t = 0: lower index
    assert np.array_equal(out["signs"][0], [1, 1, 1])


def test_fp16_round_is_nearest_even():
    ulp = 2.0 ** -10
    v = np.array([1.0 + ulp / 2, 1.0 + 3 * ulp / 2, 1.0 + ulp / 2 + 1e-9, 65504.0, 2.0 ** -25])
    assert list(oracle.fp16_round(v)) == [1.0, 1.0 + 2 * ulp, 1.0 + ulp, 65504.0, 0.0]


def test_dequantize_is_rotated_back_codebook():
    p = _hand_params()
    out = oracle.quantize(p, np.array([[6.0, -2.0, 3.0]]))
    xh = oracle.dequantize(p, out["idx"], out["norm"])
    assert np.allclose(xh[0], 7.0 * np.array([0.75, -0.25, 0.25]), atol=1e-15)


# ---------------------------------------------------------------------- estimator
def test_estimator_is_unbiased_monte_carlo():
    """Over independent draws of (Pi, S), with float64 norms, the mean of
    est(q, k) - <q, k> is zero within 3 sigma (10^5 trials at d = 16)."""
    d, trials = 16, 100000
    rng = np.random.Generator(np.random.PCG64(77))
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    c, t = lloyd_max_beta(d, 4)
    errs = np.empty(trials)
    for i in range(trials):
        p = dict(d=d, k=2, m=d, mode=MODE_PROD, Pi=haar_rotation(rng.standard_normal((d, d))),
                 S=rng.standard_normal((d, d)), centroids=c, boundaries=t)
        code = oracle.quantize(p, k[None, :])
        # float64 norms (the fp16 rounding is a separate, deterministic effect)
        nk = np.linalg.norm(k)
        u = k / nk
        code["norm"] = np.array([nk])
        code["rnorm"] = np.array([np.linalg.norm(u - c[code["idx"][0]] @ p["Pi"])])
        errs[i] = oracle.estimate_inner_products(p, q[None, :], code)[0, 0] - q @ k
    assert abs(errs.mean()) < 3.0 * errs.std() / math.sqrt(trials)
    # the QJL term matters: without it the MSE-only estimate is biased toward 0
    assert errs.std() < 0.5 * abs(q @ k) + 5.0


def test_estimator_mse_part_equals_dequantized_dot():
    p = make_params(32, 4, 17, MODE_PROD)
    rng = np.random.Generator(np.random.PCG64(1))
    k = rng.standard_normal((5, 32))
    q = rng.standard_normal((3, 32))
    code = oracle.quantize(p, k)
    code["rnorm"] = np.zeros(5)                   # switch off the QJL term
    est = oracle.estimate_inner_products(p, q, code)
    assert np.allclose(est, q @ oracle.dequantize(p, code["idx"], code["norm"]).T, rtol=1e-13, atol=1e-12)


def test_estimator_qjl_term_by_hand():
    p = _hand_params()
    code = oracle.quantize(p, np.array([[6.0, -2.0, 3.0]]))
    q = np.array([[1.0, 2.0, -1.0]])
    # <Pi q, c[idx]> = <(2, -1, 1), (-1/4, 1/4, 3/4)> = -0.5 - 0.25 + 0.75 = 0
    # S q = (1, 3, -4); signs all +1 -> <S q, 2s-1> = 0
    assert abs(oracle.estimate_inner_products(p, q, code)[0, 0]) < 1e-14
    q2 = np.array([[1.0, 0.0, 0.0]])
    # Pi q2 = (0, 0, 1): mse = 3/4 ; S q2 = (1, 1, 0): qjl = 2
    rn = code["rnorm"][0]
    expect = 7.0 * (0.75 + math.sqrt(math.pi / 2) / 3 * rn * 2.0)
    assert abs(oracle.estimate_inner_products(p, q2, code)[0, 0] - expect) < 1e-13


def test_qjl_dequantize_by_hand():
    p = _hand_params()
    code = oracle.quantize(p, np.array([[6.0, -2.0, 3.0]]))
    # Pi^T c[idx] = (3/4, -1/4, 1/4); all signs +1, so S^T (2s - 1) = column sums of S = (2, 0, 2)
    rn = code["rnorm"][0]
    kappa = math.sqrt(math.pi / 2) / 3
    expect = 7.0 * (np.array([0.75, -0.25, 0.25]) + kappa * rn * np.array([2.0, 0.0, 2.0]))
    got = oracle.dequantize_qjl(p, code["idx"], code["signs"], code["norm"], code["rnorm"])[0]
    assert np.allclose(got, expect, rtol=0, atol=1e-14)


def test_qjl_dequantize_dots_equal_the_estimator():
    """<e_i, x_hat> = est(e_i, k) for the standard basis (so the vectors are equal), and
    <q, x_hat> = est(q, k) for random q."""
    p = make_params(48, 4, 5, MODE_PROD)
    rng = np.random.Generator(np.random.PCG64(3))
    k = rng.standard_normal((7, 48))
    code = oracle.quantize(p, k)
    xh = oracle.dequantize_qjl(p, code["idx"], code["signs"], code["norm"], code["rnorm"])
    basis = oracle.estimate_inner_products(p, np.eye(48), code)         # [48, 7]
    assert np.allclose(xh, basis.T, rtol=1e-12, atol=1e-12)
    q = rng.standard_normal((5, 48))
    assert np.allclose(q @ xh.T, oracle.estimate_inner_products(p, q, code), rtol=1e-12, atol=1e-11)


def test_qjl_dequantize_is_unbiased_monte_carlo():
    """Over independent draws of (Pi, S) with float64 norms, the mean reconstruction equals
    the key within 3 sigma in every coordinate (2 x 10^4 trials at d = 8)."""
    d, trials = 8, 20000
    rng = np.random.Generator(np.random.PCG64(91))
    k = rng.standard_normal(d)
    c, t = lloyd_max_beta(d, 2)
    acc = np.zeros((trials, d))
    for i in range(trials):
        p = dict(d=d, k=1, m=d, mode=MODE_PROD, Pi=haar_rotation(rng.standard_normal((d, d))),
                 S=rng.standard_normal((d, d)), centroids=c, boundaries=t)
        code = oracle.quantize(p, k[None, :])
        nk = np.linalg.norm(k)
        code["norm"] = np.array([nk])
        code["rnorm"] = np.array([np.linalg.norm(k / nk - c[code["idx"][0]] @ p["Pi"])])
        acc[i] = oracle.dequantize_qjl(p, code["idx"], code["signs"], code["norm"], code["rnorm"])[0]
    err = acc.mean(axis=0) - k
    assert np.all(np.abs(err) < 3.0 * acc.std(axis=0) / math.sqrt(trials))


# ---------------------------------------------------------------------- attention
def _small_cache(B, Hkv, T, groups, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    D = sum(w for _, w, _, _ in groups)
    K = rng.standard_normal((B, Hkv, T, D))
    V = rng.standard_normal((B, Hkv, T, D))
    kp, vp, kc, vc = [], [], [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        kpar = make_params(w, kb, 1000 + 2 * gi, MODE_PROD)
        vpar = make_params(w, vb, 1001 + 2 * gi, MODE_MSE)
        ko = oracle.quantize(kpar, K[..., off:off + w].reshape(-1, w))
        vo = oracle.quantize(vpar, V[..., off:off + w].reshape(-1, w))
        kc.append({key: (None if ko[key] is None else ko[key].reshape(B, Hkv, T, *ko[key].shape[1:]))
                   for key in ("idx", "signs", "norm", "rnorm")})
        vc.append({key: vo[key].reshape(B, Hkv, T, *vo[key].shape[1:]) for key in ("idx", "norm")})
        kp.append(kpar)
        vp.append(vpar)
    offs = [g[0] for g in groups] + [D]
    return kp, vp, offs, kc, vc, D


def test_attention_single_token_returns_dequantized_value():
    kp, vp, offs, kc, vc, D = _small_cache(1, 2, 1, [(0, 16, 3, 3), (16, 16, 2, 2)], 3)
    q = np.random.Generator(np.random.PCG64(0)).standard_normal((1, 4, D))
    o = oracle.decode_attention(kp, vp, offs, q, kc, vc, [1], 0.25)
    for h in range(4):
        hk = h // 2
        vhat = np.concatenate([oracle.dequantize(vp[g], vc[g]["idx"][0, hk], vc[g]["norm"][0, hk])[0]
                               for g in range(2)])
        assert np.allclose(o[0, h], vhat, atol=1e-14)


def test_attention_equal_logits_average_values_and_gqa_mapping():
    kp, vp, offs, kc, vc, D = _small_cache(2, 2, 5, [(0, 16, 3, 4)], 4)
    q = np.zeros((2, 6, D))                      # q = 0: every logit is 0
    o = oracle.decode_attention(kp, vp, offs, q, kc, vc, [5, 3], 1.0)
    for b, T in ((0, 5), (1, 3)):
        for h in range(6):
            hk = h // 3
            vhat = oracle.dequantize(vp[0], vc[0]["idx"][b, hk, :T], vc[0]["norm"][b, hk, :T])
            assert np.allclose(o[b, h], vhat.mean(axis=0), atol=1e-14)


def test_attention_channel_permutation_is_a_relabelling():
    """Decoding with a per-kv-head channel permutation P equals decoding without one on
    inputs whose channels were permuted by P (keys, values and queries), with the output
    permuted back; the identity permutation changes nothing."""
    groups = ((0, 8, 3, 3), (8, 8, 2, 2))
    B, Hkv, T, D = 2, 2, 9, 16
    rng = np.random.Generator(np.random.PCG64(12))
    K = rng.standard_normal((B, Hkv, T, D))
    V = rng.standard_normal((B, Hkv, T, D))
    q = rng.standard_normal((B, 4, D))
    perm = np.stack([rng.permutation(D) for _ in range(Hkv)])
    kp = [make_params(w, kb, 1000 + 2 * gi, MODE_PROD) for gi, (_, w, kb, _) in enumerate(groups)]
    vp = [make_params(w, vb, 1001 + 2 * gi, MODE_MSE) for gi, (_, w, _, vb) in enumerate(groups)]
    offs = [0, 8, 16]

    def caches(Kx, Vx):
        kc, vc = [], []
        for gi, (off, w, _, _) in enumerate(groups):
            ko = oracle.quantize(kp[gi], Kx[..., off:off + w].reshape(-1, w))
            vo = oracle.quantize(vp[gi], Vx[..., off:off + w].reshape(-1, w))
            kc.append({k: ko[k].reshape(B, Hkv, T, *ko[k].shape[1:]) for k in ("idx", "signs", "norm", "rnorm")})
            vc.append({k: vo[k].reshape(B, Hkv, T, *vo[k].shape[1:]) for k in ("idx", "norm")})
        return kc, vc

    # group g of head h holds channels perm[h][off:off+w]: quantize those columns
    Kp = np.stack([K[:, h][..., perm[h]] for h in range(Hkv)], axis=1)
    Vp = np.stack([V[:, h][..., perm[h]] for h in range(Hkv)], axis=1)
    kc, vc = caches(Kp, Vp)
    got = oracle.decode_attention(kp, vp, offs, q, kc, vc, [T, 5], 0.3, channel_perm=perm)
    # reference: no permutation on the permuted problem, output mapped back
    qp = np.stack([q[:, hq][..., perm[hq // 2]] for hq in range(4)], axis=1)
    ref_p = oracle.decode_attention(kp, vp, offs, qp, kc, vc, [T, 5], 0.3)
    ref = np.empty_like(ref_p)
    for hq in range(4):
        ref[:, hq][..., perm[hq // 2]] = ref_p[:, hq]
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    ident = np.stack([np.arange(D)] * Hkv)
    kc0, vc0 = caches(K, V)
    assert np.array_equal(oracle.decode_attention(kp, vp, offs, q, kc0, vc0, [T, 5], 0.3, channel_perm=ident),
                          oracle.decode_attention(kp, vp, offs, q, kc0, vc0, [T, 5], 0.3))


def test_attention_is_invariant_to_token_order():
    kp, vp, offs, kc, vc, D = _small_cache(1, 1, 7, [(0, 32, 4, 4)], 5)
    q = np.random.Generator(np.random.PCG64(2)).standard_normal((1, 2, D))
    o = oracle.decode_attention(kp, vp, offs, q, kc, vc, [7], 0.2)
    perm = np.array([3, 6, 0, 1, 5, 2, 4])
    kc2 = [{k: (None if v is None else v[:, :, perm]) for k, v in kc[0].items()}]
    vc2 = [{k: v[:, :, perm] for k, v in vc[0].items()}]
    o2 = oracle.decode_attention(kp, vp, offs, q, kc2, vc2, [7], 0.2)
    assert np.allclose(o, o2, atol=1e-13)


# ------------------------------------------------------------------------- search
def test_search_ties_keep_lower_id_and_match_pairwise_loop():
    p = make_params(16, 4, 21, MODE_PROD)
    rng = np.random.Generator(np.random.PCG64(9))
    db = rng.standard_normal((40, 16))
    db[25] = db[3]
    db[31] = db[3]                               # three identical entries
    code = oracle.quantize(p, db)
    q = np.vstack([db[3], rng.standard_normal((3, 16))])
    scores, ids = oracle.search_topk(p, q, code, 10)
    assert list(ids[0][:3]) == [3, 25, 31]
    for a in range(len(q)):                      # brute force, one pair at a time
        pair = []
        for b in range(len(db)):
            one = {key: (None if v is None else v[b:b + 1]) for key, v in code.items()}
            pair.append((-oracle.estimate_inner_products(p, q[a:a + 1], one)[0, 0], b))
        pair.sort()
        assert [b for _, b in pair[:10]] == list(ids[a])
        assert np.allclose(scores[a], [-s for s, _ in pair[:10]], atol=1e-12)


def test_recall_definition():
    rng = np.random.Generator(np.random.PCG64(4))
    db = rng.standard_normal((50, 8))
    q = rng.standard_normal((6, 8))
    exact = np.argmax(q @ db.T, axis=1)
    ids = np.stack([[exact[i]] + [(exact[i] + j) % 50 for j in range(1, 10)] for i in range(6)])
    assert oracle.recall_at(ids, q, db) == 1.0
    ids[0] = [(exact[0] + j) % 50 for j in range(1, 11)]
    assert abs(oracle.recall_at(ids, q, db) - 5 / 6) < 1e-15
