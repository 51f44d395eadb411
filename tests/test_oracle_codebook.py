"""Pins for oracle.codebook: closed forms, textbook tables, quadrature, brute force."""
import json
import math
import os

import numpy as np
import pytest
from scipy import integrate
from scipy.special import gammaln

from oracle.codebook import beta_pdf, cell_moments, distortion, lloyd_max


def beta_one_bit(d):
    # E[T | T > 0] for one coordinate of a uniform point on S^{d-1}
    return math.exp(gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d + 1) / 2.0))


@pytest.mark.parametrize("sigma", [1.0, 1 / math.sqrt(128), 0.3])
def test_one_bit_gaussian_closed_form(sigma):
    c, t, _ = lloyd_max(1, "gaussian", sigma=sigma)
    ref = sigma * math.sqrt(2 / math.pi)
    assert abs(c[1] - ref) <= 1e-12 * ref and abs(c[0] + ref) <= 1e-12 * ref
    assert abs(t[0]) <= 1e-15


@pytest.mark.parametrize("d", [2, 3, 8, 128, 1536])
def test_one_bit_beta_closed_form(d):
    c, _, _ = lloyd_max(1, "beta", d=d)
    ref = beta_one_bit(d)
    assert abs(c[1] - ref) <= 1e-12 * ref
    # the Gaussian-limit value sqrt(2/(pi d)) is within a factor (1 + 1/(2d))
    lim = math.sqrt(2 / (math.pi * d))
    assert lim <= ref <= lim * (1 + 1 / (2 * d))


def test_one_bit_beta_d128_value():
    # 1-bit Beta centroid at d=128 vs its Gaussian limit (0.0706616 vs 0.0705237)
    c, _, _ = lloyd_max(1, "beta", d=128)
    assert abs(c[1] - 0.0706616) < 1e-7
    assert abs(math.sqrt(2 / (math.pi * 128)) - 0.0705237) < 1e-7


def test_max_1960_table(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "lloyd_max_gaussian.json")))
    tol = g["digits_abs_tol"]
    for levels, v in g["levels"].items():
        b = int(round(math.log2(int(levels))))
        c, t, _ = lloyd_max(b, "gaussian", sigma=1.0)
        half = c[len(c) // 2:]
        assert np.max(np.abs(half - np.array(v["centroids"]))) < tol
        if "boundaries" in v:
            assert np.max(np.abs(t[len(t) // 2:] - np.array(v["boundaries"]))) < tol
        D = distortion(c, t, "gaussian", sigma=1.0)
        assert abs(D - v["distortion"]) < 1e-4 * max(1.0, 10 * v["distortion"])


def test_one_bit_distortion_exact():
    c, t, _ = lloyd_max(1, "gaussian", sigma=1.0)
    assert abs(distortion(c, t, "gaussian", sigma=1.0) - (1 - 2 / math.pi)) < 1e-13


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("dist", ["gaussian", "beta"])
def test_bound_window(b, dist, golden_dir):
    """4^-b <= D_b <= (sqrt(3) pi / 2) 4^-b (review: Validation/Results)."""
    g = json.load(open(os.path.join(golden_dir, "pages_printed.json")))
    const = math.sqrt(3) * math.pi / 2
    assert abs(const - g["mse_upper_bound_constant"]["value"]) < 0.03
    if dist == "gaussian":
        c, t, _ = lloyd_max(b, dist, sigma=1.0)
        D = distortion(c, t, dist, sigma=1.0)
    else:
        c, t, _ = lloyd_max(b, dist, d=128)
        D = 128 * distortion(c, t, dist, d=128)
    assert 4.0 ** (-b) <= D <= const * 4.0 ** (-b)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_beta_close_to_gaussian_limit(b):
    cg, tg, _ = lloyd_max(b, "gaussian", sigma=1.0)
    cb, tb, _ = lloyd_max(b, "beta", d=128)
    Dg = distortion(cg, tg, "gaussian", sigma=1.0)
    Db = 128 * distortion(cb, tb, "beta", d=128)
    assert abs(Db - Dg) <= 0.03 * Dg


@pytest.mark.parametrize("b", [2, 3, 4])
@pytest.mark.parametrize("dist,d", [("beta", 128), ("beta", 16), ("gaussian", None)])
def test_symmetry_and_centroid_condition_by_quadrature(b, dist, d):
    sigma = None if dist == "beta" else 0.7
    c, t, _ = lloyd_max(b, dist, d=d, sigma=sigma)
    assert np.max(np.abs(c + c[::-1])) < 1e-12
    lo, hi = (-1.0, 1.0) if dist == "beta" else (-np.inf, np.inf)
    pdf = (lambda x: beta_pdf(x, d)) if dist == "beta" else \
        (lambda x: math.exp(-0.5 * (x / sigma) ** 2) / (sigma * math.sqrt(2 * math.pi)))
    edges = np.concatenate([[lo], t, [hi]])
    for k in range(len(c)):
        m, _ = integrate.quad(lambda x: float(pdf(x)), edges[k], edges[k + 1], epsabs=0, epsrel=1e-12, limit=200)
        f, _ = integrate.quad(lambda x: x * float(pdf(x)), edges[k], edges[k + 1], epsabs=0, epsrel=1e-12, limit=200)
        assert abs(f / m - c[k]) < 1e-8 * (1 if dist == "gaussian" else 1 / math.sqrt(d))
    # closed-form cell moments against quadrature
    mass, first, second = cell_moments(edges[:-1], edges[1:], dist, d, sigma)
    for k in range(len(c)):
        s2, _ = integrate.quad(lambda x: x * x * float(pdf(x)), edges[k], edges[k + 1], epsabs=0, epsrel=1e-12, limit=200)
        assert abs(s2 - second[k]) < 1e-10 * max(1.0, abs(s2))


@pytest.mark.parametrize("b", [2, 3, 4])
@pytest.mark.parametrize("dist,d", [("beta", 128), ("gaussian", None)])
def test_discretized_kmeans_agrees(b, dist, d):
    """1-D k-means on a 2*10^6-point midpoint grid converges to the same codebook.

    Cell masses and first moments come from running sums over the grid, linearly
    interpolated at the cell edges (no closed forms), so the discretisation error
    is O(h^2) with h = 1e-5 of the coordinate scale.
    """
    sigma = None if dist == "beta" else 1.0
    c, _, _ = lloyd_max(b, dist, d=d, sigma=sigma)
    scale = 1 / math.sqrt(d) if dist == "beta" else 1.0
    lo, hi = -10.0 * scale, 10.0 * scale
    n = 2_000_000
    h = (hi - lo) / n
    x = lo + (np.arange(n) + 0.5) * h
    w = (beta_pdf(x, d) if dist == "beta" else np.exp(-0.5 * x * x)) * h
    edges = lo + np.arange(n + 1) * h
    cw = np.concatenate([[0.0], np.cumsum(w)])
    cwx = np.concatenate([[0.0], np.cumsum(w * x)])
    cc = np.linspace(-scale, scale, 1 << b)
    for _ in range(20000):
        t = np.concatenate([[lo], 0.5 * (cc[1:] + cc[:-1]), [hi]])
        m = np.diff(np.interp(t, edges, cw))
        f = np.diff(np.interp(t, edges, cwx))
        new = f / m
        moved = np.max(np.abs(new - cc))
        cc = new
        if moved < 1e-14 * scale:
            break
    assert np.max(np.abs(cc - c)) < 1e-6 * scale


def test_monte_carlo_distortion_beta():
    """Empirical per-coordinate MSE of sphere samples matches D_b (within 4 sigma)."""
    rng = np.random.Generator(np.random.PCG64(11))
    d = 32
    g = rng.standard_normal((200_000, d))
    t = (g / np.linalg.norm(g, axis=1, keepdims=True))[:, 0]
    for b in (1, 2, 3):
        c, bd, _ = lloyd_max(b, "beta", d=d)
        err = (t - c[np.searchsorted(bd, t)]) ** 2
        D = distortion(c, bd, "beta", d=d)
        assert abs(err.mean() - D) < 4 * err.std() / math.sqrt(len(err))
