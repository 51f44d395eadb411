"""Lloyd-Max scalar codebooks for the post-rotation coordinate law (oracle).

R, *Method*: after a random rotation every coordinate of a unit vector follows a
known Beta law (converging to N(0, 1/d)); an optimal Lloyd-Max codebook for it is
"solved once as a continuous 1-D k-means" and then applied per coordinate.
LK, *Show HN post*: "Codebooks are fixed at init".

Two densities (``dist``):

* ``"beta"``     -- exact marginal of one coordinate of a uniform point on S^{d-1}:
  f(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - t^2)^((d-3)/2),  t in [-1, 1].
  Then t^2 ~ Beta(1/2, (d-1)/2), which gives every cell integral in closed form
  through the regularized incomplete beta function.
* ``"gaussian"`` -- N(0, sigma^2) (sigma^2 = 1/d is the limit named in R, Method;
  SpectralQuant uses sigma^2 = lambda_j per dimension).

The iteration is the textbook one: boundaries t_k = (c_k + c_{k+1}) / 2, then each
centroid moves to the conditional mean of its cell, until the largest move is
below ``tol * scale``.  Initial centroids sit at the equal-mass quantiles
(k + 1/2) / 2^b; the densities are log-concave so the fixed point is unique.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import betainc, betaincinv, gammaln, ndtr, ndtri

__all__ = ["cell_moments", "lloyd_max", "distortion", "beta_pdf", "scale_of"]


def scale_of(dist: str, d: int | None, sigma: float | None) -> float:
    """Standard deviation of one coordinate under ``dist``."""
    if dist == "beta":
        return 1.0 / math.sqrt(d)
    if dist == "gaussian":
        return float(sigma)
    raise ValueError(dist)


def beta_pdf(t, d: int):
    """Density of one coordinate of a uniform point on S^{d-1} (R, Method: "known Beta")."""
    t = np.asarray(t, dtype=np.float64)
    logc = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
    with np.errstate(divide="ignore"):
        return np.where(np.abs(t) < 1.0, np.exp(logc + (d - 3) / 2.0 * np.log1p(-t * t)), 0.0)


def _beta_cdf_parts(t: np.ndarray, d: int):
    """Return P(T <= t) and P(T > t) without cancellation in either tail."""
    beta = (d - 1) / 2.0
    t = np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0)
    x = t * t
    # P(|T| <= |t|) = I_{t^2}(1/2, beta);  P(|T| > |t|) = I_{1 - t^2}(beta, 1/2)
    inner = betainc(0.5, beta, x)
    outer = betainc(beta, 0.5, 1.0 - x)
    lower = np.where(t >= 0, 0.5 + 0.5 * inner, 0.5 * outer)   # P(T <= t)
    upper = np.where(t >= 0, 0.5 * outer, 0.5 + 0.5 * inner)   # P(T > t)
    return lower, upper


def cell_moments(a, b, dist: str, d: int | None = None, sigma: float | None = None):
    """Mass, first and second moment of the density on the cells (a_k, b_k].

    Closed forms:
      beta:     int t f = C_d / (d-1) * ((1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)),
                int t^2 f = (1/d) * [P2(b) - P2(a)],  P2(t) = 1/2 + sgn(t)/2 I_{t^2}(3/2, (d-1)/2)
      gaussian: int t phi_s = s (phi(a/s) - phi(b/s)),
                int t^2 phi_s = s^2 [Phi(z) - z phi(z)]_{a/s}^{b/s}
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if dist == "beta":
        beta = (d - 1) / 2.0
        la, ua = _beta_cdf_parts(a, d)
        lb, ub = _beta_cdf_parts(b, d)
        # mass: use the upper tails for cells right of 0, lower tails left of 0
        mass = np.where(a >= 0, ua - ub, lb - la)
        logc = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
        cd = math.exp(logc)
        ac = np.clip(a, -1.0, 1.0)
        bc = np.clip(b, -1.0, 1.0)
        ga = np.power(np.maximum(1.0 - ac * ac, 0.0), beta)
        gb = np.power(np.maximum(1.0 - bc * bc, 0.0), beta)
        first = cd / (d - 1) * (ga - gb)

        def p2(t):
            t = np.clip(t, -1.0, 1.0)
            return 0.5 + 0.5 * np.sign(t) * betainc(1.5, beta, t * t)

        second = (p2(b) - p2(a)) / d
        return mass, first, second
    if dist == "gaussian":
        s = float(sigma)
        za, zb = a / s, b / s
        phia = np.exp(-0.5 * za * za) / math.sqrt(2.0 * math.pi)
        phib = np.exp(-0.5 * zb * zb) / math.sqrt(2.0 * math.pi)
        phia = np.where(np.isfinite(za), phia, 0.0)
        phib = np.where(np.isfinite(zb), phib, 0.0)
        mass = np.where(a >= 0, ndtr(-za) - ndtr(-zb), ndtr(zb) - ndtr(za))
        first = s * (phia - phib)
        za_f = np.where(np.isfinite(za), za, 0.0)
        zb_f = np.where(np.isfinite(zb), zb, 0.0)
        # int_a^b z^2 phi = [Phi(z) - z phi(z)]; the Phi difference equals the mass
        second = s * s * (mass + za_f * phia - zb_f * phib)
        return mass, first, second
    raise ValueError(dist)


def _support(dist: str):
    return (-1.0, 1.0) if dist == "beta" else (-np.inf, np.inf)


def _quantile(p: np.ndarray, dist: str, d: int | None, sigma: float | None) -> np.ndarray:
    if dist == "gaussian":
        return sigma * ndtri(p)
    beta = (d - 1) / 2.0
    q = np.abs(2.0 * p - 1.0)              # P(|T| <= t) = q
    t = np.sqrt(betaincinv(0.5, beta, q))
    return np.sign(p - 0.5) * t


def lloyd_max(bits: int, dist: str, d: int | None = None, sigma: float | None = None,
              tol: float = 1e-13, max_iter: int = 1_000_000):
    """Lloyd-Max codebook with 2^bits levels.

    Returns ``(centroids, boundaries, iterations)``; centroids ascending (index 0
    is the most negative), boundaries ``t_k = (c_k + c_{k+1}) / 2`` (2^bits - 1 of them).
    Raises ``RuntimeError`` if the largest centroid move is still >= tol * scale
    after ``max_iter`` iterations.
    """
    if dist == "beta" and (d is None or d < 2):
        raise ValueError("beta density needs d >= 2")
    if dist == "gaussian" and not (sigma and sigma > 0):
        raise ValueError("gaussian density needs sigma > 0")
    k = 1 << bits
    scale = scale_of(dist, d, sigma)
    lo, hi = _support(dist)
    c = _quantile((np.arange(k) + 0.5) / k, dist, d, sigma)
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[1:] + c[:-1])
        a = np.concatenate([[lo], t])
        b = np.concatenate([t, [hi]])
        mass, first, _ = cell_moments(a, b, dist, d, sigma)
        c_new = first / mass
        move = np.max(np.abs(c_new - c))
        c = c_new
        if move < tol * scale:
            return c, 0.5 * (c[1:] + c[:-1]), it
    raise RuntimeError(f"Lloyd-Max did not converge: bits={bits} dist={dist}")


def distortion(centroids, boundaries, dist: str, d: int | None = None,
               sigma: float | None = None) -> float:
    """Per-coordinate mean-squared error E[(t - c(t))^2] of the scalar quantizer.

    For a unit vector rotated by Pi, E||u - Pi^T c||^2 = d * (this) under the Beta
    law (R, Method); for the Gaussian law with sigma^2 = 1/d the same product is the
    unit-variance distortion D_b.
    """
    lo, hi = _support(dist)
    a = np.concatenate([[lo], boundaries])
    b = np.concatenate([boundaries, [hi]])
    mass, first, second = cell_moments(a, b, dist, d, sigma)
    c = np.asarray(centroids, dtype=np.float64)
    return float(np.sum(second - 2.0 * c * first + c * c * mass))
