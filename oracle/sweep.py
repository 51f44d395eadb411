"""Inner-product distortion of TurboQuant-mse and TurboQuant-prod across bit widths (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

R, Figure 3(a) caption: plotted against the bit width, the inner-product distortion of
both variants lies between the proven bounds, and the curves cross: the unbiased prod
variant is better at low bit widths, the mse variant beyond about 3 bits.  R, *Results*:
the prod variant is exactly unbiased.

What is computed here: for pairs (x_i, y_i) the squared error of the inner-product
estimate, E[(<y, x_hat> - <y, x>)^2], split into the squared mean error (bias) and the
rest, for the mse variant at b bits (x_hat its reconstruction) and the prod variant at b
bits ((b-1)-bit MSE stage plus the 1-bit QJL residual, x_hat its unbiased
reconstruction).

Readings (listed in the design notes):

* The pages do not say which pairs the figure uses.  The pairs here are unit vectors x
  and queries y correlated with them, y = rho x + sqrt(1 - rho^2) z with z a unit vector
  orthogonal to x; the crossover is a property of correlated pairs (for rho = 0 the mse
  estimate has no bias to lose and wins at every width).
* Closed forms used by the pins: averaged over the rotation, the mse reconstruction of a
  unit vector is (1 - D_b) x, with D_b = d E[(t - c(t))^2] the codebook distortion (the
  centroid condition gives E[c(t) t] = E[c(t)^2]); the QJL estimate given the residual r
  has variance ((pi/2) ||r||^2 ||y'||^2 - <y', r>^2) / m with y' = Pi y.
"""
from __future__ import annotations

import numpy as np

from . import quantizer as Q

__all__ = ["correlated_pairs", "ip_errors", "sweep"]


def correlated_pairs(x, z, rho: float):
    """Queries y = rho x + sqrt(1 - rho^2) z_perp with z_perp the unit part of z orthogonal to x
    (x rows unit length)."""
    x = np.asarray(x, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    zp = z - np.sum(z * x, axis=1, keepdims=True) * x
    zp /= np.linalg.norm(zp, axis=1, keepdims=True)
    return rho * x + np.sqrt(1.0 - rho * rho) * zp


def ip_errors(x, y, kind: str, bits: int, rot, S=None, codebooks=None):
    """Per-pair errors <y_i, x_hat_i> - <y_i, x_i> of one variant at ``bits`` bits.

    ``codebooks[b]`` = (centroids, boundaries) of the b-bit Lloyd-Max codebook.
    """
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    exact = np.sum(x * y, axis=1)
    if kind == "mse":
        c, t = codebooks[bits]
        r = Q.quantize_mse(x, rot, c, t, bits)
        xh = Q.dequantize_mse(r["idx"], r["norms"], rot, c)
    elif kind == "prod":
        c, t = codebooks[bits - 1] if bits > 1 else (None, None)
        r = Q.quantize_prod(x, rot, S, c, t, bits)
        xh = Q.dequantize_prod(r["chat"], r["s"], r["norms"], r["rnorms"], rot, S)
    else:
        raise ValueError("kind must be mse or prod")
    return np.sum(xh * y, axis=1) - exact


def sweep(x, y, bits_list, rot, S, codebooks):
    """{kind: {b: (mean squared error, squared mean error)}} for kind in (mse, prod)."""
    out = {"mse": {}, "prod": {}}
    for kind in out:
        for b in bits_list:
            e = ip_errors(x, y, kind, b, rot, S, codebooks)
            out[kind][b] = (float(np.mean(e * e)), float(np.mean(e) ** 2))
    return out
