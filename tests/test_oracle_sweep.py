"""Pins for oracle.sweep: inner-product distortion of the mse and prod variants by bit width."""
import json
import math
import os

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as Q
from oracle import sweep as SW
from oracle.codebook import distortion, lloyd_max

D, N = 128, 3000
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_printed.json")


@pytest.fixture(scope="module")
def setup():
    rot = ti.haar_rotation(D, 11).astype(np.float64)
    S = ti.gaussian_matrix(D, D, 12).astype(np.float64)
    x = ti.unit_gaussian(N, D, 13)
    z = ti.unit_gaussian(N, D, 14)
    books = {b: lloyd_max(b, "beta", d=D)[:2] for b in range(1, 6)}
    return rot, S, x, z, books


def test_pairs_have_the_requested_correlation(setup):
    _, _, x, z, _ = setup
    y = SW.correlated_pairs(x, z, 0.9)
    np.testing.assert_allclose(np.sum(x * y, axis=1), 0.9, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), 1.0, atol=1e-12)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_mse_estimate_shrinks_by_the_codebook_distortion(setup, bits):
    # E[<y, x_hat>] = (1 - D_b) <y, x>: the mean relative error is -D_b
    rot, S, x, z, books = setup
    y = SW.correlated_pairs(x, z, 0.9)
    e = SW.ip_errors(x, y, "mse", bits, rot, S, books)
    c, t = books[bits]
    Db = D * distortion(c, t, "beta", d=D)
    rel = np.mean(e) / 0.9
    assert abs(rel + Db) < 0.05 * Db + 3 * np.std(e) / 0.9 / math.sqrt(N)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_prod_is_unbiased_with_the_qjl_variance(setup, bits):
    rot, S, x, z, books = setup
    y = SW.correlated_pairs(x, z, 0.9)
    e = SW.ip_errors(x, y, "prod", bits, rot, S, books)
    assert abs(np.mean(e)) < 4 * np.std(e) / math.sqrt(N)
    # conditional variance of the QJL term given the residual r (rotated unit domain):
    # ((pi/2) ||r||^2 ||y'||^2 - <y', r>^2) / m with y' = Pi y
    c, t = books[bits - 1] if bits > 1 else (None, None)
    r = Q.quantize_prod(x, rot, S, c, t, bits)["r"]
    yr = y @ rot.T
    var = ((math.pi / 2) * np.sum(r * r, 1) * np.sum(yr * yr, 1) - np.sum(yr * r, 1) ** 2) / S.shape[0]
    assert abs(np.mean(e * e) / np.mean(var) - 1.0) < 0.1


def test_curves_cross_near_three_bits_for_correlated_pairs(setup):
    g = json.load(open(GOLDEN))["ip_distortion_crossover"]
    rot, S, x, z, books = setup
    res = SW.sweep(x, SW.correlated_pairs(x, z, 0.9), range(1, 6), rot, S, books)
    k = g["crossover_bits"]
    for b in range(1, 6):
        mse, prod = res["mse"][b][0], res["prod"][b][0]
        if b <= k:
            assert prod < mse, f"b={b}: the prod variant should win at low bit widths"
        else:
            assert mse < prod, f"b={b}: the mse variant should win beyond {k} bits"
    # the mse variant's loss at low widths is its bias
    assert res["mse"][1][1] > 0.5 * res["mse"][1][0]


def test_uncorrelated_pairs_favour_mse_at_every_width(setup):
    rot, S, x, z, books = setup
    res = SW.sweep(x, SW.correlated_pairs(x, z, 0.0), range(1, 6), rot, S, books)
    assert all(res["mse"][b][0] < res["prod"][b][0] for b in range(1, 6))
