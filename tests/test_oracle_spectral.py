"""Pins for oracle.spectral: printed allocation, optimality, eigen invariants, QJL."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import tq_inputs as ti
from oracle import spectral as SP


def _best_allocation(lam, budget, max_bits):
    """Exhaustive minimum of sum lam_j 4^-b_j over integer b with sum b = budget."""
    best, arg = np.inf, None
    for b in itertools.product(range(max_bits + 1), repeat=len(lam)):
        if sum(b) != budget:
            continue
        v = sum(l * 4.0 ** (-bi) for l, bi in zip(lam, b))
        if v < best - 1e-15:
            best, arg = v, b
    return best, arg


def test_waterfill_printed_split(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pages_printed.json")))["waterfill_split"]
    lam = ti.kv_spectrum(128)[:4]
    assert list(SP.waterfill(lam, sum(g["uniform"]))) == g["waterfilled"]
    assert list(SP.waterfill(np.ones(4), 12)) == g["uniform"]


def test_waterfill_is_optimal():
    rng = np.random.Generator(np.random.PCG64(3))
    for _ in range(30):
        lam = rng.uniform(0.01, 1.0, size=4)
        b = SP.waterfill(lam, 12, 8)
        v = sum(l * 4.0 ** (-bi) for l, bi in zip(lam, b))
        best, _ = _best_allocation(lam, 12, 8)
        assert v <= best * (1 + 1e-12)


def test_printed_lambdas_cannot_give_printed_split(golden_dir):
    """lambda_0 = 0.50 and lambda_3 = 0.04 (ratio 12.5 < 16) never yield [5,3,2,2]."""
    g = json.load(open(os.path.join(golden_dir, "pages_printed.json")))["waterfill_split"]
    for l1 in np.linspace(0.04, 0.5, 24):
        for l2 in np.linspace(0.04, l1, 12):
            lam = [g["lambda0"], l1, l2, g["lambda3"]]
            assert list(SP.waterfill(lam, 12)) != g["waterfilled"]


def test_spectrum_holds_80_percent_in_4_dims(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pages_printed.json")))["signal_dims"]
    lam = ti.kv_spectrum(g["of"])
    assert abs(lam[: g["dims"]].sum() - g["variance_fraction"]) < 0.01


def test_calibration_recovers_generator():
    d, n = 128, 4096
    U = ti.haar_rotation(d, 3004).astype(np.float64)
    X = ti.anisotropic(n, d, U, 7000)
    v, w = SP.calibrate(X)
    lam = d * ti.kv_spectrum(d)
    for j in range(4):
        assert abs(w[j] - lam[j]) <= 4 * lam[j] * math.sqrt(2.0 / n)
        assert abs(v[j] @ U[:, j]) >= 0.99
    M = X.T @ X / n
    assert np.max(np.abs(v @ M @ v.T - np.diag(w))) < 1e-9 * w[0]
    assert np.max(np.abs(v @ v.T - np.eye(d))) < 1e-12
    for j in range(d):
        k = int(np.argmax(np.abs(v[j])))
        assert v[j, k] > 0


def _spectral_setup(qjl=True):
    d, n = 128, 4096
    U = ti.haar_rotation(d, 3004)
    v, w = SP.calibrate(ti.anisotropic(n, d, U, 7000))
    S4 = ti.gaussian_matrix(4, 4, 2004)
    desc = SP.build_descriptor(v, w, 4, 12, 1, qjl, S4)
    return d, U, desc


def test_descriptor_bits_and_record_size():
    d, U, desc = _spectral_setup()
    assert list(desc["bits"][:4]) == [5, 3, 2, 2]
    assert np.all(desc["bits"][4:] == 1)
    assert SP.record_words(desc) == 5          # 16 head bits + 128 tail bits -> 20 bytes


def test_spectral_codes_are_nearest_per_dim():
    d, U, desc = _spectral_setup()
    x = ti.anisotropic(64, d, U, 4004)
    out = SP.quantize_spectral(x, desc)
    for j in range(d):
        c = desc["books"][int(desc["bits"][j])][0] * desc["sigma"][j]
        best = np.argmin(np.abs(out["z"][:, j, None] - c[None, :]), axis=1)
        gap = np.sort(np.abs(out["z"][:, j, None] - c[None, :]), axis=1)
        ok = gap[:, 1] - gap[:, 0] > 1e-12
        assert np.array_equal(best[ok], out["idx"][ok, j])


def test_spectral_record_bigint():
    d, U, desc = _spectral_setup()
    x = ti.anisotropic(8, d, U, 4004)
    out = SP.quantize_spectral(x, desc)
    for i in range(8):
        head, pos = 0, 0
        for j, b in enumerate(desc["bits"][:4]):
            head += int(out["idx"][i, j]) << pos
            pos += int(b)
        for k in range(4):
            head += int(out["s"][i, k]) << (pos + k)
        tail = sum(int(out["idx"][i, j]) << j for j in range(4, d))
        words = [head] + [(tail >> (32 * w)) & 0xFFFFFFFF for w in range(4)]
        assert [int(w) for w in out["codes"][i]] == words


def test_spectral_qjl_unbiased_over_S():
    d, U, desc = _spectral_setup()
    x = ti.anisotropic(1, d, U, 4004)
    q = ti.iid_normal((1, d), 6004)
    base = SP.quantize_spectral(x, desc)
    # truth for the estimator: <q~, z> restricted model (tail uses c_hat, top uses z)
    qt = q[0] @ desc["rot"].T
    truth = float(qt[:4] @ base["z"][0, :4] + qt[4:] @ base["chat"][0, 4:])
    trials = 20000
    est = np.empty(trials)
    for i in range(trials):
        desc["S_top"] = ti.gaussian_matrix(4, 4, 90_000 + i).astype(np.float64)
        out = SP.quantize_spectral(x, desc)
        est[i] = SP.estimate_spectral(q, desc, out["chat"], out["s"], out["rnorms"])[0, 0]
    assert abs(est.mean() - truth) <= 4 * est.std(ddof=1) / math.sqrt(trials)


def _max_distortion(golden_dir, b):
    """Unit-normal Lloyd-Max distortion of b bits, from the printed Max (1960) table."""
    g = json.load(open(os.path.join(golden_dir, "lloyd_max_gaussian.json")))
    return float(g["levels"][str(2 ** b)]["distortion"])


def _recon_gap(dequant, golden_dir, n=20000):
    """(mean squared reconstruction error - its expectation) / standard error.

    The data are drawn from the generator's own eigenbasis, so rot = U^T holds the true
    eigenvectors and z_j = (rot x)_j ~ N(0, lambda_j) independently.  With rot orthogonal,
    ||x - rot^T c_hat||^2 = sum_j (z_j - c_hat_j)^2, whose expectation is
    sum_j lambda_j D_{b_j} with D_b the textbook unit-normal distortion.
    """
    d = 128
    U = ti.haar_rotation(d, 3004).astype(np.float64)
    lam = d * ti.kv_spectrum(d)
    desc = SP.build_descriptor(U.T, lam, 4, 8, 1, False)
    bits = desc["bits"]
    assert bits.max() <= 4, "the pin needs bit widths the printed table covers"
    x = ti.anisotropic(n, d, U, 4104)
    out = SP.quantize_spectral(x, desc)
    err = np.sum((x - dequant(out["chat"], desc)) ** 2, axis=1)
    expect = sum(lam[j] * _max_distortion(golden_dir, int(bits[j])) for j in range(d))
    return (err.mean() - expect) / (err.std(ddof=1) / math.sqrt(n)), err.mean() / expect


def test_dequantize_spectral_reconstruction_error(golden_dir):
    """x_hat = rot^T c_hat: the squared error equals sum_j lambda_j D_{b_j} (printed D_b)."""
    z, ratio = _recon_gap(SP.dequantize_spectral, golden_dir)
    # the Monte-Carlo standard error (~0.25 % of the mean) dwarfs the table's rounding
    assert abs(z) < 4.0, (z, ratio)


def test_dequantize_spectral_pin_rejects_transposed_rotation(golden_dir):
    """A planted mistake (x_hat = rot c_hat) must fail the reconstruction pin."""
    z, ratio = _recon_gap(lambda chat, desc: np.asarray(chat) @ desc["rot"].T, golden_dir, n=4000)
    assert ratio > 1.5 and z > 50.0


def test_dequantize_spectral_permutation_by_hand():
    """rot a permutation: dim j reads x[perm[j]] and its reconstruction returns there."""
    d = 4
    perm = [2, 0, 3, 1]                       # z_j = x[perm[j]]
    rot = np.zeros((d, d))
    for j, i in enumerate(perm):
        rot[j, i] = 1.0
    lam = np.array([4.0, 1.0, 0.25, 0.0625])  # sigma_j = 2, 1, 0.5, 0.25
    desc = SP.build_descriptor(rot, lam, 0, 0, 1, False)
    x = np.array([[0.3, -1.0, 2.0, -0.01]])
    out = SP.quantize_spectral(x, desc)
    a = math.sqrt(2.0 / math.pi)              # 1-bit unit-normal centroid magnitude
    # dim 0 <- x[2] = 2.0 (sigma 2), dim 1 <- x[0] = 0.3 (sigma 1),
    # dim 2 <- x[3] = -0.01 (sigma 0.5), dim 3 <- x[1] = -1.0 (sigma 0.25)
    want = np.array([[1.0 * a, -0.25 * a, 2.0 * a, -0.5 * a]])
    assert np.allclose(SP.dequantize_spectral(out["chat"], desc), want, rtol=1e-12, atol=0)


def test_unpack_spectral_inverts_record_layout():
    """Random codes and signs survive pack -> unpack (the record layout is a bijection)."""
    d, U, desc = _spectral_setup()
    rng = np.random.Generator(np.random.PCG64(12))
    n = 40
    idx = np.zeros((n, d), dtype=np.int64)
    for j in range(d):
        idx[:, j] = rng.integers(0, 1 << int(desc["bits"][j]), size=n)
    s = rng.integers(0, 2, size=(n, 4))
    words = np.stack([SP._pack_record(idx[i], s[i], desc) for i in range(n)])
    gi, gs = SP.unpack_spectral(words, desc)
    assert np.array_equal(gi, idx) and np.array_equal(gs, s)
