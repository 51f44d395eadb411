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
