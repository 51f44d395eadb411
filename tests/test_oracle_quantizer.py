"""Pins for oracle.quantizer: brute force, packing, bias, unbiasedness, variance."""
import itertools
import math

import numpy as np
import pytest
from scipy import stats

import tq_inputs as ti
from oracle.codebook import distortion, lloyd_max
from oracle import quantizer as Q


def _bigint_pack(codes, bits):
    total = 0
    for j, c in enumerate(codes):
        total += int(c) << (j * bits)
    nw = (len(codes) * bits + 31) // 32
    return [(total >> (32 * w)) & 0xFFFFFFFF for w in range(nw)]


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 7, 8])
@pytest.mark.parametrize("d", [8, 12, 33, 128])
def test_pack_matches_bigint_and_roundtrips(bits, d):
    rng = np.random.Generator(np.random.PCG64(bits * 100 + d))
    idx = rng.integers(0, 1 << bits, size=(5, d))
    words = Q.pack_codes(idx, bits)
    for i in range(5):
        assert [int(w) for w in words[i]] == _bigint_pack(idx[i], bits)
    assert np.array_equal(Q.unpack_codes(words, d, bits), idx)


def test_pack_hand_example():
    # 3-bit codes 5,3,7,0 -> bits 101 011 111 000 (LSB first per code) -> 0b000_111_011_101
    w = Q.pack_codes(np.array([[5, 3, 7, 0]]), 3)
    assert w.shape == (1, 1) and int(w[0, 0]) == 0b000111011101


def _nearest_codeword(u, rot, c, d):
    """Exhaustive search over the product codebook in the ORIGINAL domain."""
    cw = np.array(list(itertools.product(c, repeat=d)))          # [K^d, d] rotated-domain codewords
    recon = cw @ rot                                               # Pi^T c as rows
    dist = ((u[None, :] - recon) ** 2).sum(axis=1)
    order = np.argsort(dist)
    return cw[order[0]], dist[order[0]], dist[order[1]]


@pytest.mark.parametrize("bits,d,nvec", [(1, 8, 200), (2, 8, 60), (3, 6, 20)])
def test_brute_force_nearest_codeword(bits, d, nvec):
    c, t, _ = lloyd_max(bits, "beta", d=d)
    rot = ti.haar_rotation(d, 77 + bits).astype(np.float64)
    x = ti.iid_normal((nvec, d), 88 + bits) * 3.0
    out = Q.quantize_mse(x, rot, c, t, bits)
    for i in range(nvec):
        u = x[i] / np.linalg.norm(x[i])
        best, d0, d1 = _nearest_codeword(u, rot, c, d)
        if d1 - d0 < 1e-9:
            continue                                               # tie between codewords
        assert np.allclose(c[out["idx"][i]], best, atol=0)


def test_zero_vector():
    c, t, _ = lloyd_max(2, "beta", d=16)
    rot = ti.haar_rotation(16, 5)
    out = Q.quantize_mse(np.zeros((1, 16)), rot, c, t, 2)
    assert out["norms"][0] == 0.0
    # y = 0 sits on the middle boundary t = 0 and takes the lower cell
    assert np.all(out["idx"] == 1)


def test_dequantize_reconstruction_mse_matches_distortion():
    d, b = 64, 3
    c, t, _ = lloyd_max(b, "beta", d=d)
    rot = ti.haar_rotation(d, 9)
    x = ti.iid_normal((20000, d), 10)
    out = Q.quantize_mse(x, rot, c, t, b)
    xh = Q.dequantize_mse(out["idx"], out["norms"], rot, c)
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    err = np.sum((u - xh / out["norms"][:, None]) ** 2, axis=1)
    D = d * distortion(c, t, "beta", d=d)
    assert abs(err.mean() - D) < 4 * err.std() / math.sqrt(len(err))


def test_mse_inner_product_is_biased_by_one_minus_D():
    """E_Pi <q, x_hat> = (1 - D_b) <q, x> over Haar rotations (review, Problem)."""
    d, b, trials = 16, 2, 3000
    c, t, _ = lloyd_max(b, "beta", d=d)
    D = d * distortion(c, t, "beta", d=d)
    x = ti.iid_normal((1, d), 1)
    q = ti.iid_normal((1, d), 2)
    vals = []
    for s in range(trials):
        rot = ti.haar_rotation(d, 10_000 + s).astype(np.float64)
        out = Q.quantize_mse(x, rot, c, t, b)
        vals.append(Q.estimate_mse(q, rot, out["idx"], out["norms"], c)[0, 0])
    vals = np.array(vals)
    target = (1 - D) * float(q[0] @ x[0])
    assert abs(vals.mean() - target) < 4 * vals.std() / math.sqrt(trials)
    assert abs(target - float(q[0] @ x[0])) > 8 * vals.std() / math.sqrt(trials)


def _prod_setup(d=64, bits=3, m=None):
    m = d if m is None else m
    c, t, _ = lloyd_max(bits - 1, "beta", d=d) if bits > 1 else (None, None, 0)
    rot = ti.haar_rotation(d, 31)
    x = ti.iid_normal((1, d), 32) * 2.0
    q = ti.iid_normal((1, d), 33)
    return d, m, c, t, rot, x, q


@pytest.mark.parametrize("bits", [1, 3])
def test_prod_unbiased_and_variance_over_S(bits):
    d, m, c, t, rot, x, q = _prod_setup(bits=bits)
    trials = 10_000
    est = np.empty(trials)
    for i in range(trials):
        S = ti.gaussian_matrix(m, d, ti.SEEDS["qjl_trials"] + i)
        out = Q.quantize_prod(x, rot, S, c, t, bits)
        est[i] = Q.estimate_prod(q, rot, S, out["chat"], out["s"], out["norms"], out["rnorms"])[0, 0]
    truth = float(q[0] @ x[0])
    z = (est.mean() - truth) / (est.std(ddof=1) / math.sqrt(trials))
    assert abs(z) <= 4
    # exact variance: nu^2/m ((pi/2) gamma^2 ||q'||^2 - <q', r>^2)
    out = Q.quantize_prod(x, rot, ti.gaussian_matrix(m, d, 1), c, t, bits)
    qr = q[0] @ rot.astype(np.float64).T
    var = out["norms"][0] ** 2 / m * (math.pi / 2 * out["rnorms"][0] ** 2 * (qr @ qr) - (qr @ out["r"][0]) ** 2)
    s2 = est.var(ddof=1)
    lo = var * stats.chi2.ppf(0.0005, trials - 1) / (trials - 1)
    hi = var * stats.chi2.ppf(0.9995, trials - 1) / (trials - 1)
    # kurtosis of the per-draw estimate widens the interval a little; allow 10 %
    assert 0.9 * lo <= s2 <= 1.1 * hi


def test_prod_unbiased_over_rotation_and_S():
    d, m, c, t, _, x, q = _prod_setup(d=32, bits=2)
    trials = 6000
    est = np.empty(trials)
    for i in range(trials):
        rot = ti.haar_rotation(d, 50_000 + i)
        S = ti.gaussian_matrix(m, d, 60_000 + i)
        out = Q.quantize_prod(x, rot, S, c, t, 2)
        est[i] = Q.estimate_prod(q, rot, S, out["chat"], out["s"], out["norms"], out["rnorms"])[0, 0]
    truth = float(q[0] @ x[0])
    assert abs(est.mean() - truth) <= 4 * est.std(ddof=1) / math.sqrt(trials)


def test_prod_dequantize_consistent_with_estimator():
    d, m, c, t, rot, x, q = _prod_setup()
    S = ti.gaussian_matrix(m, d, 3)
    out = Q.quantize_prod(x, rot, S, c, t, 3)
    xh = Q.dequantize_prod(out["chat"], out["s"], out["norms"], out["rnorms"], rot, S)
    e1 = float(q[0] @ xh[0])
    e2 = Q.estimate_prod(q, rot, S, out["chat"], out["s"], out["norms"], out["rnorms"])[0, 0]
    assert abs(e1 - e2) < 1e-9 * max(1.0, abs(e1))


def test_signs_bitwise():
    d, m, c, t, rot, x, q = _prod_setup()
    S = ti.gaussian_matrix(m, d, 3)
    out = Q.quantize_prod(x, rot, S, c, t, 3)
    bits = [(int(out["signs"][0, i // 32]) >> (i % 32)) & 1 for i in range(m)]
    assert bits == [1 if v >= 0 else 0 for v in out["proj"][0]]
