"""Pins for oracle.split (outlier-channel split into independent TurboQuant instances)."""
import json
import os

import numpy as np
import pytest

import tq_inputs as ti
from oracle import attention as A
from oracle import quantizer as Q
from oracle import split as SP
from oracle.codebook import distortion, lloyd_max

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_printed.json")


def _mse_instance(d, bits, seed):
    c, t, _ = lloyd_max(bits, "beta", d=d)
    return {"kind": "mse", "rot": ti.haar_rotation(d, seed).astype(np.float64),
            "centroids": c, "boundaries": t, "bits": bits}


def _prod_instance(d, bits, seed):
    c, t, _ = lloyd_max(bits - 1, "beta", d=d)
    return {"kind": "prod", "rot": ti.haar_rotation(d, seed).astype(np.float64),
            "S": ti.gaussian_matrix(d, d, seed + 1).astype(np.float64),
            "centroids": c, "boundaries": t, "bits": bits}


def test_pages_setting_bit_width():
    # the printed 2.5 is the code bits (2.25 per channel) plus one 16-bit norm per group
    g = json.load(open(GOLDEN))["outlier_split_2p5"]
    groups = SP.split_groups(g["d"], np.arange(g["outlier_channels"]))
    assert [len(x) for x in groups] == [g["outlier_channels"], g["d"] - g["outlier_channels"]]
    bits = [g["outlier_bits"], g["other_bits"]]
    assert SP.effective_bits(groups, bits) == 2.25
    assert SP.effective_bits(groups, bits, norm_bits=16) == g["printed_bits"]


def test_detection_finds_planted_channels():
    planted = [3, 17, 40, 41, 90, 127]
    x = ti.planted_outliers(2000, 128, planted, 6.0, 11)
    assert SP.outlier_channels(x, len(planted)).tolist() == planted


def test_detection_ties_go_to_the_lower_channel():
    x = np.ones((5, 10))
    x[:, 7] = 2.0
    assert SP.outlier_channels(x, 3).tolist() == [0, 1, 7]
    assert SP.outlier_channels(x, 0).tolist() == []


def test_groups_must_partition_the_channels():
    x = np.zeros((2, 4))
    ins = [_mse_instance(2, 2, 1), _mse_instance(2, 2, 2)]
    with pytest.raises(ValueError):
        SP.quantize_split(x, [np.array([0, 1]), np.array([1, 2])], ins)
    with pytest.raises(ValueError):
        SP.split_groups(4, [4])


def test_one_group_in_natural_order_is_the_single_instance():
    d, bits = 32, 3
    ins = _mse_instance(d, bits, 5)
    x = ti.iid_normal((50, d), 6)
    q = ti.iid_normal((7, d), 7)
    rec = SP.quantize_split(x, [np.arange(d)], [ins])[0]
    ref = Q.quantize_mse(x, ins["rot"], ins["centroids"], ins["boundaries"], bits)
    assert np.array_equal(rec["codes"], ref["codes"])
    np.testing.assert_allclose(rec["norms"], ref["norms"], rtol=1e-15)      # summation order only
    est = SP.estimate_split(q, [rec], [np.arange(d)], [ins])
    np.testing.assert_allclose(est, Q.estimate_mse(q, ins["rot"], ref["idx"], ref["norms"], ins["centroids"]),
                               rtol=1e-14, atol=1e-14)


def test_channel_order_within_a_group_is_a_relabelling():
    # listing a group's channels in another order, with the rotation's columns permuted to
    # match, quantizes the same rotated vector: identical codes, norms and estimates
    d = 128
    out = np.array([5, 9, 33, 70, 71, 100, 101, 120])
    groups = SP.split_groups(d, out)
    ins = [_mse_instance(len(groups[0]), 3, 21), _mse_instance(len(groups[1]), 2, 22)]
    perm = np.random.Generator(np.random.PCG64(3)).permutation(len(out))
    groups2 = [groups[0][perm], groups[1]]
    ins2 = [dict(ins[0], rot=ins[0]["rot"][:, perm]), ins[1]]
    x = ti.planted_outliers(40, d, out, 5.0, 23)
    q = ti.iid_normal((3, d), 24)
    r1 = SP.quantize_split(x, groups, ins)
    r2 = SP.quantize_split(x, groups2, ins2)
    for a, b in zip(r1, r2):
        assert np.array_equal(a["idx"], b["idx"])
        np.testing.assert_allclose(a["norms"], b["norms"], rtol=1e-15)
    np.testing.assert_allclose(SP.estimate_split(q, r1, groups, ins), SP.estimate_split(q, r2, groups2, ins2),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["mse", "prod"])
def test_estimate_is_the_inner_product_with_the_reconstruction(kind):
    d = 64
    groups = SP.split_groups(d, [0, 1, 2, 3, 60, 61, 62, 63])
    mk = _mse_instance if kind == "mse" else _prod_instance
    ins = [mk(len(groups[0]), 3, 31), mk(len(groups[1]), 2, 32)]
    x = ti.planted_outliers(30, d, groups[0], 4.0, 33)
    q = ti.iid_normal((5, d), 34)
    rec = SP.quantize_split(x, groups, ins)
    xh = SP.dequantize_split(rec, groups, ins, d)
    np.testing.assert_allclose(SP.estimate_split(q, rec, groups, ins), q @ xh.T, rtol=1e-10, atol=1e-10)


def test_reconstruction_error_is_the_sum_of_the_group_distortions():
    # E||x - x_hat||^2 = sum_g D_{b_g}(d_g) E||x_g||^2 with D the Beta-law distortion of
    # the group's own dimension: checks that each group uses its own norm, rotation and
    # codebook and that the reconstruction lands on the right channels
    d, n = 128, 6000
    out = np.arange(0, 128, 4)                                      # 32 outlier channels
    groups = SP.split_groups(d, out)
    ins = [_mse_instance(32, 3, 41), _mse_instance(96, 2, 42)]
    x = ti.planted_outliers(n, d, out, 4.0, 43)
    rec = SP.quantize_split(x, groups, ins)
    err = np.sum((x - SP.dequantize_split(rec, groups, ins, d)) ** 2)
    pred = 0.0
    for ch, g in zip(groups, ins):
        D = len(ch) * distortion(g["centroids"], g["boundaries"], "beta", d=len(ch))
        pred += D * np.sum(x[:, ch] ** 2)
    assert abs(err / pred - 1.0) < 0.03


def _split_attention_error(bits):
    B, Hkv, Hq, N, d = 1, 2, 4, 64, 32
    out = [1, 2, 17, 30]
    groups = SP.split_groups(d, out)
    ins = [_mse_instance(4, bits, 51), _mse_instance(28, bits, 52)]
    K = ti.planted_outliers(B * Hkv * N, d, out, 5.0, 53).reshape(B, Hkv, N, d)
    V = ti.iid_normal((B, Hkv, N, d), 54)
    q = ti.iid_normal((B, Hq, d), 55)
    seq = [N]
    kr = [[SP.quantize_split(K[b, h], groups, ins) for h in range(Hkv)] for b in range(B)]
    vr = [[SP.quantize_split(V[b, h], groups, ins) for h in range(Hkv)] for b in range(B)]
    scale = 1.0 / np.sqrt(d)
    got = A.decode_attention(q, seq, Hkv,
                             lambda b, h, qs: SP.estimate_split(qs, kr[b][h], groups, ins),
                             lambda b, h, n: SP.dequantize_split(vr[b][h], groups, ins, d)[:n], scale)
    ref = A.exact_attention(q, K, V, seq, scale)
    return np.max(np.abs(got - ref)) / np.max(np.abs(ref))


def test_split_attention_converges_to_exact_attention():
    # attention over the split cache approaches exact attention as the groups get bits
    # (a misrouted channel would leave an O(1) error at any width)
    e4, e6 = _split_attention_error(4), _split_attention_error(6)
    assert e6 < 0.06 and e6 < 0.5 * e4
