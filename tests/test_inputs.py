"""Pins of the seeded input generators (rotations, planted outlier channels; no GPU)."""
import numpy as np
import pytest

import tq_inputs as ti


@pytest.mark.parametrize("d", [2, 8, 64, 128, 256])
def test_hadamard_rotation_is_orthogonal_pm1(d):
    r = ti.hadamard_rotation(d, 1234)
    assert r.dtype == np.float32 and r.shape == (d, d)
    c = np.float32(1.0 / np.sqrt(d))
    assert np.all(np.abs(r) == c)
    r64 = r.astype(np.float64)
    assert np.max(np.abs(r64 @ r64.T - np.eye(d))) < 1e-6


def test_hadamard_rotation_structure():
    d = 16
    r = ti.hadamard_rotation(d, 7) * np.float32(np.sqrt(d))
    s = np.sign(r[0])                       # row 0 of Sylvester H is all ones: it carries the signs
    h = r / s[None, :]
    # Sylvester recursion: H_2n = [[H_n, H_n], [H_n, -H_n]]
    n = d // 2
    assert np.array_equal(h[:n, :n], h[:n, n:]) and np.array_equal(h[n:, :n], h[:n, :n])
    assert np.array_equal(h[n:, n:], -h[:n, :n])
    # H_1 = [1]
    assert h[0, 0] == 1.0
    # the signs are the seeded draw: different seeds differ, equal seeds agree
    assert np.array_equal(ti.hadamard_rotation(d, 7), ti.hadamard_rotation(d, 7))
    assert not np.array_equal(ti.hadamard_rotation(d, 7), ti.hadamard_rotation(d, 8))


def test_hadamard_rotation_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        ti.hadamard_rotation(96, 1)


def test_planted_outliers_scales_exactly_the_listed_channels():
    base = ti.iid_normal((50, 16), 5)
    x = ti.planted_outliers(50, 16, [2, 9], 6.0, 5)
    for j in range(16):
        np.testing.assert_array_equal(x[:, j], base[:, j] * (6.0 if j in (2, 9) else 1.0))
