"""Pins for the oracle's sign vector and Hadamard rotation (CPU).

[ADAPTQ §How it works, item 1] (AdapTQ PyPI page): y = (1/sqrt d)·H·D·x.
Checked against scipy's Sylvester construction, H·H = d·I, orthonormality,
and SplitMix64's published reference outputs.
"""
import numpy as np
import pytest
import scipy.linalg

from conftest import golden_rows
from oracle import rotation as rot


def test_splitmix64_reference_outputs():
    for row in golden_rows("splitmix64.txt"):
        seed = int(row[0])
        want = [int(v) for v in row[1:]]
        assert rot.splitmix64(seed, len(want)) == want


def test_sign_vector_definition():
    d = 128
    outs = rot.splitmix64(7, d)
    sv = rot.sign_vector(7, d)
    assert set(np.unique(sv)) <= {-1.0, 1.0}
    for i in range(d):
        assert (sv[i] < 0) == (outs[i] >= 1 << 63)
    # roughly balanced for a 64-bit generator
    assert 40 < int((rot.sign_vector(0, 128) < 0).sum()) < 88


@pytest.mark.parametrize("d", [1, 2, 4, 64, 128, 256])
def test_hadamard_is_sylvester(d):
    h = rot.hadamard(d)
    np.testing.assert_array_equal(h, scipy.linalg.hadamard(d).astype(np.float64))
    np.testing.assert_array_equal(h @ h, d * np.eye(d))
    np.testing.assert_array_equal(h, h.T)


def test_hadamard_recursion():
    h = rot.hadamard(64)
    h2 = rot.hadamard(128)
    np.testing.assert_array_equal(h2, np.block([[h, h], [h, -h]]))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_orthonormal(d):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, d))
    y = rot.rotate(x, 0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1),
                               rtol=1e-14)
    np.testing.assert_allclose(rot.unrotate(y, 0), x, atol=1e-13)
    # matches the dense product (1/sqrt d)·H·diag(D)·x built from scipy
    dm = np.diag(rot.sign_vector(0, d))
    r = scipy.linalg.hadamard(d) @ dm / np.sqrt(d)
    np.testing.assert_allclose(y, x @ r.T, atol=1e-13)


def test_rotation_spreads_an_outlier():
    """One large channel ends up spread evenly: |y_i| = |x_k|/sqrt(d)."""
    d = 128
    x = np.zeros(d)
    x[17] = 20.0
    y = rot.rotate(x[None], 3)[0]
    np.testing.assert_allclose(np.abs(y), 20.0 / np.sqrt(d), rtol=1e-14)
