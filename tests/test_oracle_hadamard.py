"""Pins for the oracle's block-wise Hadamard micro-rotation.

"Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", technical summary s2 and s3.1: block-wise Hadamard rotations of
weights and activations.  The rotation must be the Sylvester Hadamard matrix
(scipy's textbook construction), orthonormal after the 1/sqrt(k) factor, its
own inverse, norm preserving, and applied independently to each run of k
consecutive elements.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle

KS = [2, 4, 8, 16, 32, 64, 128, 256]


@pytest.mark.parametrize("k", KS)
def test_matches_sylvester_construction(k):
    eye = np.eye(k, dtype=np.float32)
    cols = np.stack([oracle.hadamard(eye[j], k) for j in range(k)], axis=1)   # column j = R e_j
    integer = np.rint(cols.astype(np.float64) * np.sqrt(k)).astype(np.int64)
    assert np.array_equal(integer, scipy.linalg.hadamard(k))
    # H H^T = k I, exactly, in integers
    assert np.array_equal(integer @ integer.T, k * np.eye(k, dtype=np.int64))


@pytest.mark.parametrize("k", [16, 32, 128])
def test_involution_and_parseval(k):
    rng = np.random.default_rng(k)
    x = rng.standard_normal(64 * k).astype(np.float32)
    y = oracle.hadamard(x, k)
    z = oracle.hadamard(y, k)
    assert np.max(np.abs(z - x)) <= 4e-6 * np.max(np.abs(x))
    xs, ys = x.reshape(-1, k).astype(np.float64), y.reshape(-1, k).astype(np.float64)
    assert np.allclose((ys ** 2).sum(1), (xs ** 2).sum(1), rtol=1e-6)


def test_chunks_are_independent():
    rng = np.random.default_rng(0)
    a = rng.standard_normal(32).astype(np.float32)
    b = rng.standard_normal(32).astype(np.float32)
    both = oracle.hadamard(np.concatenate([a, b]), 32)
    assert np.array_equal(both, np.concatenate([oracle.hadamard(a, 32), oracle.hadamard(b, 32)]))


def test_exact_for_power_of_four_sizes():
    """k = 16: 1/sqrt(16) = 1/4 is exact, so small-integer inputs give exact sums."""
    x = np.arange(16, dtype=np.float32) - 7
    y = oracle.hadamard(x, 16)
    ref = scipy.linalg.hadamard(16).astype(np.float64) @ x.astype(np.float64) / 4.0
    assert np.array_equal(y, ref.astype(np.float32))


def test_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.hadamard(np.zeros(24, np.float32), 16)
    with pytest.raises(ValueError):
        oracle.hadamard(np.zeros(24, np.float32), 12)
