"""Pins for the oracle's activation outlier statistics (Diagnosing FP4
inference, Methodology and Results C: Max and 99.9th percentile of the
activations, and the Max/P99.9 ratio, per projection).

Reading pinned here: statistics of |x|; the p-quantile by nearest rank, the
k-th smallest magnitude with k = ceil(p N) (fp64), which is numpy's
"inverted_cdf" percentile; per-channel maxima over the columns of a
[tokens, channels] matrix.

- hand-worked tensors of small integers (exact in bf16);
- numpy's inverted-CDF percentile and column maxima on Student-t activations;
- the rank property: at least k magnitudes are <= the quantile, fewer than k
  are below it;
- the activation recipe's seeded outlier channels are the channels with the
  largest maxima.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_hand_worked_ranks():
    assert oracle.nearest_rank(0.999, 1000) == 999
    assert oracle.nearest_rank(0.999, 256) == 256        # ceil(255.744)
    assert oracle.nearest_rank(0.5, 256) == 128
    assert oracle.nearest_rank(1.0, 7) == 7
    assert oracle.nearest_rank(1e-9, 7) == 1
    assert oracle.nearest_rank(0.5, 0) == 0


def test_hand_worked_tensor():
    v = torch.arange(1, 257, dtype=torch.float32)
    for sign in (1.0, -1.0):
        x = (sign * v).reshape(2, 128).to(torch.bfloat16)
        mx, q999, col = oracle.outlier_stats(_bits(x), 0.999)
        assert mx == 256.0 and q999 == 256.0
        _, q50, _ = oracle.outlier_stats(_bits(x), 0.5)
        assert q50 == 128.0
        _, q90, _ = oracle.outlier_stats(_bits(x), 0.9)
        assert q90 == 231.0                               # ceil(230.4) = 231
        assert np.array_equal(col, np.arange(129, 257, dtype=np.float32))


def test_empty_tensor_and_bad_p():
    mx, q, col = oracle.outlier_stats(np.zeros((0, 16), np.uint16))
    assert mx == 0.0 and q == 0.0 and (col == 0).all()
    x = np.zeros((1, 16), np.uint16)
    for p in (0.0, -0.5, 1.5):
        with pytest.raises(ValueError):
            oracle.outlier_stats(x, p)


@pytest.mark.parametrize("p", [0.5, 0.9, 0.99, 0.999, 0.9999, 1.0])
def test_numpy_inverted_cdf(p):
    x, _ = workloads.student_t_outliers_bf16(96, 640, seed=13)
    xb = _bits(x)
    a = np.abs(x.float().numpy())
    mx, q, col = oracle.outlier_stats(xb, p)
    assert mx == a.max()
    assert q == np.percentile(a.ravel(), 100.0 * p, method="inverted_cdf")
    assert np.array_equal(col, a.max(0))
    k = oracle.nearest_rank(p, a.size)
    assert (a <= q).sum() >= k and (a < q).sum() < k


def test_outlier_channels_have_the_largest_maxima():
    x, channels = workloads.student_t_outliers_bf16(512, 1024, seed=5)
    mx, q, col = oracle.outlier_stats(_bits(x), 0.999)
    top = np.sort(np.argsort(col)[-len(channels):])
    assert np.array_equal(top, channels.numpy())
    assert mx / q > 5.0                                   # the outlier channels dominate the maximum
