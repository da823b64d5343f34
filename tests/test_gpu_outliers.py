"""Parity of fp4q_outlier_stats (activation Max, nearest-rank P99.9 and
per-channel maxima, "Diagnosing FP4 inference", Methodology and Results C)
with the oracle through the C ABI.  Every output is a bf16 value chosen by
integer counts, so the bar is bit-exact."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _check(fq, x: torch.Tensor, p: float, ws=None):
    stats, col = fq.fp4q_outlier_stats(x.cuda(), p, workspace=ws)
    torch.cuda.synchronize()
    mx, q, ocol = oracle.outlier_stats(bf16_bits(x), p)
    g = stats.cpu().numpy()
    assert g[0] == np.float32(mx) and g[1] == np.float32(q), (g, mx, q)
    assert np.array_equal(col.cpu().numpy().view(np.uint32), ocol.view(np.uint32))
    return float(g[0]), float(g[1])


@pytest.mark.parametrize("p", [0.999, 0.5, 0.9999, 1.0, 1e-9])
def test_activation_slice(fq, p):
    x, _ = workloads.student_t_outliers_bf16(1024, 5120, seed=21)
    _check(fq, x, p)


@pytest.mark.parametrize("rows,cols", [(1, 8), (3, 24), (7, 1000), (130, 4104), (2, 1 << 20)])
def test_ragged_and_odd_shapes(fq, rows, cols):
    x = workloads.gaussian_bf16(rows, cols, 0.02, seed=rows + cols)
    _check(fq, x, 0.999)


def test_full_activation_tensor(fq):
    """The 8192 x 5120 activation workload: the seeded outlier channels hold
    the largest channel maxima, and the Max/P99.9 ratio shows them."""
    x, channels = workloads.student_t_outliers_bf16(8192, 5120, seed=77)
    mx, q = _check(fq, x, 0.999)
    assert mx / q > 5.0
    _, col = fq.fp4q_outlier_stats(x.cuda(), 0.999)
    top = np.sort(np.argsort(col.cpu().numpy())[-len(channels):])
    assert np.array_equal(top, channels.numpy())


def test_unrepresentative_sample_falls_back(fq):
    """Tensors of 2^22 elements or more are first sampled every s-th row (s <= 16)
    to set a threshold below the quantile.  Here the sampled rows hold all the
    large values, so the threshold lands above the quantile; the count below it
    shows that, and the gated pass completes the histogram: still exact."""
    x = workloads.gaussian_bf16(512, 8192, 0.01, seed=9).float()
    x[::16] *= 1000.0
    x = x.to(torch.bfloat16)
    for p in (0.999, 0.99, 0.9999):
        _check(fq, x, p)


@pytest.mark.parametrize("p", [0.999, 0.5])
def test_sampled_path_shapes(fq, p):
    """Sampled path with few rows (stride capped by the row count) and with a
    row count that is not a multiple of the stride."""
    for rows, cols in [(4, 1 << 20), (1001, 4104)]:
        x = workloads.gaussian_bf16(rows, cols, 0.03, seed=rows)
        _check(fq, x, p)


@pytest.mark.parametrize("rows,cols", [(2049, 4104), (40, 114944), (8191, 520)])
@pytest.mark.parametrize("p", [0.999, 0.99])
def test_sparse_main_pass_column_blocks(fq, rows, cols, p):
    """The sampled path's streaming main pass works on tiles of 4 rows x 256
    channels: a partial last column block (4104 = 16 x 256 + 8), a row count
    that is not a multiple of 4, and 449 column blocks (a prime: the warps'
    column block changes from tile to tile, so channel maxima are flushed on
    every change) all stay exact."""
    x, _ = workloads.student_t_outliers_bf16(rows, cols, seed=rows + cols, n_outlier=min(8, cols))
    _check(fq, x, p)


def test_workspace_reuse_and_no_channels(fq):
    ws = torch.empty((fq.lib().fp4q_outlier_stats_workspace_size(),), dtype=torch.uint8, device="cuda")
    for seed in (1, 2):
        x = workloads.gaussian_bf16(64, 512, 0.05, seed=seed)
        _check(fq, x, 0.999, ws)
    stats, col = fq.fp4q_outlier_stats(workloads.gaussian_bf16(8, 64, 1.0, seed=3).cuda(), channels=False)
    assert col is None and stats.shape == (2,)


def test_special_values(fq):
    """Signed zeros, subnormals, equal magnitudes of both signs."""
    v = torch.tensor([0.0, -0.0, 1e-40, -1e-40, 3.0, -3.0, 2.0, -0.5], dtype=torch.float32)
    x = v.repeat(4, 2).to(torch.bfloat16)
    for p in (0.1, 0.25, 0.5, 0.75, 1.0):
        _check(fq, x, p)
    z = torch.zeros((5, 16), dtype=torch.bfloat16)
    mx, q = _check(fq, z, 0.999)
    assert mx == 0.0 and q == 0.0


def test_empty_and_errors(fq):
    stats, col = fq.fp4q_outlier_stats(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert (stats.cpu() == 0).all() and (col.cpu() == 0).all()
    x = workloads.gaussian_bf16(4, 64, 0.02, seed=1).cuda()
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_outlier_stats(x[:, :60].contiguous())          # cols not a multiple of 8
    for p in (0.0, 1.5, -1.0):
        with pytest.raises(fq.Fp4qError):
            fq.fp4q_outlier_stats(x, p)
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_outlier_stats(x, 0.999, workspace=torch.empty((1024,), dtype=torch.uint8, device="cuda"))
