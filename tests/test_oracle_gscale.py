"""Pins for the oracle's MSE-optimised per-tensor scale ("Bridging the Gap",
s3.2, MR-GPTQ item 2: the global scale optimised together with the group
scales).  Reading: candidates G_j = fp32(G0 (16 + j) / 16), j in [-below,
above], tried as j = 0, 1, -1, 2, -2, ...; under each, block scales by the max
rule; the exact per-tensor squared error decides, a strictly smaller error
replaces the best, so G0 = amax / 2688 wins every tie.

- the empty window is the max rule (codes, scales and G bit-exact);
- brute force on small tensors: numpy quantizes every candidate from first
  principles (nearest UE4M3 / UE5M3 value of m / 6G with even-code ties,
  IEEE fp32 quotients, nearest E2M1 point) and takes the argmin in the same
  order; the oracle's choice, codes and errors must match;
- the chosen error is never above G0's, nor above any candidate's;
- scale equivariance: doubling the tensor doubles G* and keeps every code and
  scale byte (the rule depends only on ratios to the tensor maximum);
- hand-built tensors, worked by hand: one where G0 is kept, one where a
  larger candidate makes every block exact.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
U4, U5 = oracle.UE4M3, oracle.UE5M3


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _table(fmt):
    n = 127 if fmt == U4 else 255
    dec = oracle.ue4m3_decode if fmt == U4 else oracle.ue5m3_decode
    return np.array([dec(c) for c in range(n)], np.float64)


def _nearest(values, table):
    """Nearest table entry (ties to the even code) for each value."""
    d = np.abs(values[..., None] - table)
    cand = d == d.min(-1, keepdims=True)
    even = cand & (np.arange(len(table)) % 2 == 0)
    return np.where(even.any(-1), even.argmax(-1), cand.argmax(-1))


def _brute_force_error(y, fmt, block, G):
    """Per-tensor MSE of y (fp32 values) under per-tensor scale G, from first principles."""
    table = _table(fmt)
    yb = y.reshape(-1, block).astype(np.float32)
    m = np.abs(yb).max(1).astype(np.float32)
    denom = np.float32(np.float32(6.0) * np.float32(G))
    ratio = (m / denom).astype(np.float32)                      # IEEE fp32 quotient
    codes = _nearest(ratio.astype(np.float64), table)
    S = (table[codes] * np.float64(G)).astype(np.float32)
    err = 0.0
    for i in range(yb.shape[0]):
        if S[i] == 0:
            v = np.zeros(block)
        else:
            q = (yb[i] / S[i]).astype(np.float32)
            d = np.abs(np.abs(q.astype(np.float64))[:, None] - GRID)
            cand = d == d.min(-1, keepdims=True)
            ev = cand & (np.arange(8) % 2 == 0)
            k = np.where(ev.any(-1), ev.argmax(-1), cand.argmax(-1))
            v = (GRID[k] * np.where(np.signbit(q), -1.0, 1.0) * np.float64(S[i])).astype(np.float32)
        err += float(np.sum((yb[i].astype(np.float64) - v.astype(np.float64)) ** 2))
    return err / y.size


def _g0(y):
    amax = np.float32(np.abs(y).max())
    return 1.0 if amax == 0 else float(np.float32(amax / np.float32(2688.0)))


@pytest.mark.parametrize("fmt,block,rot", [(U4, 16, 0), (U4, 16, 32), (U5, 16, 0), (U4, 64, 0)])
def test_empty_window_is_the_max_rule(fmt, block, rot):
    x = _bits(workloads.gaussian_bf16(16, 512, 0.02, seed=5))
    c, s, g, errs = oracle.global_scale_search(x, fmt, block, rot, 0, 0)
    c0, s0, g0 = oracle.quantize(x, fmt, block, rot, oracle.G_COMPUTE)
    assert np.array_equal(c, c0) and np.array_equal(s, s0) and np.float32(g) == np.float32(g0)
    _, t = oracle.block_mse(x, c0, s0, g0, fmt, block, rot)
    assert errs[0] == t[0]


@pytest.mark.parametrize("fmt,block,sigma", [(U4, 16, 0.02), (U4, 8, 0.002), (U5, 16, 0.01)])
def test_brute_force_small_tensors(fmt, block, sigma):
    rng = np.random.default_rng(int(sigma * 1e4) + block + fmt)
    y = (rng.standard_t(3, size=(6, 64)) * sigma).astype(np.float32)
    below, above = 8, 15
    c, s, g, errs = oracle.global_scale_search(y, fmt, block, 0, below, above)
    g0 = _g0(y)
    order = [0] + [v for j in range(1, 16) for v in (j, -j)]
    best, best_err = None, None
    for j in order:
        if j > above or -j > below:
            continue
        G = float(np.float32(np.float64(g0) * (16 + j) / 16))
        e = _brute_force_error(y, fmt, block, G)
        assert errs[j + below] == pytest.approx(e, rel=1e-12, abs=1e-300), j
        if best is None or e < best_err:
            best, best_err = j, e
    assert np.float32(g) == np.float32(np.float64(g0) * (16 + best) / 16)
    cg, sg, _ = oracle.quantize(y, fmt, block, 0, oracle.G_GIVEN, g)
    assert np.array_equal(c, cg) and np.array_equal(s, sg)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_never_worse_than_any_candidate(seed):
    x, _ = workloads.student_t_outliers_bf16(32, 1024, seed=seed)
    c, s, g, errs = oracle.global_scale_search(_bits(x), U4, 16, 0, 8, 15)
    _, t = oracle.block_mse(_bits(x), c, s, g, U4, 16, 0)
    assert t[0] == np.nanmin(errs) and t[0] <= errs[8]


def test_scale_equivariance():
    x = workloads.gaussian_bf16(32, 512, 0.01, seed=9)
    a = oracle.global_scale_search(_bits(x), U4, 16, 0, 8, 15)
    b = oracle.global_scale_search(_bits(x * 2), U4, 16, 0, 8, 15)      # exact in bf16
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.float32(b[2]) == np.float32(2 * a[2])
    assert np.allclose(b[3], 4 * a[3], rtol=0, atol=0)


def test_hand_built_tensors():
    """Two blocks of 16: block A holds the tensor maximum M = 2688 (so G0 = 1)
    and 15 zeros, block B one value and 15 zeros.

    B = 28.6875, window j in [0, 1]: under G0 = 1, A's ratio 2688 / 6 = 448 is a
    UE4M3 value (A exact) and B's 4.78125 rounds to 5, S = 5, 28.6875 / 5 =
    5.7375 rounds to 6: error 1.3125^2.  Under G_1 = 17/16, B's ratio 4.5 is a
    UE4M3 value (B exact), but A's 448 * 16 / 17 = 421.6 rounds to 416, S = 442,
    2688 / 442 = 6.08 rounds to 6, v = 2652: error 36^2.  G0 is kept.

    B = 23.625, window j in [0, 15]: under G_12 = 1.75, A's ratio is 256 (A
    exact: S = 256 * 1.75 = 448, 2688 / 448 = 6) and B's 23.625 / 10.5 = 2.25
    is a UE4M3 value (B exact): error 0.  Under G0, B's ratio 3.9375 rounds to
    4, S = 4, 23.625 / 4 = 5.906 rounds to 6: error 0.375^2.  G_12 wins."""
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 2688.0
    x[0, 16] = 28.6875
    c, s, g, errs = oracle.global_scale_search(x, U4, 16, 0, 0, 1)
    assert g == 1.0
    assert errs[0] == 1.3125 ** 2 / 32 and errs[1] == 36.0 ** 2 / 32
    x[0, 16] = 23.625
    c, s, g, errs = oracle.global_scale_search(x, U4, 16, 0, 0, 15)
    assert g == 1.75 and errs[12] == 0.0 and errs[0] == 0.375 ** 2 / 32
    assert list(s[0]) == [oracle.ue4m3_encode(256.0), oracle.ue4m3_encode(2.25)]
    assert np.array_equal(oracle.dequantize(c, s, g, 1, 32, U4, 16), x)


def test_rejects_bad_windows_and_e8m0():
    x = np.zeros((1, 32), np.float32)
    for below, above in [(-1, 0), (9, 0), (0, 16)]:
        with pytest.raises(ValueError):
            oracle.global_scale_search(x, U4, 16, 0, below, above)
    with pytest.raises(ValueError):
        oracle.global_scale_search(x, oracle.E8M0, 32, 0, 1, 1)
