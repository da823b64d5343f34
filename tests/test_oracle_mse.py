"""Pins for the oracle's per-block / per-tensor MSE and its three-term split.

"Finer is better? Limits of micro-scaling formats in LLMs", Theoretical
framework and Results: the MSE of Normal weights splits into non-max, block-max
and zero-rounded-block terms, and a first-principles model of those terms
matches experiment.  Here the oracle's Monte-Carlo split on fp32 N(0, sigma^2)
tensors must match the independently derived model (oracle/theory.py) within
4 standard errors per term; the rotated-domain MSE must equal the
original-domain MSE (orthonormal rotation); zero-rounded blocks must carry
their whole energy in the zero term.
"""
import numpy as np
import pytest

import oracle
import workloads
from oracle import theory


def _mc_terms(fmt, block, sigma, G, reps=12, rows=64, blocks_per_row=128, seed=0):
    out = []
    rng = np.random.default_rng(seed)
    gmode = oracle.G_NONE if (fmt == oracle.E8M0 or G == 1.0) else oracle.G_GIVEN
    for _ in range(reps):
        x = (rng.standard_normal((rows, block * blocks_per_row)) * sigma).astype(np.float32)
        codes, scales, g = oracle.quantize(x, fmt, block, 0, gmode, G)
        _, terms = oracle.block_mse(x, codes, scales, g, fmt, block, 0)
        out.append(terms)
    out = np.array(out)
    return out.mean(0), out.std(0, ddof=1) / np.sqrt(reps)


THEORY_CASES = [
    (oracle.E8M0, 32, 0.02, 1.0),
    (oracle.E8M0, 8, 0.005, 1.0),
    (oracle.UE4M3, 16, 0.02, 1.0),
    (oracle.UE4M3, 16, 0.005, 1.0),
    (oracle.UE4M3, 8, 0.002, 1.0),
    (oracle.UE4M3, 64, 0.002, 1.0),
    (oracle.UE4M3, 16, 0.02, 4.5 * 0.02 / 2688.0),      # with a per-tensor scale
    (oracle.UE5M3, 16, 0.002, 1.0),
]


@pytest.mark.parametrize("fmt,block,sigma,G", THEORY_CASES)
def test_three_terms_match_gaussian_theory(fmt, block, sigma, G):
    mean, se = _mc_terms(fmt, block, sigma, G)
    th = np.array(theory.three_terms(fmt, block, sigma, G))
    total = th.sum()
    for i in range(3):
        tol = 4.0 * se[i + 1] + 1e-9 * total
        assert abs(mean[i + 1] - th[i]) <= tol, (i, mean[i + 1], th[i], se[i + 1])
    assert abs(mean[0] - total) <= 4.0 * se[0] + 1e-9 * total


def test_terms_add_up_to_the_total():
    x = workloads.gaussian_f32(32, 1024, 0.005, seed=9).numpy()
    codes, scales, G = oracle.quantize(x, oracle.UE4M3, 16)
    bm, terms = oracle.block_mse(x, codes, scales, G, oracle.UE4M3, 16)
    assert terms[3] > 0 and terms[1] > 0 and terms[2] > 0
    assert terms[0] == pytest.approx(terms[1] + terms[2] + terms[3], rel=1e-12)
    assert bm.mean() == pytest.approx(terms[0], rel=1e-12)


def test_block_mse_matches_dequantized_error():
    x = workloads.gaussian_f32(16, 512, 0.02, seed=2).numpy()
    for fmt, block in [(oracle.E8M0, 32), (oracle.UE4M3, 16), (oracle.UE4M3, 128)]:
        codes, scales, G = oracle.quantize(x, fmt, block)
        v = oracle.dequantize(codes, scales, G, 16, 512, fmt, block).astype(np.float64)
        bm, _ = oracle.block_mse(x, codes, scales, G, fmt, block)
        ref = ((x.astype(np.float64) - v) ** 2).reshape(16, -1, block).mean(-1)
        assert np.allclose(bm, ref, rtol=1e-12, atol=0)


@pytest.mark.parametrize("rot", [16, 32, 128])
def test_rotated_domain_mse_equals_original_domain_mse(rot):
    """The rotation is orthonormal, so the error measured on y = Hx/sqrt(k)
    equals the error between x and the rotated-back dequantized tensor."""
    x, _ = workloads.student_t_outliers_bf16(32, 1024, seed=rot)
    xb = x.view(__import__("torch").int16).numpy().view(np.uint16)
    xf = oracle.bf16_bits_to_f32(xb)
    for fmt, block in [(oracle.E8M0, 32), (oracle.UE4M3, 16)]:
        codes, scales, G = oracle.quantize(xb, fmt, block, rot, oracle.G_NONE)
        _, terms = oracle.block_mse(xb, codes, scales, G, fmt, block, rot)
        back = oracle.dequantize(codes, scales, G, 32, 1024, fmt, block, rot).astype(np.float64)
        orig = np.mean((xf.astype(np.float64) - back) ** 2)
        assert terms[0] == pytest.approx(orig, rel=1e-5)


def test_zero_rounded_block_energy_goes_to_zero_term():
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = np.linspace(-0.004, 0.005, 16)             # max/6 < 2^-10: zero-rounded
    x[0, 16:] = np.linspace(-1.0, 2.0, 16)
    codes, scales, G = oracle.quantize(x, oracle.UE4M3, 16)
    assert scales[0, 0] == 0
    bm, terms = oracle.block_mse(x, codes, scales, G, oracle.UE4M3, 16)
    e0 = np.sum(x[0, :16].astype(np.float64) ** 2)
    assert bm[0, 0] == pytest.approx(e0 / 16, rel=1e-12)
    assert terms[3] == pytest.approx(e0 / 32, rel=1e-12)


def test_max_term_is_the_error_of_the_largest_element():
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 7.0                                            # S = 1: saturates to 6, error 1
    x[0, 1] = 0.3                                            # -> 0.5, error 0.04
    codes, scales, G = oracle.quantize(x, oracle.E8M0, 32)
    _, terms = oracle.block_mse(x, codes, scales, G, oracle.E8M0, 32)
    assert terms[2] * 32 == pytest.approx(1.0, rel=1e-12)
    assert terms[1] * 32 == pytest.approx(np.float64(np.float32(0.3) - 0.5) ** 2, rel=1e-12)


def test_small_block_inversion_under_ue4m3():
    """Narrow distributions under UE4M3 scales without a per-tensor scale get a
    larger MSE at smaller blocks ("Finer is better?", Problem definition and
    Contributions 1); theory and the oracle agree on the ordering."""
    sigma = 0.002
    th = {b: theory.total_mse(oracle.UE4M3, b, sigma) for b in (8, 16, 32)}
    assert th[8] > th[16] > th[32]
    mc = {b: _mc_terms(oracle.UE4M3, b, sigma, 1.0, reps=4, blocks_per_row=2048 // b)[0][0]
          for b in (8, 16, 32)}
    assert mc[8] > mc[16] > mc[32]
    # a per-tensor scale (UE4M3-S) removes the inversion at this sigma
    G = 4.5 * sigma / 2688.0
    ths = {b: theory.total_mse(oracle.UE4M3, b, sigma, G) for b in (8, 16, 32)}
    assert ths[8] < ths[16] < ths[32]
    # so does UE5M3 without any per-tensor scale
    th5 = {b: theory.total_mse(oracle.UE5M3, b, sigma) for b in (8, 16, 32)}
    assert th5[8] < th5[16] < th5[32]


def test_theory_converged():
    a = theory.three_terms(oracle.UE4M3, 16, 0.005, 1.0, nodes=48)
    b = theory.three_terms(oracle.UE4M3, 16, 0.005, 1.0, nodes=96)
    assert np.allclose(a, b, rtol=1e-9, atol=0)
