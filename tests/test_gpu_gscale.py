"""Parity of fp4q_global_scale_search (MSE-optimised per-tensor scale, "Bridging
the Gap", s3.2, MR-GPTQ item 2) with the oracle, through the C ABI.

The oracle decides on the exact (fp64) per-tensor error of every candidate;
the kernel on sums of fp32 block errors (each within (b + 4) 2^-24 relative of
the exact block error).  So:
- every per-candidate error within (b + 4) 2^-24 relative of the oracle's
  (unrotated), 1e-5 (rotated: fp32 butterflies against an fp64 rotation);
- the kernel's own max-rule G0 equal to the oracle's (unrotated), or within
  2^-21 relative (rotated: its tensor maximum comes from fp32 butterflies);
- the chosen candidate index equal to the oracle's, each on its own G0 grid,
  unless the oracle's exact errors of the two choices agree within twice that
  bound (then either is right);
- the hand-worked two-block tensors of the oracle's pins give their hand
  results on the GPU too.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits

pytestmark = pytest.mark.gpu

U4, U5 = 1, 2


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _check(fq, x, fmt, block, rot, below, above):
    xb = bf16_bits(x)
    g, errs = fq.fp4q_global_scale_search(x.cuda(), fmt, block, rot, below, above)
    torch.cuda.synchronize()
    g, errs = float(g.item()), errs.cpu().numpy()
    _, _, og, oerrs = oracle.global_scale_search(xb, fmt, block, rot, below, above)
    tol = (block + 4) * 2.0 ** -24 if rot == 0 else 1e-5
    assert np.allclose(errs, oerrs, rtol=tol, atol=0.0), np.max(np.abs(errs - oerrs) / oerrs)
    # the candidate grids: the oracle's from its G0, the kernel's from its own
    # (equal unrotated; rotated, its maximum comes from fp32 butterflies, so its
    # G0 may differ from the oracle's through that maximum, as the rotated-path
    # rule allows: a few fp32 ulps)
    g0, g0k = _g0(xb, rot), _g0_kernel(fq, x, rot)
    if rot == 0:
        assert np.float32(g0k) == np.float32(g0), (g0k, g0)
    else:
        assert abs(g0k - g0) <= 2.0 ** -21 * g0, (g0k, g0)
    if np.float32(g) != np.float32(og):
        # only between candidates whose exact errors agree to the kernel's rounding
        jg = [j for j in range(-below, above + 1) if np.float32(g) == _candidate(g0k, j)]
        jo = [j for j in range(-below, above + 1) if np.float32(og) == _candidate(g0, j)]
        assert jg and jo, (g, og)
        if jg[0] != jo[0]:
            e1, e2 = oerrs[jg[0] + below], oerrs[jo[0] + below]
            assert abs(e1 - e2) <= 2 * tol * max(e1, e2), (g, og, e1, e2)
    return g, og, errs


def _candidate(g0, j):
    """Candidate j of the per-tensor scale grid: fp32(G0 (16 + j) / 16)."""
    return np.float32(np.float32(g0) * np.float32((16 + j) / 16))


def _g0_kernel(fq, x, rot):
    """The kernel's max-rule G0: its tensor maximum (of the rotated values, for
    rot > 0) / 2688, correctly rounded in fp32, 1 for an all-zero tensor."""
    amax = float(fq.fp4q_tensor_amax(x.cuda(), rot).item())
    return float(np.float32(amax) / np.float32(2688.0)) if amax > 0 else 1.0


def _g0(xb, rot):
    y = oracle.bf16_bits_to_f32(xb)
    if rot:
        y = oracle.hadamard(y, rot)
    return oracle.global_scale_from_amax(oracle.tensor_amax(y))


@pytest.mark.parametrize("fmt,block,sigma", [(U4, 16, 0.02), (U4, 16, 0.002), (U4, 8, 0.005), (U5, 16, 0.02),
                                             (U4, 64, 0.02)])
def test_weights_unrotated(fq, fmt, block, sigma):
    x = workloads.gaussian_bf16(96, 2048, sigma, seed=int(sigma * 1e5) + block)
    _check(fq, x, fmt, block, 0, 8, 15)


@pytest.mark.parametrize("rot", [16, 32, 128])
def test_activations_rotated(fq, rot):
    x, _ = workloads.student_t_outliers_bf16(64, 5120, seed=rot)
    _check(fq, x, U4, 16, rot, 8, 15)


@pytest.mark.parametrize("below,above", [(0, 0), (1, 1), (8, 0), (0, 15)])
def test_windows(fq, below, above):
    x, _ = workloads.student_t_outliers_bf16(40, 1024, seed=3)
    g, og, errs = _check(fq, x, U4, 16, 0, below, above)
    if below == above == 0:
        assert np.float32(g) == np.float32(_g0(bf16_bits(x), 0))


def test_full_size_activations(fq):
    """The 8192 x 5120 activation tensor (41.9 M elements, many CTAs and the
    last-CTA reduction over all of them)."""
    x, _ = workloads.student_t_outliers_bf16(8192, 5120, seed=77, device="cuda")
    g, errs = fq.fp4q_global_scale_search(x, U4, 16, 0, 1, 1)
    torch.cuda.synchronize()
    _, _, og, oerrs = oracle.global_scale_search(bf16_bits(x), U4, 16, 0, 1, 1)
    assert np.allclose(errs.cpu().numpy(), oerrs, rtol=20 * 2.0 ** -24, atol=0.0)
    e = oerrs
    if np.float32(g.item()) != np.float32(og):
        assert abs(np.sort(e)[0] - np.sort(e)[1]) <= 40 * 2.0 ** -24 * e.max()


def test_hand_built_tensors(fq):
    """The oracle's hand-worked tensors with bf16-exact values.  B = 25.5: under
    G0 = 1 its ratio 4.25 ties between the UE4M3 values 4 and 4.5 and goes to
    the even code (4), 25.5 / 4 = 6.375 rounds to 6, error 1.5^2; under G_1 =
    17/16 its ratio is 4 exactly, but block A (2688) loses 36^2.  B = 23.625:
    G_12 = 1.75 makes both blocks exact."""
    x = torch.zeros((1, 32), dtype=torch.float32)
    x[0, 0] = 2688.0
    x[0, 16] = 25.5
    g, errs = fq.fp4q_global_scale_search(x.to(torch.bfloat16).cuda(), U4, 16, 0, 0, 1)
    torch.cuda.synchronize()
    assert float(g.item()) == 1.0 and errs.cpu().tolist() == [1.5 ** 2 / 32, 36.0 ** 2 / 32]
    x[0, 16] = 23.625
    g, errs = fq.fp4q_global_scale_search(x.to(torch.bfloat16).cuda(), U4, 16, 0, 0, 15)
    torch.cuda.synchronize()
    assert float(g.item()) == 1.75
    e = errs.cpu().numpy()
    assert e[12] == 0.0 and e[0] == 0.375 ** 2 / 32


def test_empty_tensor_and_errors(fq):
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    g, errs = fq.fp4q_global_scale_search(x, U4, 16, 0, 2, 3)
    torch.cuda.synchronize()
    assert float(g.item()) == 1.0 and not errs.any()
    with pytest.raises(Exception):
        fq.fp4q_global_scale_search(torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda"), 0, 32, 0, 1, 1)
    with pytest.raises(Exception):
        fq.fp4q_global_scale_search(torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda"), U4, 16, 0, 9, 1)
