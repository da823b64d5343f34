"""Parity of fp4q_quantize_search (MSE-optimised block scales, "Bridging the
Gap", s3, MR-GPTQ item 2) with the oracle, through the C ABI.

The oracle decides each block on the exact squared error (an fp64 sum of
fp64 squared differences); the kernel decides on fp32 sums (two interleaved
running sums of fused multiply-adds).  Each fp32 sum of b non-negative rounded
terms is within (b + 4) 2^-24 relative of the exact one, so the two choices may
differ only between two codes whose exact errors agree to that rounding:
|E1 - E2| <= 2 (b + 4) 2^-24 max(E1, E2), with E the fp64 errors the oracle
measures for each choice.  Everything else is unique:
 * unrotated: the chosen scale lies in the window around the max-rule code,
   and the codes are bit-exact against the oracle's quantizer for the GPU's
   scale bytes; where the scale bytes agree they are simply equal;
 * rotated (fp32 butterflies against fp64): the same, with the rotated-path
   rule for codes and a 1e-5 relative allowance on the errors.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits, check_rotated

pytestmark = pytest.mark.gpu

E8, U4, U5 = 0, 1, 2
NONE, COMP, GIVEN = 0, 1, 2
LAST = {E8: 0xFE, U4: 0x7E, U5: 0xFE}


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _gpu(fq, x, fmt, block, rot, gmode, below, above, gval=None):
    xd = x.cuda()
    gs = torch.tensor([gval], dtype=torch.float32, device="cuda") if gmode == GIVEN else None
    c0, s0, g0 = fq.fp4q_quantize(xd, fmt, block, rot, gmode, gscale=None if gs is None else gs.clone())
    c1, s1, g1 = fq.fp4q_quantize_search(xd, fmt, block, rot, gmode, below, above, gscale=gs)
    torch.cuda.synchronize()
    G = float(g1.item()) if g1 is not None else 1.0
    return c0.cpu().numpy(), s0.cpu().numpy(), c1.cpu().numpy(), s1.cpu().numpy(), G


def _errors(xb, scales, G, fmt, block, rot):
    codes = oracle.quantize_with_scales(xb, scales, G, fmt, block, rot)
    bm, _ = oracle.block_mse(xb, codes, scales, G, fmt, block, rot)
    return bm * block, codes


def _check(fq, x, fmt, block, rot, gmode, below, above, gval=None):
    xb = bf16_bits(x)
    c0, s0, c1, s1, G = _gpu(fq, x, fmt, block, rot, gmode, below, above, gval)
    oc, os_, oG = oracle.quantize_search(xb, fmt, block, rot, gmode, 1.0 if gval is None else gval, below, above)
    if rot == 0:
        assert np.float32(G) == np.float32(oG)
    # the window around the GPU's own max-rule code (itself pinned elsewhere)
    d = s1.astype(np.int64) - s0.astype(np.int64)
    assert ((d >= -below) & (d <= above)).all(), "scale outside the window"
    assert (s1 <= LAST[fmt]).all()
    e_gpu, oc_g = _errors(xb, s1, G, fmt, block, rot)
    e_orc, _ = _errors(xb, os_, oG, fmt, block, rot)
    differ = s1 != os_
    tol = 2.0 * (block + 4) * 2.0 ** -24 + (1e-5 if rot else 0.0)
    gap = np.abs(e_gpu - e_orc)
    bad = differ & (gap > tol * np.maximum(e_gpu, e_orc) + 1e-300)
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5].tolist())
    assert differ.sum() <= max(2, 1e-3 * differ.size), (int(differ.sum()), differ.size)
    if rot == 0:
        assert np.array_equal(c1, oc_g), "codes differ from the oracle's for the GPU's scale bytes"
    else:
        xf = oracle.bf16_bits_to_f32(xb)
        check_rotated({"codes": c1, "scales": s1, "G": G}, {"codes": oc_g, "scales": s1, "G": G},
                      xf, fmt, block, rot)
    return int(differ.sum()), int((s1 != s0).sum())


@pytest.mark.parametrize("fmt,block,gmode,sigma", [
    (E8, 32, NONE, 0.02),
    (U4, 16, COMP, 0.02),
    (U4, 16, NONE, 0.005),          # zero-rounded blocks without a per-tensor scale
    (U4, 8, NONE, 0.002),
    (U5, 16, NONE, 0.02),
    (U4, 256, NONE, 0.02),
    (E8, 64, NONE, 0.05),
])
@pytest.mark.parametrize("below,above", [(0, 0), (1, 1), (3, 1), (0, 2)])
def test_search_unrotated(fq, fmt, block, gmode, sigma, below, above):
    x = workloads.gaussian_bf16(37, 1024, sigma, seed=block + 7 * fmt)      # 37 tiles
    n_diff, n_moved = _check(fq, x, fmt, block, 0, gmode, below, above)
    if below == above == 0:
        assert n_moved == 0
    else:
        assert n_moved > 0


@pytest.mark.parametrize("rot", [16, 32, 128])
@pytest.mark.parametrize("fmt,block,gmode", [(E8, 32, NONE), (U4, 16, COMP), (U4, 64, NONE)])
def test_search_rotated(fq, rot, fmt, block, gmode):
    x, _ = workloads.student_t_outliers_bf16(64, 5120, seed=rot + block)
    _check(fq, x, fmt, block, rot, gmode, 2, 1)


@pytest.mark.parametrize("rows,cols,block", [(1, 256, 16), (3, 384, 32), (29, 768, 8), (5, 2560, 256)])
def test_search_ragged_tails(fq, rows, cols, block):
    """Element counts that end inside a 1024-element tile."""
    x = workloads.gaussian_bf16(rows, cols, 0.02, seed=rows * cols)
    for fmt, gmode in [(E8, NONE), (U4, COMP), (U5, NONE)]:
        _check(fq, x, fmt, block, 0, gmode, 2, 1)


@pytest.mark.parametrize("gval", [1e-30, 1e30, 7.5e-5])
def test_search_extreme_given_scales(fq, gval):
    """Per-tensor scales that send some candidates outside the range of the
    remainder-corrected quotient (the kernel divides there)."""
    x = workloads.gaussian_bf16(16, 1024, 0.02, seed=3)
    _check(fq, x, U4, 16, 0, GIVEN, 3, 2, gval)


def test_search_hand_worked_blocks(fq):
    """The golden blocks, packed into one tensor per (format, block) and run on
    the GPU: the scale bytes the hand arithmetic gives."""
    import json
    import os
    golden = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scale_search_blocks.json")))
    for case in golden["cases"]:
        x = torch.tensor([case["x"]], dtype=torch.float32).to(torch.bfloat16)
        assert torch.equal(x.float(), torch.tensor([case["x"]], dtype=torch.float32))   # exact in bf16
        for below, above, want in case["expect"]:
            xd = x.cuda()
            _, s, _ = fq.fp4q_quantize_search(xd, case["fmt"], case["block"], 0, "none", below, above)
            assert int(s.item()) == want, (case["name"], below, above, int(s.item()), want)


def test_search_empty_and_errors(fq):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    c, s, _ = fq.fp4q_quantize_search(x, U4, 16, 0, "none", 1, 1)
    assert c.numel() == 0 and s.numel() == 0
    x = workloads.gaussian_bf16(4, 64, 0.02, seed=1).cuda()
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_quantize_search(x, U4, 16, 0, "none", 17, 0)
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_quantize_search(x, U4, 16, 0, "none", 0, -1)


def test_search_full_size_sampled_rows(fq):
    """The scale search on a whole Qwen2.5-7B MLP weight (gate 18944 x 3584,
    sigma 0.005, the benchmark's first tensor) in the benchmark's configuration: NVFP4 b16 with the per-tensor
    scale derived from the tensor maximum, window 2 below / 1 above.  Sampled
    rows against the oracle with the same G (blocks never cross a row)."""
    name, x = next(iter(workloads.nvfp4_mlp_tensors(device="cuda")))
    amax = fq.fp4q_tensor_amax(x)
    gs = torch.zeros((2,), dtype=torch.float32, device="cuda")
    gs[0] = amax[0]
    c1, s1, _ = fq.fp4q_quantize_search(x, U4, 16, 0, "from_amax", 2, 1, gscale=gs)
    c0, s0, _ = fq.fp4q_quantize(x, U4, 16, 0, "from_amax", gscale=gs.clone())
    torch.cuda.synchronize()
    G = float(gs[1].item())
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, x.shape[0] - 1], rng.integers(0, x.shape[0], 40)]))
    ri = torch.from_numpy(rows).cuda()
    xb = bf16_bits(x[ri])
    g_codes, g_scales = c1[ri].cpu().numpy(), s1[ri].cpu().numpy()
    oc, os_, _ = oracle.quantize_search(xb, U4, 16, 0, GIVEN, G, 2, 1)
    d = g_scales.astype(np.int64) - s0[ri].cpu().numpy().astype(np.int64)
    assert ((d >= -2) & (d <= 1)).all()
    e_gpu, oc_g = _errors(xb, g_scales, G, U4, 16, 0)
    e_orc, _ = _errors(xb, os_, G, U4, 16, 0)
    differ = g_scales != os_
    tol = 2.0 * (16 + 4) * 2.0 ** -24
    assert not (differ & (np.abs(e_gpu - e_orc) > tol * np.maximum(e_gpu, e_orc) + 1e-300)).any()
    assert differ.sum() <= max(2, 1e-3 * differ.size)
    assert np.array_equal(g_codes, oc_g)
    assert (g_scales != s0[ri].cpu().numpy()).mean() > 0.01     # the search moves a share of the blocks
