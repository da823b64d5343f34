"""Rotations of 16 and 32 ("Bridging the Gap", s3.1: block-wise rotation fused
with quantization), through the C ABI, at the edges of the kernels' work
decomposition: one partial tile, exactly one and two 1024-element tiles, many
tiles per warp (the shared-memory ring wrapping round many times), and every
scale format; the fused kernel's codes, scales, dequantized values and MSE, and
the rotated maximum.  The results obey the rotated-path rule against the
oracle's fp64 rotation; the device fault word stays 0.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits, check_rotated, gpu_run, oracle_run, assert_mse_close

pytestmark = pytest.mark.gpu

E8, U4, U5 = 0, 1, 2
NONE, COMP = 0, 1


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    assert m.fp4q_device_fault(clear=True) in (0, 1)
    return m


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 1024), (4, 1024), (8, 1024), (7, 4096), (300, 2048)])
@pytest.mark.parametrize("rot", [16, 32])
def test_tile_edges(fq, rows, cols, rot):
    """n = 32 (one row of one partial tile), 3072, 4096, 8192, 28672 and
    614400 elements."""
    x, _ = workloads.student_t_outliers_bf16(rows, cols, seed=rows * cols + rot, n_outlier=min(8, cols))
    xb = bf16_bits(x)
    for fmt, block, gmode in [(E8, 32, NONE), (U4, 16, COMP), (U4, 8, NONE), (U5, 32, NONE)]:
        g = gpu_run(fq, x, fmt, block, rot, gmode, want_deq=False)
        o = oracle_run(xb, fmt, block, rot, gmode, want_mse=False, want_deq=False)
        check_rotated(g, o, oracle.bf16_bits_to_f32(xb), fmt, block, rot)
    assert fq.fp4q_device_fault() == 0


@pytest.mark.parametrize("rot", [16, 32])
def test_many_tiles_per_warpgroup_fused(fq, rot):
    """2048 x 5120 elements: 10240 tiles of 1024, several per warp; the fused
    kernel's codes, scales, dequantized values and MSE against the oracle."""
    x, _ = workloads.student_t_outliers_bf16(2048, 5120, seed=11 + rot)
    xd = x.cuda()
    xb = bf16_bits(x)
    for fmt, block, gmode in [(E8, 32, "none"), (U4, 16, "compute")]:
        codes, scales, gs, y, bm, terms = fq.fp4q_quantize_mse_dequantize(xd, fmt, block, rot, gmode)
        torch.cuda.synchronize()
        G = float(gs.item()) if gs is not None else 1.0
        g = {"codes": codes.cpu().numpy(), "scales": scales.cpu().numpy(), "G": G}
        o = dict(zip(("codes", "scales", "G"), oracle.quantize(xb, fmt, block, rot, COMP if gmode == "compute"
                                                                 else NONE)))
        check_rotated(g, o, oracle.bf16_bits_to_f32(xb), fmt, block, rot)
        # the dequantized output is the dequantization of the GPU's own codes
        want = oracle.dequantize(g["codes"], g["scales"], G, 2048, 5120, fmt, block, 0)
        got = y.cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, oracle.f32_to_bf16_bits(want))
        o_bm, o_terms = oracle.block_mse(xb, g["codes"], g["scales"], G, fmt, block, rot)
        assert_mse_close(bm.cpu().numpy(), terms.cpu().numpy(), o_bm, o_terms, 1e-5)
    assert fq.fp4q_device_fault() == 0


@pytest.mark.parametrize("rot", [16, 32])
def test_rotated_amax(fq, rot):
    """max |y| of the rotated tensor against the exact rotation: equal up to the
    rotation's rounding."""
    x, _ = workloads.student_t_outliers_bf16(1000, 2048, seed=rot)
    amax = fq.fp4q_tensor_amax(x.cuda(), rot)
    torch.cuda.synchronize()
    xf = oracle.bf16_bits_to_f32(bf16_bits(x))
    want = oracle.tensor_amax(oracle.hadamard(xf, rot))
    l1 = np.abs(xf.astype(np.float64)).reshape(-1, rot).sum(1).max() / np.sqrt(rot)
    assert abs(float(amax.item()) - want) <= (np.log2(rot) + 2) * 2.0 ** -24 * l1 + 2.0 ** -23 * want
    assert fq.fp4q_device_fault() == 0


@pytest.mark.parametrize("rot", [16, 32, 128])
def test_exact_cancellations_give_positive_zero(fq, rot):
    """Runs whose rotated values cancel exactly: the oracle's rotation sums from
    +0, so every zero rotated value is +0 and takes nibble 0x0, never the
    negative-zero nibble 0x8.  Rows of pairwise-equal values make every odd
    position of a run 0, rows of a value and its negation every even one, and
    an all-zero row and one of -0 give 0 everywhere; the codes (and the scales)
    are bit-exact there."""
    rows, cols = 64, 1024
    x, _ = workloads.student_t_outliers_bf16(rows, cols, seed=900 + rot, n_outlier=0)
    x = x.float()
    x[0::4, 1::2] = x[0::4, 0::2]                       # x1 = x0: odd Sylvester sums cancel
    x[1::4, 1::2] = -x[1::4, 0::2]                      # x1 = -x0: even sums cancel
    x[2] = 0.0
    x[3] = -0.0
    x = x.to(torch.bfloat16)
    xb = bf16_bits(x)
    for fmt, block, gmode in [(E8, 32, NONE), (U4, 16, COMP)]:
        g = gpu_run(fq, x, fmt, block, rot, gmode, want_deq=False)
        o = oracle_run(xb, fmt, block, rot, gmode, want_mse=False, want_deq=False)
        gn = oracle.unpack_nibbles(g["codes"]).reshape(rows, cols)
        on = oracle.unpack_nibbles(o["codes"]).reshape(rows, cols)
        y, _ = __import__("_helpers").exact_rotation(oracle.bf16_bits_to_f32(xb), rot)
        zero = y == 0.0
        assert zero.sum() >= rows * cols // 4
        assert (on[zero] == 0).all() and (gn[zero] == 0).all()
        check_rotated(g, o, oracle.bf16_bits_to_f32(xb), fmt, block, rot)
