"""Full-size workloads, in the launch configuration the benchmark times.

The CUDA path runs on whole tensors; the oracle checks sampled rows one by one
(the per-tensor scale G is recomputed by the oracle from the whole tensor, then
the sampled rows are quantized with that G), and whole-tensor properties are
checked at every size: G bit-exact, the three MSE terms add up to the total,
the total equals the mean of the per-block MSE, and for Gaussian weights every
layer's MSE split matches the Gaussian model within Monte-Carlo error.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import assert_exact, assert_mse_close, bf16_bits, check_rotated, oracle_run
from oracle import theory

pytestmark = pytest.mark.gpu

E8, U4 = 0, 1
NONE, COMP, GIVEN = 0, 1, 2


@pytest.fixture(scope="module")
def fq():
    import microscaling_fp4_quantization_block_b200 as m
    return m


def _sample_rows(rows: int, k: int, seed: int):
    rng = np.random.default_rng(seed)
    r = np.unique(np.concatenate([[0, rows - 1], rng.integers(0, rows, k)]))
    return torch.from_numpy(r).cuda()


def _run_full(fq, xd, fmt, block, rot, gmode):
    rows, cols = xd.shape
    codes, scales, gs = fq.fp4q_quantize(xd, fmt, block, rot, gmode)
    gptr = gs if fmt != E8 else None
    bm, terms = fq.fp4q_block_mse(xd, codes, scales, gptr, fmt, block, rot)
    return codes, scales, gs, bm, terms


def _check_sampled(fq, xd, codes, scales, gs, bm, fmt, block, rot, gmode, G_oracle, rows_idx):
    xs = bf16_bits(xd[rows_idx])
    g = {"codes": codes[rows_idx].cpu().numpy(), "scales": scales[rows_idx].cpu().numpy(),
         "G": float(gs.item()) if gs is not None else 1.0, "bm": bm[rows_idx].cpu().numpy()}
    mode = NONE if gmode == NONE else GIVEN
    if rot == 0:
        o = oracle_run(xs, fmt, block, 0, mode, G_oracle, want_deq=False)
        assert_exact(g, o, what=("codes", "scales"))
        assert np.allclose(g["bm"], o["bm"], rtol=2e-6, atol=1e-30)
    else:
        o = oracle_run(xs, fmt, block, rot, mode, G_oracle, want_mse=False, want_deq=False)
        check_rotated(g, o, oracle.bf16_bits_to_f32(xs), fmt, block, rot)


def _terms_consistent(bm, terms):
    """The GPU sums each block's squared errors in fp32 (all of them, and
    separately the non-max ones), so the parts add up to the total to fp32
    rounding; the total is the mean of the per-block MSE to the same bound."""
    t = terms.cpu().numpy()
    assert t[0] == pytest.approx(t[1] + t[2] + t[3], rel=2e-6, abs=1e-300)
    assert t[0] == pytest.approx(bm.double().mean().item(), rel=2e-6)


def test_nvfp4_qwen25_7b_mlp_full(fq):
    """NVFP4 b16 + FP32 per-tensor scale on gate/up 18944x3584 and down
    3584x18944 at sigma 0.005 / 0.02 / 0.05."""
    for idx, (name, x) in enumerate(workloads.nvfp4_mlp_tensors(device="cuda")):
        codes, scales, gs, bm, terms = _run_full(fq, x, U4, 16, 0, COMP)
        torch.cuda.synchronize()
        xh = bf16_bits(x)
        amax = oracle.tensor_amax(oracle.bf16_bits_to_f32(xh))
        G = oracle.global_scale_from_amax(amax)
        assert np.float32(gs.item()) == np.float32(G), name
        _check_sampled(fq, x, codes, scales, gs, bm, U4, 16, 0, COMP, G, _sample_rows(x.shape[0], 24, idx))
        _terms_consistent(bm, terms)
        if idx % 3 == 0:     # whole-tensor oracle MSE on one matrix per sigma
            o_codes, o_scales, o_G = oracle.quantize(xh, U4, 16, 0, GIVEN, G)
            assert np.array_equal(o_codes, codes.cpu().numpy())
            assert np.array_equal(o_scales, scales.cpu().numpy())
            _, o_terms = oracle.block_mse(xh, o_codes, o_scales, G, U4, 16, 0)
            t = terms.cpu().numpy()
            for i in range(4):
                assert abs(t[i] - o_terms[i]) <= 2e-6 * o_terms[0]


def _check_whole_rotated(x, codes, scales, gs, fmt, block, rot, gmode):
    """The whole tensor against the oracle's own run, per-tensor scale included:
    G (COMPUTE mode) from the oracle's fp64 rotation of every element, then
    every scale byte and every code under the rotated-path rule."""
    xh = bf16_bits(x)
    o_codes, o_scales, o_G = oracle.quantize(xh, fmt, block, rot, gmode)
    g = {"codes": codes.cpu().numpy(), "scales": scales.cpu().numpy(),
         "G": float(gs.item()) if gs is not None else 1.0}
    return check_rotated(g, {"codes": o_codes, "scales": o_scales, "G": o_G},
                         oracle.bf16_bits_to_f32(xh), fmt, block, rot)


def test_rotated_activations_full_8192x5120(fq):
    """Every rotation size with MXFP4 (sampled rows against the oracle) and
    NVFP4 with a computed per-tensor scale (the whole tensor against the
    oracle's own run, so the rotated G is the oracle's, not the GPU's)."""
    x, _ = workloads.student_t_outliers_bf16(8192, 5120, seed=77, device="cuda")
    for rot in workloads.ACT_ROTATIONS:
        for fmt, block, gmode in [(E8, 32, NONE), (U4, 16, COMP)]:
            codes, scales, gs, bm, terms = _run_full(fq, x, fmt, block, rot, gmode)
            torch.cuda.synchronize()
            if gmode == COMP:
                xf = oracle.bf16_bits_to_f32(bf16_bits(x))
                if rot == 0:
                    assert np.float32(gs.item()) == np.float32(
                        oracle.global_scale_from_amax(oracle.tensor_amax(xf)))
                    _check_sampled(fq, x, codes, scales, gs, bm, fmt, block, rot, gmode, float(gs.item()),
                                   _sample_rows(8192, 12, rot + block))
                else:
                    _check_whole_rotated(x, codes, scales, gs, fmt, block, rot, gmode)
            else:
                _check_sampled(fq, x, codes, scales, gs, bm, fmt, block, rot, gmode, 1.0,
                               _sample_rows(8192, 12, rot + block))
            _terms_consistent(bm, terms)


def test_qwen25_14b_weight_pass(fq):
    """48 layers x {q, k, v, o, gate, up, down}, sigma_l = 0.02 * U(0.5, 1.5);
    MXFP4 and NVFP4 (per-tensor scale), without and with a 32-wide rotation.
    Sampled rows of every layer's first tensor (and of every tensor of every
    sixth layer) against the oracle, quantized with the GPU's G; the whole k
    projection of every fourth layer against the oracle's MSE terms and, with
    the rotation, against the oracle's own whole run (its own rotated G, every
    scale byte and code); every layer's split against the
    Gaussian model as a sanity bound (bf16 rounding of the inputs moves block
    maxima onto the power-of-two and scale-code boundaries where the
    max-element error jumps, so the continuous model is only good to ~1-2%
    for the max term at this size)."""
    sigmas = workloads.layer_sigmas(workloads.QWEN25_14B_LAYERS, 0.02, 0.5, seed=14)
    variants = [(E8, 32, 0, NONE), (U4, 16, 0, COMP), (E8, 32, 32, NONE), (U4, 16, 32, COMP)]
    for layer, sigma in enumerate(sigmas):
        got = {v: np.zeros(4) for v in variants}
        want = {v: np.zeros(3) for v in variants[:2]}
        layer_n = 0
        for ti, t in enumerate(workloads.QWEN25_14B_LAYER):
            n = t.rows * t.cols
            x = workloads.gaussian_bf16(t.rows, t.cols, sigma, seed=100000 + 16 * layer + ti, device="cuda")
            layer_n += n
            check = (layer % 6 == 0) or ti == 0
            whole = (layer % 4 == 0) and t.name == "k"
            xh = bf16_bits(x) if whole else None
            for v in variants:
                fmt, block, rot, gmode = v
                codes, scales, gs, bm, terms = _run_full(fq, x, fmt, block, rot, gmode)
                tt = terms.cpu().numpy()
                got[v] += tt * n
                G = float(gs.item()) if gs is not None else 1.0
                if v in want:
                    want[v] += np.array(theory.three_terms(fmt, block, sigma, G)) * n
                if check:
                    _check_sampled(fq, x, codes, scales, gs, bm, fmt, block, rot, gmode, G,
                                   _sample_rows(t.rows, 2, layer * 7 + ti))
                if whole and rot:
                    # the rotated per-tensor scale and every code against the oracle's own whole run
                    _check_whole_rotated(x, codes, scales, gs, fmt, block, rot, gmode)
                if whole and (rot == 0 or layer % 12 == 0):
                    _, o_terms = oracle.block_mse(xh, codes.cpu().numpy(), scales.cpu().numpy(), G, fmt,
                                                  block, rot)
                    for i in range(4):
                        assert abs(tt[i] - o_terms[i]) <= (2e-6 if rot == 0 else 1e-5) * o_terms[0]
        for v in variants:
            tl = got[v] / layer_n
            assert tl[0] == pytest.approx(tl[1] + tl[2] + tl[3], rel=2e-6)
            if v in want:
                th = want[v] / layer_n
                assert tl[1] == pytest.approx(th[0], rel=1e-2), (layer, v, tl, th)
                assert tl[2] == pytest.approx(th[1], rel=4e-2), (layer, v, tl, th)
