"""CUDA path (through the C ABI) against the oracle on the same seeded bf16 bytes.

Sizes the oracle finishes in seconds that still span many warp-tiles and end
in a ragged tail; the full-size workloads are in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import (assert_exact, assert_mse_close, bf16_bits, check_rotated, gpu_run,
                      oracle_run)

pytestmark = pytest.mark.gpu

E8, U4, U5 = 0, 1, 2
NONE, COMP, GIVEN, FROM_AMAX = 0, 1, 2, 3


@pytest.fixture(scope="module")
def fq():
    import microscaling_fp4_quantization_block_b200 as m
    return m


def _parity_exact(fq, x, fmt, block, gmode=NONE, gval=None, rtol=2e-6):
    xb = bf16_bits(x)
    g = gpu_run(fq, x, fmt, block, 0, gmode, gval)
    o = oracle_run(xb, fmt, block, 0, gmode, gval)
    assert_exact(g, o)
    assert_mse_close(g["bm"], g["terms"], o["bm"], o["terms"], rtol)
    return g, o


def test_mxfp4_gaussian_1024x1024_seed0(fq):
    """MXFP4 b32, E8M0, no rotation: 1024 x 1024 N(0, 0.02^2) from seed 0."""
    x = workloads.gaussian_bf16(1024, 1024, 0.02, seed=0)
    g, o = _parity_exact(fq, x, E8, 32)
    assert g["terms"][3] == 0.0                     # MX never zero-rounds at this sigma


@pytest.mark.parametrize("sigma", workloads.QWEN25_7B_SIGMAS)
@pytest.mark.parametrize("gmode", [COMP, GIVEN, NONE])
def test_nvfp4_mlp_slice(fq, sigma, gmode):
    """NVFP4 b16 on a 1184 x 3584 slice of a Qwen2.5-7B gate/up shape (ragged:
    4,243,456 elements is not a multiple of a warp tile)."""
    x = workloads.gaussian_bf16(1184, 3584, sigma, seed=11)
    gval = 4.5 * sigma / 2688.0 if gmode == GIVEN else None
    _parity_exact(fq, x, U4, 16, gmode, gval)


@pytest.mark.parametrize("block", workloads.SWEEP_BLOCKS)
@pytest.mark.parametrize("fmt", [U4, E8, U5])
def test_block_size_sweep(fq, block, fmt):
    """The block-size sweep (UE4M3 without a per-tensor scale, E8M0, UE5M3) at the
    four sigmas, on a 512 x 4096 slice of the 4096 x 4096 sweep matrix."""
    for sigma in workloads.SWEEP_SIGMAS:
        x = workloads.gaussian_bf16(512, 4096, sigma, seed=int(sigma * 1e4) + block)
        _parity_exact(fq, x, fmt, block)


def test_block_size_sweep_full_4096(fq):
    x = workloads.gaussian_bf16(4096, 4096, 0.002, seed=3)
    for block in (8, 16, 256):
        _parity_exact(fq, x, U4, block)
    _parity_exact(fq, x, U4, 16, COMP)


@pytest.mark.parametrize("rot", [16, 32, 128])
@pytest.mark.parametrize("fmt,block,gmode", [(E8, 32, NONE), (U4, 16, COMP), (U4, 16, NONE)])
def test_rotated_activations(fq, rot, fmt, block, gmode):
    """Hadamard micro-rotation fused with MXFP4 / NVFP4 on Student-t(3)
    activations with 8 outlier channels x50 (a 512 x 5120 slice)."""
    x, _ = workloads.student_t_outliers_bf16(512, 5120, seed=rot + block)
    xb = bf16_bits(x)
    g = gpu_run(fq, x, fmt, block, rot, gmode)
    o = oracle_run(xb, fmt, block, rot, gmode, want_mse=False)
    xf = oracle.bf16_bits_to_f32(xb)
    n_codes, n_scales = check_rotated(g, o, xf, fmt, block, rot)
    # MSE: the oracle measures the GPU's own codes, so only the rotation differs
    bm, terms = oracle.block_mse(xb, g["codes"], g["scales"], g["G"], fmt, block, rot)
    assert_mse_close(g["bm"], g["terms"], bm, terms, 1e-5)


@pytest.mark.parametrize("rot", [16, 32, 128])
def test_rotated_gaussian_weights(fq, rot):
    x = workloads.gaussian_bf16(256, 5120, 0.02, seed=rot)
    xb = bf16_bits(x)
    for fmt, block, gmode in [(E8, 32, NONE), (U4, 16, COMP), (U4, 8, NONE), (E8, 256, NONE),
                              (U5, 64, NONE)]:
        g = gpu_run(fq, x, fmt, block, rot, gmode)
        o = oracle_run(xb, fmt, block, rot, gmode, want_mse=False)
        check_rotated(g, o, oracle.bf16_bits_to_f32(xb), fmt, block, rot)
        bm, terms = oracle.block_mse(xb, g["codes"], g["scales"], g["G"], fmt, block, rot)
        assert_mse_close(g["bm"], g["terms"], bm, terms, 1e-5)


@pytest.mark.parametrize("rot", [16, 32, 128])
def test_dequantize_rotates_back(fq, rot):
    x, _ = workloads.student_t_outliers_bf16(64, 1024, seed=5)
    xb = bf16_bits(x)
    for fmt, block in [(E8, 32), (U4, 16)]:
        codes, scales, G = oracle.quantize(xb, fmt, block, rot, NONE)
        want = oracle.dequantize(codes, scales, G, 64, 1024, fmt, block, rot)
        got = fq.fp4q_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), None,
                                 64, 1024, fmt, block, rot, torch.float32).cpu().numpy()
        v = oracle.dequantize(codes, scales, G, 64, 1024, fmt, block, 0)
        l1 = np.abs(v.astype(np.float64)).reshape(-1, rot).sum(1, keepdims=True) / np.sqrt(rot)
        tol = ((np.log2(rot) + 3) * 2.0 ** -24 * l1 * np.ones((1, rot))).reshape(64, 1024)
        assert (np.abs(got.astype(np.float64) - want) <= tol).all()


def test_dequantize_uses_given_scale_and_decodes_every_code(fq):
    """All 16 nibbles x all 127 finite UE4M3 scales x a non-trivial G."""
    rows, cols = 127, 256
    nib = np.tile(np.arange(16, dtype=np.uint8), (rows, cols // 16))
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = np.repeat(np.arange(127, dtype=np.uint8)[:, None], cols // 16, axis=1)
    G = np.float32(0.0123)
    want = oracle.dequantize(codes, scales, float(G), rows, cols, U4, 16, 0)
    got = fq.fp4q_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                             torch.tensor([G]).cuda(), rows, cols, U4, 16, 0, torch.float32).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # E8M0: every exponent
    scales8 = np.repeat(np.arange(255, dtype=np.uint8)[:, None], 2, axis=1)
    codes8 = np.tile(codes[:1, :32], (255, 1))
    want8 = oracle.dequantize(codes8, scales8, 1.0, 255, 64, E8, 32, 0)
    got8 = fq.fp4q_dequantize(torch.from_numpy(codes8).cuda(), torch.from_numpy(scales8).cuda(), None,
                              255, 64, E8, 32, 0, torch.float32).cpu().numpy()
    assert np.array_equal(got8.view(np.uint32), want8.view(np.uint32))


# ----------------------------------------------------------------------------- edge cases
@pytest.mark.parametrize("rows,cols,block,rot", [
    (1, 8, 8, 0), (3, 24, 8, 0), (1, 32, 32, 0), (3, 64, 32, 0), (7, 48, 16, 16), (5, 96, 32, 32),
    (3, 128, 8, 128), (2, 256, 256, 128), (1, 256, 256, 0), (33, 40, 8, 0), (129, 272, 16, 16),
])
def test_small_and_ragged_shapes(fq, rows, cols, block, rot):
    x = workloads.gaussian_bf16(rows, cols, 0.02, seed=rows * 1000 + cols)
    xb = bf16_bits(x)
    for fmt, gmode in [(E8, NONE), (U4, COMP), (U4, NONE), (U5, NONE)]:
        g = gpu_run(fq, x, fmt, block, rot, gmode)
        if rot == 0:
            o = oracle_run(xb, fmt, block, 0, gmode)
            assert_exact(g, o)
            assert_mse_close(g["bm"], g["terms"], o["bm"], o["terms"], 2e-6)
        else:
            o = oracle_run(xb, fmt, block, rot, gmode, want_mse=False)
            check_rotated(g, o, oracle.bf16_bits_to_f32(xb), fmt, block, rot)


def test_empty_tensors(fq):
    for rows, cols in [(0, 64), (4, 0)]:
        x = torch.zeros((rows, cols), dtype=torch.bfloat16, device="cuda")
        codes, scales, gs = fq.fp4q_quantize(x, U4, 16, 0, COMP)
        bm, terms = fq.fp4q_block_mse(x, codes, scales, gs, U4, 16)
        y = fq.fp4q_dequantize(codes, scales, gs, rows, cols, U4, 16)
        torch.cuda.synchronize()
        assert gs.item() == 1.0 and codes.numel() == 0 and y.numel() == 0
        assert terms.cpu().tolist() == [0.0, 0.0, 0.0, 0.0]


def test_special_blocks(fq):
    """All-zero, single non-zero, all-equal, exact powers of two and their
    neighbours, the NVFP4 zero-rounding threshold, negative zeros, bf16
    subnormals and the largest bf16 values, in one tensor."""
    rows, cols = 16, 256
    xb = np.zeros((rows, cols), np.uint16)
    xb[1, 5] = 0x3F80                                   # 1.0 alone
    xb[2, :] = 0xBE00                                   # all -0.125
    xb[3, ::3] = 0x4000                                 # 2.0
    xb[3, 1::3] = 0x3FFF                                # just below 2
    xb[4, :] = np.arange(256) | 0x0000                  # positive bf16 subnormals
    xb[5, :] = (np.arange(256) | 0x8000).astype(np.uint16)
    xb[6, :16] = 0x3BC0                                 # 6 * 2^-10: UE4M3 tie to zero (G = 1)
    xb[6, 16:32] = 0x3BC1
    xb[7, :] = 0x8000                                   # negative zeros
    xb[8, :] = 0x7F7F                                   # largest finite bf16
    xb[8, 1::2] = 0xFF7F
    xb[9, :] = np.random.default_rng(0).integers(0, 0x7F7F, 256).astype(np.uint16)   # wide exponents
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    for fmt, block, gmode in [(E8, 32, NONE), (U4, 16, NONE), (U4, 16, COMP), (U4, 8, NONE),
                              (U5, 16, NONE), (E8, 256, NONE), (U4, 256, COMP)]:
        g = gpu_run(fq, x, fmt, block, 0, gmode, want_mse=False)
        o = oracle_run(xb, fmt, block, 0, gmode, want_mse=False)
        assert_exact(g, o)
        # per-block MSE is an fp32 quantity: rows 8 and 9 (errors near 1e37) overflow it,
        # so the MSE is compared on the other rows
        keep = np.r_[0:8, 10:rows]
        xk = torch.from_numpy(xb[keep].view(np.int16)).view(torch.bfloat16)
        gk = gpu_run(fq, xk, fmt, block, 0, gmode)
        ok = oracle_run(xb[keep], fmt, block, 0, gmode)
        assert_mse_close(gk["bm"], gk["terms"], ok["bm"], ok["terms"], 2e-6)


@pytest.mark.parametrize("gval", [1e-30, 1e-38, 3e-39, 1e-42, 1e30, 7.5e-5])
def test_extreme_given_global_scales(fq, gval):
    """Scales whose reciprocal is not a normal float take the divide path; tiny G
    saturates every block at 448 and large G zero-rounds them."""
    x = workloads.gaussian_bf16(64, 1024, 0.02, seed=8)
    for fmt in (U4, U5):
        g = gpu_run(fq, x, fmt, 16, 0, GIVEN, gval)
        o = oracle_run(bf16_bits(x), fmt, 16, 0, GIVEN, gval)
        assert_exact(g, o)


def test_all_zero_tensor_compute_mode(fq):
    x = torch.zeros((64, 512), dtype=torch.bfloat16)
    g = gpu_run(fq, x, U4, 16, 0, COMP)
    o = oracle_run(bf16_bits(x), U4, 16, 0, COMP)
    assert g["G"] == 1.0
    assert_exact(g, o)
    assert g["terms"].tolist() == [0.0, 0.0, 0.0, 0.0]


def test_tensor_amax_entry_point(fq):
    x, _ = workloads.student_t_outliers_bf16(256, 2048, seed=1)
    xb = bf16_bits(x)
    xf = oracle.bf16_bits_to_f32(xb)
    for rot in (0, 16, 32, 128):
        got = fq.fp4q_tensor_amax(x.cuda(), rot).item()
        if rot == 0:
            assert got == float(np.abs(xf).max())
        else:
            y, bound = __import__("_helpers").exact_rotation(xf, rot)
            assert abs(got - np.abs(y).max()) <= bound.max() + 2 ** -23 * got


def test_split_per_tensor_scale_equals_compute_mode(fq):
    """amax -> global scale -> GIVEN-mode quantize gives COMPUTE mode's result."""
    x, _ = workloads.student_t_outliers_bf16(512, 2048, seed=9)
    xd = x.cuda()
    for rot in (0, 32):
        c1, s1, g1 = fq.fp4q_quantize(xd, U4, 16, rot, COMP)
        amax = fq.fp4q_tensor_amax(xd, rot)
        g2 = fq.fp4q_global_scale(amax)
        c2, s2, _ = fq.fp4q_quantize(xd, U4, 16, rot, GIVEN, gscale=g2)
        torch.cuda.synchronize()
        assert g1.item() == g2.item()
        assert torch.equal(c1, c2) and torch.equal(s1, s2)
    z = torch.zeros(1, device="cuda")
    assert fq.fp4q_global_scale(z).item() == 1.0


@pytest.mark.parametrize("fmt,rot", [(U4, 0), (U4, 32), (U5, 0), (U4, 128)])
def test_from_amax_mode_equals_compute_mode(fq, fmt, rot):
    """amax pass -> quantize with G derived in-kernel (FROM_AMAX) gives COMPUTE
    mode's G, codes and scales; the fused MSE call gives the same terms."""
    x, _ = workloads.student_t_outliers_bf16(512, 2048, seed=19 + rot)
    xd = x.cuda()
    c1, s1, g1 = fq.fp4q_quantize(xd, fmt, 16, rot, COMP)
    _, _, _, bm1, t1 = fq.fp4q_quantize_mse(xd, fmt, 16, rot, COMP)
    g2 = torch.empty(2, dtype=torch.float32, device="cuda")
    fq.fp4q_tensor_amax(xd, rot, amax=g2[:1])
    c2, s2, _ = fq.fp4q_quantize(xd, fmt, 16, rot, FROM_AMAX, gscale=g2)
    g3 = g2.clone()
    g3[1] = -1.0
    c3, s3, _, bm3, t3 = fq.fp4q_quantize_mse(xd, fmt, 16, rot, FROM_AMAX, gscale=g3)
    torch.cuda.synchronize()
    assert g2[1].item() == g1.item() == g3[1].item()
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(c1, c3) and torch.equal(s1, s3)
    assert torch.equal(bm1, bm3) and t1.cpu().numpy().tobytes() == t3.cpu().numpy().tobytes()


def test_from_amax_mode_empty_and_zero_tensors(fq):
    for rows, cols in [(0, 64), (4, 64)]:
        x = torch.zeros((rows, cols), dtype=torch.bfloat16, device="cuda")
        g = torch.empty(2, dtype=torch.float32, device="cuda")
        fq.fp4q_tensor_amax(x, 0, amax=g[:1])
        fq.fp4q_quantize(x, U4, 16, 0, FROM_AMAX, gscale=g)
        torch.cuda.synchronize()
        assert g[0].item() == 0.0 and g[1].item() == 1.0
    with pytest.raises(ValueError):
        fq.fp4q_quantize(x, U4, 16, 0, FROM_AMAX)


def test_mse_workspace_counter_is_left_zero_and_reusable(fq):
    """The in-kernel reduction's completion counter (first 16 workspace bytes)
    is zero after every call, so one zero-filled workspace serves many calls of
    any size: each kernel's terms equal those it gives with a fresh workspace,
    bit for bit (the fused and the separate kernels sum in different orders)."""
    big = workloads.gaussian_bf16(1024, 4096, 0.02, seed=31).cuda()
    small = workloads.gaussian_bf16(16, 512, 0.02, seed=32).cuda()
    ws = torch.zeros(fq.fp4q_block_mse_workspace_size(1024, 4096, 16), dtype=torch.uint8, device="cuda")
    for x in (big, small, big, small):
        c, s, g, bm, t_shared = fq.fp4q_quantize_mse(x, U4, 16, 0, COMP, workspace=ws)
        _, _, _, _, t_fresh = fq.fp4q_quantize_mse(x, U4, 16, 0, COMP)
        _, u_fresh = fq.fp4q_block_mse(x, c, s, g, U4, 16, want_block_mse=False)
        _, u_shared = fq.fp4q_block_mse(x, c, s, g, U4, 16, want_block_mse=False, workspace=ws)
        torch.cuda.synchronize()
        assert not ws[:16].any().item(), "completion counter not reset"
        assert t_shared.cpu().numpy().tobytes() == t_fresh.cpu().numpy().tobytes()
        assert u_shared.cpu().numpy().tobytes() == u_fresh.cpu().numpy().tobytes()
        assert np.allclose(t_shared.cpu().numpy(), u_shared.cpu().numpy(), rtol=1e-6, atol=0)


@pytest.mark.parametrize("rot", [0, 32])
def test_amax_accumulate_over_shards(fq, rot):
    """Row shards folded into one slot give the whole tensor's maximum; a larger
    value already in the slot is kept."""
    x, _ = workloads.student_t_outliers_bf16(768, 1024, seed=41 + rot)
    xd = x.cuda()
    whole = fq.fp4q_tensor_amax(xd, rot)
    acc = torch.zeros(1, dtype=torch.float32, device="cuda")
    for r0 in range(0, 768, 256):
        fq.fp4q_tensor_amax_accumulate(xd[r0:r0 + 256], acc, rot)
    big = torch.full((1,), 1e30, dtype=torch.float32, device="cuda")
    fq.fp4q_tensor_amax_accumulate(xd, big, rot)
    torch.cuda.synchronize()
    assert acc.item() == whole.item() and big.item() == np.float32(1e30)


FUSED_CASES = [(E8, 32, 0, NONE), (U4, 16, 0, COMP), (U4, 16, 0, NONE), (U4, 8, 0, NONE), (E8, 256, 0, NONE),
               (U5, 64, 0, NONE), (E8, 32, 32, NONE), (U4, 16, 128, COMP), (U4, 256, 16, NONE),
               (E8, 8, 128, NONE)]


@pytest.mark.parametrize("fmt,block,rot,gmode", FUSED_CASES)
def test_fused_quantize_mse_matches_separate_calls(fq, fmt, block, rot, gmode):
    """fp4q_quantize_mse: the same codes, scales and G as fp4q_quantize; block MSE
    and the three terms equal the oracle's on those codes (2e-6 unrotated,
    1e-5 rotated)."""
    x, _ = workloads.student_t_outliers_bf16(333, 1024, seed=block + rot)
    xd = x.cuda()
    c1, s1, g1 = fq.fp4q_quantize(xd, fmt, block, rot, gmode)
    c2, s2, g2, bm, terms = fq.fp4q_quantize_mse(xd, fmt, block, rot, gmode)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)
    G = float(g2.item()) if g2 is not None else 1.0
    if g1 is not None:
        assert g1.item() == g2.item()
    xb = bf16_bits(x)
    o_bm, o_terms = oracle.block_mse(xb, c2.cpu().numpy(), s2.cpu().numpy(), G, fmt, block, rot)
    assert_mse_close(bm.cpu().numpy(), terms.cpu().numpy(), o_bm, o_terms, 2e-6 if rot == 0 else 1e-5)


@pytest.mark.parametrize("fmt,block,rot,gmode", FUSED_CASES)
def test_fused_dequantized_output_equals_dequantize(fq, fmt, block, rot, gmode):
    """fp4q_quantize_mse_dequantize: codes, scales, G and MSE as fp4q_quantize_mse,
    and y bit for bit what fp4q_dequantize (bf16, quantized domain) writes."""
    x, _ = workloads.student_t_outliers_bf16(333, 1024, seed=7 * block + rot)
    xd = x.cuda()
    c1, s1, g1, bm1, t1 = fq.fp4q_quantize_mse(xd, fmt, block, rot, gmode)
    c2, s2, g2, y, bm2, t2 = fq.fp4q_quantize_mse_dequantize(xd, fmt, block, rot, gmode)
    ref = fq.fp4q_dequantize(c2, s2, g2 if fmt != E8 else None, 333, 1024, fmt, block, 0, torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(bm1, bm2)
    assert t1.cpu().numpy().tobytes() == t2.cpu().numpy().tobytes()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_fused_dequantized_output_zero_blocks_and_signed_zeros(fq):
    """Zero-rounded blocks give +0, a negative value that rounds to zero -0, and a
    ragged tail; all as fp4q_dequantize."""
    for fmt, block, gmode, gval in [(U4, 16, GIVEN, 1.0), (U4, 8, NONE, None), (E8, 32, NONE, None)]:
        cols = 4096 + block                      # 9 rows: the last unit is partial for b8 and b16
        x = workloads.gaussian_bf16(9, cols, 0.02, seed=12)
        x[0, :64] = 0.0
        x[1, :16] = 1e-7
        x[1, 16:32] = -1e-7
        x[2, 5] = -0.0
        xd = x.cuda()
        gs = torch.tensor([gval], dtype=torch.float32, device="cuda") if gval is not None else None
        c, s, g, y, bm, t = fq.fp4q_quantize_mse_dequantize(xd, fmt, block, 0, gmode, gscale=gs)
        ref = fq.fp4q_dequantize(c, s, g if fmt != E8 else None, 9, cols, fmt, block, 0, torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), fmt


def test_fused_quantize_mse_full_gaussian(fq):
    x = workloads.gaussian_bf16(2048, 3584, 0.005, seed=21)
    xb = bf16_bits(x)
    for fmt, block, gmode in [(U4, 16, COMP), (U4, 8, NONE), (E8, 32, NONE)]:
        c, s, g, bm, terms = fq.fp4q_quantize_mse(x.cuda(), fmt, block, 0, gmode)
        torch.cuda.synchronize()
        o = oracle_run(xb, fmt, block, 0, gmode, want_deq=False)
        assert np.array_equal(c.cpu().numpy(), o["codes"]) and np.array_equal(s.cpu().numpy(), o["scales"])
        assert_mse_close(bm.cpu().numpy(), terms.cpu().numpy(), o["bm"], o["terms"], 2e-6)


def test_block_mse_without_per_block_output_and_determinism(fq):
    x = workloads.gaussian_bf16(2048, 2048, 0.005, seed=4).cuda()
    codes, scales, gs = fq.fp4q_quantize(x, U4, 16, 0, NONE)
    _, t1 = fq.fp4q_block_mse(x, codes, scales, None, U4, 16, want_block_mse=False)
    _, t2 = fq.fp4q_block_mse(x, codes, scales, None, U4, 16, want_block_mse=False)
    bm, t3 = fq.fp4q_block_mse(x, codes, scales, None, U4, 16)
    torch.cuda.synchronize()
    assert t1.cpu().numpy().tobytes() == t2.cpu().numpy().tobytes() == t3.cpu().numpy().tobytes()


def test_errors_leave_the_stream_usable(fq):
    x = workloads.gaussian_bf16(64, 256, 0.02, seed=2).cuda()
    base = torch.empty(64 * 256 + 16, dtype=torch.bfloat16, device="cuda")
    mis = base[1:1 + 64 * 256].view(64, 256)                 # 2-byte offset: misaligned
    L = fq.lib()
    codes = torch.empty((64, 128), dtype=torch.uint8, device="cuda")
    scales = torch.empty((64, 16), dtype=torch.uint8, device="cuda")
    st = L.fp4q_quantize(mis.data_ptr(), 64, 256, U4, 16, 0, NONE, codes.data_ptr(), scales.data_ptr(),
                         None, torch.cuda.current_stream().cuda_stream)
    assert st == -3
    st = L.fp4q_quantize(x.data_ptr(), 64, 250, U4, 16, 0, NONE, codes.data_ptr(), scales.data_ptr(),
                         None, torch.cuda.current_stream().cuda_stream)
    assert st == -2
    c, s, _ = fq.fp4q_quantize(x, U4, 16)
    torch.cuda.synchronize()
    o = oracle_run(bf16_bits(x.cpu()), U4, 16, 0, NONE, want_mse=False, want_deq=False)
    assert np.array_equal(c.cpu().numpy(), o["codes"])


def test_runs_on_a_side_stream(fq):
    x = workloads.gaussian_bf16(512, 1024, 0.02, seed=6).cuda()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        c, sc, gs = fq.fp4q_quantize(x, U4, 16, 0, COMP, stream=s)
    s.synchronize()
    o = oracle_run(bf16_bits(x.cpu()), U4, 16, 0, COMP, want_mse=False, want_deq=False)
    assert np.array_equal(c.cpu().numpy(), o["codes"]) and np.array_equal(sc.cpu().numpy(), o["scales"])
