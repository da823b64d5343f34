"""The block-scaled FP4 GEMM consumer (fp4q_gemm) and the MMA scale layout of
fp4q_quantize_mma, through the C ABI, against the oracle's exact product
(orc_fp4_gemm: Y = G_A G_B sum_k q_A s_A q_B s_B, "Bridging the Gap", s3.4 and
s4: FP4 GEMMs take the codes and block scales of both operands).

Bar:
- fp4q_quantize_mma: codes and G bit-exact against fp4q_quantize's; every scale
  byte equal to fp4q_quantize's after the documented 128 x 4 atom permutation;
- lossless operands (grid values times power-of-two block scales, exponents
  within 2^-1..2^1, so every partial sum is exact in fp32): Y bit-exact;
- any other operands: |Y - Y_exact| <= (k / 16 + 8) 2^-24 G_A G_B sum_k
  |q_A s_A q_B s_B| + 2^-23 |Y_exact|: one fp32 rounding of the accumulator per
  group of products the tensor core adds (at most one per 16 values of k),
  slack for its internal alignment, and the final scaling by fp32(G_A G_B).
Shapes cover partial 128-row / 128-column tiles and k tails that end inside a
256-element stage.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits

pytestmark = pytest.mark.gpu

E8, U4 = 0, 1
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _mma_offset(r, j, sf_kt):
    return ((r // 128) * sf_kt + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)


def _unpermute(sm: np.ndarray, rows: int, nsf: int) -> np.ndarray:
    sf_kt = (nsf + 3) // 4
    r, j = np.meshgrid(np.arange(rows), np.arange(nsf), indexing="ij")
    return sm[_mma_offset(r, j, sf_kt)]


def _operands(fq, x: torch.Tensor, fmt: int, gmode: str):
    """(codes, mma scales, G tensor or None) on the GPU, and the row-major scales
    of fp4q_quantize, checked equal to the MMA layout's."""
    block = 16 if fmt == U4 else 32
    xd = x.cuda()
    c1, s1, g1 = fq.fp4q_quantize(xd, fmt, block, 0, gmode)
    c2, s2, g2 = fq.fp4q_quantize_mma(xd, fmt, block, 0, gmode)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    if g1 is not None:
        assert np.float32(g1.item()) == np.float32(g2.item())
    rows, cols = x.shape
    assert s2.numel() == fq.fp4q_mma_scales_size(rows, cols, block)
    assert np.array_equal(_unpermute(s2.cpu().numpy(), rows, cols // block), s1.cpu().numpy())
    return c2, s2, g2, s1.cpu().numpy()


def _lossless(rows, k, rng, fmt):
    """Grid values times 2^e per block (e in -1..1), one element of each block at
    +-6 2^e, so the max rule keeps 2^e as the block scale (E8M0: floor(log2 6) - 2
    = 0; UE4M3: 6 2^e / 6 = 2^e is a UE4M3 value)."""
    block = 16 if fmt == U4 else 32
    nb = k // block
    e = rng.integers(-1, 2, size=(rows, nb))
    q = GRID[rng.integers(0, 8, size=(rows, k))] * np.where(rng.random((rows, k)) < 0.5, -1.0, 1.0)
    q = q.reshape(rows, nb, block)
    q[:, :, 3] = 6.0 * np.where(rng.random((rows, nb)) < 0.5, -1, 1)
    return torch.from_numpy((q * (2.0 ** e)[..., None]).reshape(rows, k).astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", [E8, U4])
@pytest.mark.parametrize("m,n,k", [(128, 128, 256), (256, 384, 512), (200, 72, 320), (7, 130, 64)])
def test_lossless_operands_exact(fq, fmt, m, n, k):
    rng = np.random.default_rng(m * 7 + n * 3 + k + fmt)
    a, b = _lossless(m, k, rng, fmt), _lossless(n, k, rng, fmt)
    ca, sa, _, sa_rm = _operands(fq, a, fmt, "none")
    cb, sb, _, sb_rm = _operands(fq, b, fmt, "none")
    y = fq.fp4q_gemm(ca, sa, None, cb, sb, None, fmt)
    torch.cuda.synchronize()
    block = 16 if fmt == U4 else 32
    want = oracle.fp4_gemm(ca.cpu().numpy(), sa_rm, 1.0, cb.cpu().numpy(), sb_rm, 1.0, k, fmt, block)
    assert np.array_equal(want, a.double().numpy() @ b.double().numpy().T)     # the operands are lossless
    got = y.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]
    assert fq.fp4q_device_fault() == 0


def _bound(ca, sa_rm, ga, cb, sb_rm, gb, k, fmt, block):
    """G_A G_B sum_k |q_A s_A q_B s_B| through the oracle on magnitude codes."""
    abs_a = ca.cpu().numpy() & 0x77
    abs_b = cb.cpu().numpy() & 0x77
    return oracle.fp4_gemm(abs_a, sa_rm, ga, abs_b, sb_rm, gb, k, fmt, block)


@pytest.mark.parametrize("fmt,gmode", [(E8, "none"), (U4, "compute"), (U4, "none")])
@pytest.mark.parametrize("m,n,k", [(300, 200, 1024), (128, 256, 5120), (129, 1, 192)])
def test_quantized_gaussian_and_activations(fq, fmt, gmode, m, n, k):
    """Weights N(0, 0.02^2) as B; heavy-tailed activations with outlier channels as A."""
    a, _ = workloads.student_t_outliers_bf16(m, k, seed=m + k, n_outlier=min(8, k))
    b = workloads.gaussian_bf16(n, k, 0.02, seed=n + k)
    ca, sa, ga_t, sa_rm = _operands(fq, a, fmt, gmode)
    cb, sb, gb_t, sb_rm = _operands(fq, b, fmt, gmode)
    y = fq.fp4q_gemm(ca, sa, ga_t, cb, sb, gb_t, fmt)
    torch.cuda.synchronize()
    block = 16 if fmt == U4 else 32
    ga = float(ga_t.item()) if ga_t is not None else 1.0
    gb = float(gb_t.item()) if gb_t is not None else 1.0
    want = oracle.fp4_gemm(ca.cpu().numpy(), sa_rm, ga, cb.cpu().numpy(), sb_rm, gb, k, fmt, block)
    mag = _bound(ca, sa_rm, ga, cb, sb_rm, gb, k, fmt, block)
    tol = (k / 16 + 8) * 2.0 ** -24 * mag + 2.0 ** -23 * np.abs(want)
    err = np.abs(y.cpu().numpy().astype(np.float64) - want)
    assert (err <= tol).all(), (float(err.max()), float((err / np.maximum(tol, 1e-300)).max()))
    assert fq.fp4q_device_fault() == 0


def test_gemm_edge_cases(fq):
    import ctypes
    L = fq.lib()
    x = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    c, s, _ = fq.fp4q_quantize_mma(x, E8, 32)
    y = torch.empty((128, 128), dtype=torch.float32, device="cuda")
    # k not a multiple of 64
    assert L.fp4q_gemm(c.data_ptr(), s.data_ptr(), None, 128, c.data_ptr(), s.data_ptr(), None, 128, 32, E8,
                       y.data_ptr(), None) == -2
    # E8M0 takes no per-tensor scale; UE5M3 is not an MMA scale type
    g = torch.ones((1,), dtype=torch.float32, device="cuda")
    assert L.fp4q_gemm(c.data_ptr(), s.data_ptr(), g.data_ptr(), 128, c.data_ptr(), s.data_ptr(), None, 128, 64,
                       E8, y.data_ptr(), None) == -4
    assert L.fp4q_gemm(c.data_ptr(), s.data_ptr(), None, 128, c.data_ptr(), s.data_ptr(), None, 128, 64, 2,
                       y.data_ptr(), None) == -4
    # empty m or n: nothing to do
    assert L.fp4q_gemm(c.data_ptr(), s.data_ptr(), None, 0, c.data_ptr(), s.data_ptr(), None, 128, 64, E8,
                       y.data_ptr(), None) == 0
    # a zero operand gives zero
    yz = fq.fp4q_gemm(c, s, None, c, s, None, E8)
    torch.cuda.synchronize()
    assert not yz.any()
    # the MMA layout rejects other formats and block sizes
    with pytest.raises(Exception):
        fq.fp4q_quantize_mma(x, U4, 32)
    assert fq.fp4q_device_fault() == 0


@pytest.mark.parametrize("fmt", [E8, U4])
@pytest.mark.parametrize("m,n,k", [(4096, 1024, 256), (8192, 2048, 128)])
def test_persistent_many_tiles(fq, fmt, m, n, k):
    """More 128 x 128 tiles than CTAs (256 and 1024 tiles on 148 SMs): both
    accumulator buffers and every barrier phase are reused; lossless operands,
    so every element of Y is checked exactly."""
    rng = np.random.default_rng(m + n + k + fmt)
    a, b = _lossless(m, k, rng, fmt), _lossless(n, k, rng, fmt)
    ca, sa, _, sa_rm = _operands(fq, a, fmt, "none")
    cb, sb, _, sb_rm = _operands(fq, b, fmt, "none")
    y = fq.fp4q_gemm(ca, sa, None, cb, sb, None, fmt)
    torch.cuda.synchronize()
    want = a.cuda().double() @ b.cuda().double().T          # exact: the operands are lossless
    assert torch.equal(y.double(), want)
    block = 16 if fmt == U4 else 32
    rows = np.r_[0:3, m - 3:m]
    sub = oracle.fp4_gemm(ca.cpu().numpy()[rows], sa_rm[rows], 1.0, cb.cpu().numpy(), sb_rm, 1.0, k, fmt, block)
    assert np.array_equal(sub, want.cpu().numpy()[rows])
    assert fq.fp4q_device_fault() == 0
