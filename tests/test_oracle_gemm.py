"""Pins for the oracle's FP4 GEMM consumer, Y = G_A G_B sum_k q_A s_A q_B s_B
(the product of two block-scaled FP4 operands that the QuTLASS kernels of
"Bridging the Gap" s3-4 compute; "Diagnosing FP4 inference", Methodology:
dequantized for the compute).

- lossless operands: values on the E2M1 grid times a power-of-two block scale,
  with every block holding a magnitude of 4 or 6 times its scale, quantize to
  themselves under MXFP4, so the FP4 product equals numpy's A @ B.T exactly;
- against the pinned dequantizer: Y equals dequantize(A) @ dequantize(B).T
  (numpy, fp64) for MXFP4 and for UE4M3 without a per-tensor scale, where every
  dequantized value is exact; with a per-tensor scale the dequantizer rounds
  S = decode(s) G to fp32 first, so the two agree to 2^-22 relative;
- swapping the operands transposes Y; a zero operand gives zero.
"""
import numpy as np
import pytest

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _lossless_mx(rows, k, rng, block=32):
    """Random MXFP4-representable matrix: grid values times 2^e per block, one
    element of each block at +-4 or +-6 times 2^e so the max rule keeps e."""
    nb = k // block
    e = rng.integers(-4, 3, size=(rows, nb))
    q = GRID[rng.integers(0, 8, size=(rows, k))] * np.where(rng.random((rows, k)) < 0.5, -1.0, 1.0)
    q = q.reshape(rows, nb, block)
    q[:, :, 0] = np.where(rng.random((rows, nb)) < 0.5, 4.0, 6.0) * np.where(rng.random((rows, nb)) < 0.5, -1, 1)
    return (q * (2.0 ** e)[..., None]).reshape(rows, k).astype(np.float32)


def test_lossless_operands_give_the_exact_matmul():
    rng = np.random.default_rng(7)
    M, N, K = 24, 20, 256
    a, b = _lossless_mx(M, K, rng), _lossless_mx(N, K, rng)
    ca, sa, ga = oracle.quantize(a, oracle.E8M0, 32)
    cb, sb, gb = oracle.quantize(b, oracle.E8M0, 32)
    assert np.array_equal(oracle.dequantize(ca, sa, ga, M, K, oracle.E8M0, 32), a)   # lossless
    y = oracle.fp4_gemm(ca, sa, ga, cb, sb, gb, K, oracle.E8M0, 32)
    assert np.array_equal(y, a.astype(np.float64) @ b.astype(np.float64).T)


@pytest.mark.parametrize("fmt,block,gmode,rtol", [
    (oracle.E8M0, 32, oracle.G_NONE, 1e-13),
    (oracle.UE4M3, 64, oracle.G_NONE, 1e-13),
    (oracle.UE4M3, 16, oracle.G_COMPUTE, 2.0 ** -22),
    (oracle.UE5M3, 16, oracle.G_NONE, 1e-13),
])
def test_matches_dequantize_then_matmul(fmt, block, gmode, rtol):
    rng = np.random.default_rng(fmt * 10 + block)
    M, N, K = 16, 12, 512
    a = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    b = rng.standard_t(3, size=(N, K)).astype(np.float32)
    ca, sa, ga = oracle.quantize(a, fmt, block, 0, gmode)
    cb, sb, gb = oracle.quantize(b, fmt, block, 0, gmode)
    y = oracle.fp4_gemm(ca, sa, ga, cb, sb, gb, K, fmt, block)
    da = oracle.dequantize(ca, sa, ga, M, K, fmt, block).astype(np.float64)
    db = oracle.dequantize(cb, sb, gb, N, K, fmt, block).astype(np.float64)
    ref = da @ db.T
    scale = np.abs(da) @ np.abs(db).T                       # bound the cancellation in the sums
    assert np.all(np.abs(y - ref) <= rtol * scale + 1e-300)


def test_operand_swap_transposes_and_zero_operand():
    rng = np.random.default_rng(3)
    K = 128
    a = rng.standard_normal((8, K)).astype(np.float32)
    b = rng.standard_normal((5, K)).astype(np.float32)
    ca, sa, ga = oracle.quantize(a, oracle.UE4M3, 16, 0, oracle.G_COMPUTE)
    cb, sb, gb = oracle.quantize(b, oracle.UE4M3, 16, 0, oracle.G_COMPUTE)
    y = oracle.fp4_gemm(ca, sa, ga, cb, sb, gb, K, oracle.UE4M3, 16)
    yt = oracle.fp4_gemm(cb, sb, gb, ca, sa, ga, K, oracle.UE4M3, 16)
    assert np.array_equal(y, yt.T)
    z = np.zeros((3, K), np.float32)
    cz, sz, gz = oracle.quantize(z, oracle.UE4M3, 16, 0, oracle.G_COMPUTE)
    assert (oracle.fp4_gemm(cz, sz, gz, cb, sb, gb, K, oracle.UE4M3, 16) == 0).all()
