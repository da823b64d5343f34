"""fp4q_block_mse_noalloc (fixed device scratch, no workspace argument) against
fp4q_block_mse (caller workspace) through the C ABI, on two calls in a row.

Collected last on purpose: it must pass both in a fresh process and after
every other GPU test has run in the same process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

RTOL = 2e-6   # the MSE tolerance of the parity tests (fp32 block sums)


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _reference(fq, xd, codes, scales, gs, fmt, block, rot):
    bm, terms = fq.fp4q_block_mse(xd, codes, scales, gs, fmt, block, rot)
    return bm, terms


def _close(a: torch.Tensor, b: torch.Tensor, rtol: float):
    a64, b64 = a.double().cpu().numpy(), b.double().cpu().numpy()
    scale = np.maximum(np.abs(b64), 1e-30)
    return float(np.max(np.abs(a64 - b64) / scale)) if a64.size else 0.0


@pytest.mark.parametrize("fmt,block,rot,gmode,shape", [
    (1, 16, 0, 1, (1000, 4096)),     # NVFP4 b16 with a per-tensor scale, ~1000 partial slots
    (0, 32, 32, 0, (333, 1024)),      # MXFP4 b32, rotated, ragged tile count
])
def test_noalloc_matches_workspace_entry_point_twice(fq, fmt, block, rot, gmode, shape):
    rows, cols = shape
    x = workloads.student_t_outliers_bf16(rows, cols, seed=4242 + rows)[0]
    xd = x.cuda()
    codes, scales, gs = fq.fp4q_quantize(xd, fmt, block, rot, gmode)
    gptr = gs if fmt != 0 else None
    ref_bm, ref_terms = _reference(fq, xd, codes, scales, gptr, fmt, block, rot)

    # outputs allocated up front: the entry point itself allocates nothing
    bm = torch.empty((rows, cols // block), dtype=torch.float32, device="cuda")
    terms = torch.empty((4,), dtype=torch.float64, device="cuda")
    for call in range(2):
        bm.fill_(float("nan"))
        terms.fill_(float("nan"))
        fq.fp4q_block_mse_noalloc(xd, codes, scales, gptr, fmt, block, rot, block_mse=bm, terms=terms)
        torch.cuda.synchronize()
        assert _close(bm, ref_bm, RTOL) <= RTOL, f"call {call}: per-block MSE differs"
        rel = np.abs(terms.cpu().numpy() - ref_terms.cpu().numpy())
        assert (rel <= RTOL * abs(float(ref_terms[0])) + 1e-300).all(), (call, terms, ref_terms)


def test_noalloc_smaller_tensor_after_larger(fq):
    """A small tensor right after a large one: stale partials of the larger
    launch must not leak into the smaller one's terms."""
    big = workloads.gaussian_bf16(2048, 4096, 0.02, seed=1).cuda()
    small = workloads.gaussian_bf16(8, 256, 0.02, seed=2).cuda()
    terms = torch.empty((4,), dtype=torch.float64, device="cuda")
    for x in (big, small):
        codes, scales, gs = fq.fp4q_quantize(x, 1, 16, 0, 1)
        _, ref_terms = _reference(fq, x, codes, scales, gs, 1, 16, 0)
        fq.fp4q_block_mse_noalloc(x, codes, scales, gs, 1, 16, 0, block_mse=None, terms=terms)
        torch.cuda.synchronize()
        rel = np.abs(terms.cpu().numpy() - ref_terms.cpu().numpy())
        assert (rel <= RTOL * abs(float(ref_terms[0])) + 1e-300).all(), (x.shape, terms, ref_terms)


def test_noalloc_rejects_bad_arguments(fq):
    x = workloads.gaussian_bf16(4, 64, 0.02, seed=3).cuda()
    codes, scales, gs = fq.fp4q_quantize(x, 1, 16, 0, 1)
    terms = torch.empty((4,), dtype=torch.float64, device="cuda")
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_block_mse_noalloc(x, codes, scales, gs, 1, 24, 0, terms=terms)     # block not a power of two
    st = fq.lib().fp4q_block_mse_noalloc(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), gs.data_ptr(),
                                         4, 64, 1, 16, 0, None, None, None)
    assert st == -1                                                                  # terms is NULL
