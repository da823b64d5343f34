"""fp4q_quantize_mse_dequantize_batched through the C ABI: a model layer's
tensors quantized in one launch ("Finer is better?", Theoretical framework:
per-tensor MSE and its three terms; "Diagnosing FP4 inference", Methodology:
quantized, then dequantized for the compute).  Every tensor's codes, scale
bytes, per-tensor scale, dequantized values and per-block MSE equal the
single call's bit for bit; its tensor terms agree to fp64 reassociation (the
batch sums the same squared errors in another grouping); and a small batch
meets the oracle directly (bit-exact unrotated, the rotated-path rule
rotated).  Batches mix empty, one-row, ragged and multi-tile tensors, run
past one launch's 8 tensors, and cover every rotation and scale mode."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits, check_rotated, oracle_run, assert_mse_close

pytestmark = pytest.mark.gpu

E8, U4 = 0, 1
NONE, COMP, GIVEN, FROM_AMAX = 0, 1, 2, 3


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _shapes(rot, count):
    u = max(rot, 32)
    base = [(257, 16 * u), (0, 4 * u), (1, u), (3, 8 * u), (33, 2 * u), (64, 40 * u), (5, 1024 if u <= 1024 else u)]
    return [base[i % len(base)] for i in range(count)]


def _tensors(rot, count, seed):
    xs = []
    for i, (r, c) in enumerate(_shapes(rot, count)):
        if r == 0:
            xs.append(torch.zeros((0, c), dtype=torch.bfloat16, device="cuda"))
        else:
            x, _ = workloads.student_t_outliers_bf16(r, c, seed=seed + i, n_outlier=min(8, c))
            xs.append((x.float() * (0.02 * (1 + i % 3))).to(torch.bfloat16).cuda())
    return xs


def _single(fq, x, fmt, block, rot, gmode, g):
    gs = None
    if gmode == FROM_AMAX:
        gs = g.clone()
    elif gmode == GIVEN:
        gs = g[1:2].clone()
    return fq.fp4q_quantize_mse_dequantize(x, fmt, block, rot, gmode, gscale=gs)


@pytest.mark.parametrize("rot", [0, 16, 32, 128])
@pytest.mark.parametrize("fmt,block,gmode", [(E8, 32, NONE), (U4, 16, FROM_AMAX), (U4, 16, GIVEN), (U4, 16, COMP)])
def test_batch_equals_single_calls(fq, fmt, block, gmode, rot):
    count = 11 if (rot, gmode) == (32, FROM_AMAX) else 7
    xs = _tensors(rot, count, seed=1000 + rot + 10 * gmode)
    gpairs = []
    for x in xs:                                   # [amax, G] per tensor, as the weight pass keeps them
        g = torch.zeros(2, dtype=torch.float32, device="cuda")
        fq.fp4q_tensor_amax(x, rot, amax=g[:1])
        g[1] = 0.75 + 0.25 * len(gpairs)           # a given G for GIVEN mode
        gpairs.append(g)
    if gmode == FROM_AMAX:
        gs = [g.clone() for g in gpairs]
    elif gmode == GIVEN:
        gs = [g[1:2].clone() for g in gpairs]
    else:
        gs = None
    outs = fq.fp4q_quantize_mse_dequantize_batched(xs, fmt, block, rot, gmode, gscales=gs)
    singles = [_single(fq, x, fmt, block, rot, gmode, g) for x, g in zip(xs, gpairs)]
    torch.cuda.synchronize()
    for i, (o, s) in enumerate(zip(outs, singles)):
        for k, name in enumerate(("codes", "scales", "gscale", "y", "block_mse")):
            a, b = o[k], s[k]
            if a is None and b is None:
                continue
            assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                               b.view(torch.uint8) if b.dtype == torch.bfloat16 else b), (i, name)
        t_b, t_s = o[5].cpu().numpy(), s[5].cpu().numpy()
        assert np.allclose(t_b, t_s, rtol=1e-12, atol=0.0), (i, t_b, t_s)


@pytest.mark.parametrize("fmt,block,rot", [(E8, 32, 0), (U4, 16, 0), (U4, 16, 32)])
def test_small_batch_against_oracle(fq, fmt, block, rot):
    xs = _tensors(rot, 4, seed=77 + rot)
    gmode = COMP if fmt == U4 else NONE
    outs = fq.fp4q_quantize_mse_dequantize_batched(xs, fmt, block, rot, gmode)
    torch.cuda.synchronize()
    for x, o in zip(xs, outs):
        if x.numel() == 0:
            assert not o[5].any().item()
            continue
        xb = bf16_bits(x.cpu())
        ref = oracle_run(xb, fmt, block, rot, gmode, want_deq=False)
        g = {"codes": o[0].cpu().numpy(), "scales": o[1].cpu().numpy(),
             "G": float(o[2].item()) if o[2] is not None else 1.0}
        if rot == 0:
            assert np.array_equal(g["codes"], ref["codes"]) and np.array_equal(g["scales"], ref["scales"])
            assert np.float32(g["G"]) == np.float32(ref["G"])
            assert_mse_close(o[4].cpu().numpy(), o[5].cpu().numpy(), ref["bm"], ref["terms"], 2e-6)
        else:
            check_rotated(g, ref, oracle.bf16_bits_to_f32(xb), fmt, block, rot)


def test_empty_batch_and_all_empty_tensors(fq):
    assert fq.fp4q_quantize_mse_dequantize_batched([], "nvfp4", 16) == []
    xs = [torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    g = [torch.tensor([0.0, -1.0], device="cuda") for _ in xs]
    outs = fq.fp4q_quantize_mse_dequantize_batched(xs, "nvfp4", 16, 0, FROM_AMAX, gscales=g)
    torch.cuda.synchronize()
    for o, gg in zip(outs, g):
        assert not o[5].any().item() and gg[1].item() == 1.0


def test_workspace_is_left_zero_and_reusable(fq):
    """Each tensor's completion counter returns to 0, so one zero-filled
    workspace serves repeated calls; the results repeat bit for bit."""
    xs = _tensors(0, 5, seed=5)
    ws = torch.zeros(fq.fp4q_quantize_batch_workspace_size(5), dtype=torch.uint8, device="cuda")
    a = fq.fp4q_quantize_mse_dequantize_batched(xs, "mxfp4", 32, workspace=ws)
    b = fq.fp4q_quantize_mse_dequantize_batched(xs, "mxfp4", 32, workspace=ws)
    torch.cuda.synchronize()
    stride = ws.numel() // 5
    for i in range(5):
        assert not ws[i * stride:i * stride + 16].any().item()
        assert a[i][5].cpu().numpy().tobytes() == b[i][5].cpu().numpy().tobytes()
        assert torch.equal(a[i][0], b[i][0]) and torch.equal(a[i][4], b[i][4])
