"""fp4q_tensor_amax_batched through the C ABI: the maxima of many tensors in
one pass ("Finer is better?", Results: the per-tensor scale of UE4M3 needs the
tensor maximum first; a model's weight pass takes it for every projection).
Each slot equals the single-tensor call's maximum bit for bit, and the oracle's
maximum (exactly unrotated; within the butterfly's bound rotated), for batches
that mix empty, one-row, ragged and multi-tile tensors, more than one launch's
worth of tensors, strided slots, and both slot modes."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _helpers import bf16_bits, exact_rotation

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _tensors(rot, count, seed):
    unit = max(rot, 8)
    shapes = [(0, 4 * unit), (1, unit), (3, 8 * unit), (33, 2 * unit), (257, 16 * unit), (5, 1024 if rot <= 128 else unit)]
    xs = []
    for i in range(count):
        r, c = shapes[i % len(shapes)]
        x, _ = workloads.student_t_outliers_bf16(r, c, seed=seed + i, n_outlier=min(8, c)) if r else (
            torch.zeros((0, c), dtype=torch.bfloat16), None)
        xs.append(x.cuda())
    return xs


def _want(x, rot):
    xf = oracle.bf16_bits_to_f32(bf16_bits(x.cpu()))
    if xf.size == 0:
        return 0.0, 0.0
    if rot == 0:
        return float(np.abs(xf).max()), 0.0
    y, bound = exact_rotation(xf, rot)
    return float(np.abs(y).max()), float(bound.max())


@pytest.mark.parametrize("rot", [0, 16, 32, 128])
@pytest.mark.parametrize("count", [1, 7, 40])
def test_batch_equals_single_calls_and_oracle(fq, rot, count):
    xs = _tensors(rot, count, seed=100 * rot + count)
    got = fq.fp4q_tensor_amax_batched(xs, rot)
    single = [fq.fp4q_tensor_amax(x, rot).item() if x.numel() else 0.0 for x in xs]
    torch.cuda.synchronize()
    got = got.cpu().numpy()
    for i, x in enumerate(xs):
        assert got[i] == np.float32(single[i]), (i, got[i], single[i])
        want, bound = _want(x, rot)
        assert abs(float(got[i]) - want) <= bound + 2 ** -23 * want, (i, got[i], want)


@pytest.mark.parametrize("rot", [0, 32])
def test_overwrite_and_accumulate_modes_and_strided_slots(fq, rot):
    xs = _tensors(rot, 9, seed=7 + rot)
    single = torch.tensor([fq.fp4q_tensor_amax(x, rot).item() if x.numel() else 0.0 for x in xs])
    # slots every other float, as [amax, G] pairs
    pairs = torch.full((len(xs), 2), 1e30, dtype=torch.float32, device="cuda")
    import ctypes
    L = fq.lib()
    n = len(xs)
    arr = lambda t, v: (t * n)(*v)
    st = L.fp4q_tensor_amax_batched(n, arr(ctypes.c_void_p, [x.data_ptr() for x in xs]),
                                    arr(ctypes.c_int64, [x.shape[0] for x in xs]),
                                    arr(ctypes.c_int64, [x.shape[1] for x in xs]), rot,
                                    arr(ctypes.c_void_p, [pairs[i].data_ptr() for i in range(n)]), 0,
                                    torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0
    assert torch.equal(pairs[:, 0].cpu(), single) and (pairs[:, 1] == 1e30).all()
    # accumulate: a larger value in place is kept, a smaller one is raised
    acc = torch.zeros(n, dtype=torch.float32, device="cuda")
    acc[0] = 1e30
    fq.fp4q_tensor_amax_batched(xs, rot, amax=acc, accumulate=True)
    torch.cuda.synchronize()
    assert acc[0].item() == np.float32(1e30)
    assert torch.equal(acc[1:].cpu(), single[1:])
    # the same tensors twice into one accumulating slot each: unchanged
    fq.fp4q_tensor_amax_batched(xs, rot, amax=acc, accumulate=True)
    torch.cuda.synchronize()
    assert torch.equal(acc[1:].cpu(), single[1:])


def test_weight_pass_layer_shapes(fq):
    """One Qwen2.5-14B layer's seven projections (275 M elements) in one call,
    against the single-tensor calls."""
    xs = [workloads.gaussian_bf16(t.rows, t.cols, 0.02, seed=50 + i, device="cuda")
          for i, t in enumerate(workloads.QWEN25_14B_LAYER)]
    for rot in (0, 32):
        got = fq.fp4q_tensor_amax_batched(xs, rot)
        single = [fq.fp4q_tensor_amax(x, rot).item() for x in xs]
        torch.cuda.synchronize()
        assert got.cpu().tolist() == single
