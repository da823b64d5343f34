"""The benchmark's step does the work it claims: the weight-pass pipeline with
batched amax and batched quantizer calls (what bench.py times) leaves every
output buffer -- codes, scale bytes, [amax, G], dequantized values, per-block
MSE -- bit for bit as the pipeline of one C-ABI call per tensor does, and the
MSE terms to fp64 reassociation, on a small model of the same structure (three
layers of seven projections, four variants), replayed as a CUDA graph too."""
import numpy as np
import pytest
import torch

import bench
import workloads

pytestmark = pytest.mark.gpu

SHAPES = [(64, 512), (16, 512), (16, 512), (64, 512), (96, 512), (96, 512), (64, 1536)]


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import microscaling_fp4_quantization_block_b200 as m
    m.lib()
    return m


def _pipes(fq):
    dev = torch.device("cuda", 0)
    xs = []
    for layer in range(3):
        for t, (r, c) in enumerate(SHAPES):
            xs.append((f"L{layer}.{t}", workloads.gaussian_bf16(r, c, 0.01 * (layer + 1), seed=50 + 8 * layer + t,
                                                               device=dev)))
    items, groups = bench.weight_pass_items(xs, len(SHAPES))
    stream = torch.cuda.Stream(dev)
    a = bench.Pipeline(fq, items, dev, stream, groups=groups)
    b = bench.Pipeline(fq, items, dev, stream, groups=groups, batch_amax=False, batch_quantize=False)
    return items, stream, a, b


def _compare(items, a, b):
    for i in range(len(items)):
        # deq: one buffer per input tensor, rewritten by each variant in turn in both pipelines
        for name in ("codes", "scales", "gscale", "deq", "bm"):
            assert torch.equal(a.bufs[i][name].view(torch.uint8), b.bufs[i][name].view(torch.uint8)), (i, name)
        ta, tb = a.bufs[i]["terms"].cpu().numpy(), b.bufs[i]["terms"].cpu().numpy()
        assert np.allclose(ta, tb, rtol=1e-12, atol=0.0), (i, ta, tb)


def test_batched_step_equals_per_tensor_step(fq):
    items, stream, a, b = _pipes(fq)
    assert any("batched" in fn.__name__ for _, fn, _, _ in a.step_calls)
    with torch.cuda.stream(stream):
        a.step(stream)
        b.step(stream)
    torch.cuda.synchronize()
    _compare(items, a, b)


def test_graph_replay_equals_direct_step(fq):
    items, stream, a, b = _pipes(fq)
    with torch.cuda.stream(stream):
        b.step(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        a.step(stream)
    with torch.cuda.stream(stream):
        g.replay()
        g.replay()
    torch.cuda.synchronize()
    _compare(items, a, b)
