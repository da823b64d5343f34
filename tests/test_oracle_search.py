"""Pins for the oracle's MSE-optimised block scales.

The pages ("Bridging the Gap Between Promise and Performance for Microscaling
FP4 Quantization", technical summary s3, MR-GPTQ item 2) only say that block
scales are chosen to minimise the squared reconstruction error instead of by
the max rule.  The reading pinned here: candidates are the max-rule code s0,
then s0+1 .. s0+above, then s0-1 .. s0-below, codes outside the finite range
skipped; a candidate wins only with a strictly smaller error.

- hand-worked blocks (tests/golden/scale_search_blocks.json): the byte chosen
  for several windows and the squared error of every candidate, by hand;
- a window of width 0 is the max rule itself, bit for bit;
- invariants on random tensors: the chosen byte lies in the window, its error
  is no larger than that of any code in the window (each quantized on its own
  with the given-scale quantizer) and widening the window never raises a
  block's error;
- brute force on small random blocks: the error of every candidate from
  numpy's IEEE division and a nearest-point search over the E2M1 grid.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = json.load(open(os.path.join(HERE, "golden", "scale_search_blocks.json")))
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
LAST = {oracle.E8M0: 0xFE, oracle.UE4M3: 0x7E, oracle.UE5M3: 0xFE}


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _decode_scale(fmt: int, c: int, G: float) -> np.float32:
    if fmt == oracle.E8M0:
        return np.float32(oracle.e8m0_decode(c))
    dec = oracle.ue4m3_decode(c) if fmt == oracle.UE4M3 else oracle.ue5m3_decode(c)
    return np.float32(np.float64(dec) * np.float64(G))


def _sse_of(x, scales, G, fmt, block):
    """Per-block squared error of x quantized with the given scale bytes."""
    codes = oracle.quantize_with_scales(x, scales, G, fmt, block)
    bm, _ = oracle.block_mse(x, codes, scales, G, fmt, block)
    return bm * block


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=[c["name"] for c in GOLDEN["cases"]])
def test_hand_worked_blocks(case):
    fmt, block = case["fmt"], case["block"]
    x = np.array([case["x"]], np.float32)
    # the hand-computed error of every candidate the case lists
    for code, sse in case["sse"].items():
        got = _sse_of(x, np.array([[int(code)]], np.uint8), 1.0, fmt, block)
        assert got[0, 0] == sse, (code, got[0, 0], sse)
    for below, above, want in case["expect"]:
        codes, scales, G = oracle.quantize_search(x, fmt, block, 0, oracle.G_NONE, 1.0, below, above)
        assert int(scales[0, 0]) == want, (below, above, int(scales[0, 0]), want)
        assert np.array_equal(codes, oracle.quantize_with_scales(x, scales, 1.0, fmt, block))


@pytest.mark.parametrize("fmt,block,gmode,rot", [
    (oracle.E8M0, 32, oracle.G_NONE, 0),
    (oracle.UE4M3, 16, oracle.G_COMPUTE, 0),
    (oracle.UE4M3, 64, oracle.G_NONE, 32),
    (oracle.UE5M3, 8, oracle.G_NONE, 0),
])
def test_empty_window_is_the_max_rule(fmt, block, gmode, rot):
    x = _bf16_bits(workloads.gaussian_bf16(24, 256, 0.02, seed=11))
    a = oracle.quantize(x, fmt, block, rot, gmode)
    b = oracle.quantize_search(x, fmt, block, rot, gmode, 1.0, 0, 0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


@pytest.mark.parametrize("fmt,block,gmode,sigma", [
    (oracle.E8M0, 32, oracle.G_NONE, 0.02),
    (oracle.UE4M3, 16, oracle.G_COMPUTE, 0.02),
    (oracle.UE4M3, 16, oracle.G_NONE, 0.005),      # many zero-rounded blocks without G
    (oracle.UE5M3, 32, oracle.G_NONE, 0.02),
])
def test_window_invariants(fmt, block, gmode, sigma):
    x = _bf16_bits(workloads.gaussian_bf16(32, 512, sigma, seed=5))
    below, above = 2, 1
    c0, s0, G = oracle.quantize(x, fmt, block, 0, gmode)
    c1, s1, G1 = oracle.quantize_search(x, fmt, block, 0, gmode, 1.0, below, above)
    assert G1 == G
    d = s1.astype(np.int64) - s0.astype(np.int64)
    assert ((d >= -below) & (d <= above)).all()
    err = _sse_of(x, s1, G, fmt, block)
    assert (err <= _sse_of(x, s0, G, fmt, block)).all()
    for delta in range(-below, above + 1):
        cand = s0.astype(np.int64) + delta
        ok = (cand >= 0) & (cand <= LAST[fmt])
        e = _sse_of(x, np.clip(cand, 0, LAST[fmt]).astype(np.uint8), G, fmt, block)
        assert (err[ok] <= e[ok]).all(), delta
    # strictly better somewhere: the search does something on real-looking data
    assert (s1 != s0).any()
    # a wider window never raises a block's error
    _, s2, _ = oracle.quantize_search(x, fmt, block, 0, gmode, 1.0, below + 2, above + 1)
    assert (_sse_of(x, s2, G, fmt, block) <= err).all()


def _nearest_code(r: np.ndarray) -> np.ndarray:
    d = np.abs(np.abs(r.astype(np.float64))[..., None] - GRID)
    cand = d == d.min(-1, keepdims=True)
    even = cand & (np.arange(8) % 2 == 0)
    return np.where(even.any(-1), even.argmax(-1), cand.argmax(-1))


@pytest.mark.parametrize("fmt,block", [(oracle.E8M0, 32), (oracle.UE4M3, 8), (oracle.UE5M3, 16)])
def test_brute_force_small_blocks(fmt, block):
    rng = np.random.default_rng(2024 + fmt)
    rows = 40
    y = (rng.standard_t(3, size=(rows, block)) * 0.01).astype(np.float32)
    below, above = 3, 2
    _, s0, _ = oracle.quantize(y, fmt, block, 0, oracle.G_NONE)
    _, s1, _ = oracle.quantize_search(y, fmt, block, 0, oracle.G_NONE, 1.0, below, above)
    for r in range(rows):
        first = int(s0[r, 0])
        order = [first] + [first + j for j in range(1, above + 1)] + [first - j for j in range(1, below + 1)]
        best, best_err = None, None
        for c in order:
            if c < 0 or c > LAST[fmt]:
                continue
            S = _decode_scale(fmt, c, 1.0)
            if S == 0:
                v = np.zeros(block)
            else:
                q = (np.float32(y[r]) / S).astype(np.float32)       # IEEE fp32 division
                v = (GRID[_nearest_code(q)] * np.where(np.signbit(q), -1.0, 1.0) * np.float64(S))
                v = v.astype(np.float32).astype(np.float64)
            e = float(np.sum((y[r].astype(np.float64) - v) ** 2))
            if best is None or e < best_err:
                best, best_err = c, e
        assert int(s1[r, 0]) == best, (r, int(s1[r, 0]), best)


def test_rejects_bad_windows():
    x = np.zeros((1, 32), np.float32)
    with pytest.raises(ValueError):
        oracle.quantize_search(x, oracle.E8M0, 32, 0, oracle.G_NONE, 1.0, -1, 0)
    with pytest.raises(ValueError):
        oracle.quantize_search(x, oracle.E8M0, 32, 0, oracle.G_NONE, 1.0, 0, 17)
