"""Pins for the oracle's quantizer and dequantizer.

Brute force on small tensors: every element's code must be a nearest E2M1
point to fp32(y / S) (numpy's IEEE division, the 16 codes enumerated), every
UE4M3 scale the nearest table value to the block maximum over 6 G, every E8M0
scale the power of two that puts the block maximum in [4, 8).  Hand-built
blocks pin the boundaries: the zero-rounding threshold of "Finer is better?"
(Theoretical framework), the power-of-two steps of E8M0 ("Bridging the Gap",
s2, dead zone), the sign of zero, the nibble order, the per-tensor scale.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
UE4M3 = np.array([oracle.ue4m3_decode(c) for c in range(127)], np.float64)


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _nearest_code(r: np.ndarray) -> np.ndarray:
    d = np.abs(np.abs(r.astype(np.float64))[..., None] - GRID)
    cand = d == d.min(-1, keepdims=True)
    even = cand & (np.arange(8) % 2 == 0)
    idx = np.where(even.any(-1), even.argmax(-1), cand.argmax(-1))
    return (idx | (np.signbit(r) * 8)).astype(np.uint8)


def _check_tensor(y: np.ndarray, codes, scales, G, fmt, block):
    """Brute-force check of codes/scales against the rotated-domain values y."""
    rows, cols = y.shape
    nib = oracle.unpack_nibbles(codes).reshape(rows, cols // block, block)
    yb = y.reshape(rows, cols // block, block)
    m = np.abs(yb).max(-1)
    for (r, c), sc in np.ndenumerate(scales):
        if fmt == oracle.E8M0:
            S = np.float32(oracle.e8m0_decode(int(sc)))
            if m[r, c] > 2.0 ** -120:
                assert 4.0 <= m[r, c] / S < 8.0
        else:
            sf = np.float32(m[r, c]) / (np.float32(6.0) * np.float32(G))
            d = np.abs(UE4M3 - float(min(sf, 448.0)))
            best = np.flatnonzero(d == d.min())
            want = best[best % 2 == 0][0] if len(best) > 1 else best[0]
            assert sc == want, (r, c, sf)
            S = np.float32(UE4M3[sc] * np.float64(G))
        if S == 0:
            assert (nib[r, c] == 0).all()
        else:
            q = (yb[r, c].astype(np.float32) / S).astype(np.float32)
            assert np.array_equal(nib[r, c], _nearest_code(q)), (r, c)


CASES = [
    # fmt, block, rot, gmode
    (oracle.E8M0, 32, 0, oracle.G_NONE),
    (oracle.UE4M3, 16, 0, oracle.G_NONE),
    (oracle.UE4M3, 16, 0, oracle.G_COMPUTE),
    (oracle.UE4M3, 8, 0, oracle.G_NONE),
    (oracle.UE4M3, 256, 0, oracle.G_NONE),
    (oracle.E8M0, 64, 0, oracle.G_NONE),
    (oracle.E8M0, 32, 16, oracle.G_NONE),
    (oracle.E8M0, 32, 32, oracle.G_NONE),
    (oracle.UE4M3, 16, 128, oracle.G_COMPUTE),
    (oracle.E8M0, 32, 128, oracle.G_NONE),
]


@pytest.mark.parametrize("fmt,block,rot,gmode", CASES)
@pytest.mark.parametrize("sigma", [0.002, 0.02])
def test_brute_force_small_tensors(fmt, block, rot, gmode, sigma):
    x = workloads.gaussian_bf16(6, 512, sigma, seed=block + rot + gmode)
    xb = _bf16_bits(x)
    codes, scales, G = oracle.quantize(xb, fmt, block, rot, gmode)
    xf = oracle.bf16_bits_to_f32(xb)
    y = oracle.hadamard(xf, rot).reshape(xf.shape) if rot else xf
    if gmode == oracle.G_COMPUTE:
        assert G == np.float32(np.abs(y).max()) / np.float32(2688.0)
        # the block holding the tensor's maximum gets the top UE4M3 code (448)
        r, c = np.unravel_index(np.abs(y).argmax(), y.shape)
        assert scales[r, c // block] == 0x7E
    else:
        assert G == 1.0
    _check_tensor(y, codes, scales, G, fmt, block)


def test_heavy_tailed_activations_brute_force():
    x, ch = workloads.student_t_outliers_bf16(16, 1024, seed=3)
    xb = _bf16_bits(x)
    for fmt, block, rot, gmode in [(oracle.E8M0, 32, 32, 0), (oracle.UE4M3, 16, 16, 1)]:
        codes, scales, G = oracle.quantize(xb, fmt, block, rot, gmode)
        xf = oracle.bf16_bits_to_f32(xb)
        y = oracle.hadamard(xf, rot).reshape(xf.shape)
        _check_tensor(y, codes, scales, G, fmt, block)


def test_given_global_scale_is_used():
    x = _bf16_bits(workloads.gaussian_bf16(4, 64, 0.02, seed=1))
    g = 0.0123
    codes, scales, G = oracle.quantize(x, oracle.UE4M3, 16, 0, oracle.G_GIVEN, g)
    assert G == np.float32(g)
    _check_tensor(oracle.bf16_bits_to_f32(x), codes, scales, G, oracle.UE4M3, 16)


def test_nvfp4_zero_rounding_threshold():
    """A block whose maximum over 6 is at or below half the smallest UE4M3 value
    (2^-10) gets scale 0 and all-zero codes; one bf16 step above, scale 2^-9."""
    at_bits = int(np.array([6 * 2.0 ** -10], np.float32).view(np.uint32)[0] >> 16)   # exact in bf16
    assert at_bits == 0x3BC0
    for bits, want_scale in [(at_bits, 0), (at_bits + 1, 1)]:
        blk = np.zeros((1, 16), np.uint16)
        blk[0, 3] = bits
        blk[0, 5] = bits | 0x8000                      # a negative copy
        blk[0, 7] = 0x3A80                              # 2^-10 * 1: small positive
        codes, scales, _ = oracle.quantize(blk, oracle.UE4M3, 16)
        assert scales[0, 0] == want_scale
        nib = oracle.unpack_nibbles(codes)[0]
        if want_scale == 0:
            assert (nib == 0).all()                     # zero-rounded: plain 0x0 even for negatives
        else:
            assert nib[3] != 0 and nib[5] == (nib[3] | 8)
            assert nib[0] == 0 and nib[1] == 0


def test_e8m0_zero_block_and_powers_of_two():
    blk = np.zeros((1, 64), np.uint16)
    blk[0, 32 + 4] = 0x4000                              # 2.0 in block 1
    codes, scales, _ = oracle.quantize(blk, oracle.E8M0, 32)
    assert scales[0, 0] == 0 and scales[0, 1] == 127 + 1 - 2
    nib = oracle.unpack_nibbles(codes)[0]
    assert (nib[:32] == 0).all()
    assert nib[36] == 6                                   # 2.0 / 2^-1 = 4.0 -> code 6


def test_negative_values_rounding_to_zero_keep_their_sign():
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 4.0
    x[0, 1] = -0.001
    x[0, 2] = 0.001
    codes, scales, _ = oracle.quantize(x, oracle.E8M0, 32)
    nib = oracle.unpack_nibbles(codes)[0]
    assert nib[1] == 0x8 and nib[2] == 0x0 and nib[0] == 6


def test_nibble_order_low_is_even_element():
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1] = 6.0, -1.0                        # S = 1: codes 7 and 0xA
    codes, _, _ = oracle.quantize(x, oracle.E8M0, 32)
    assert codes[0, 0] == 0xA7


def test_grid_values_round_trip_through_dequantize():
    rng = np.random.default_rng(0)
    for fmt, block in [(oracle.E8M0, 32), (oracle.UE4M3, 16)]:
        g = GRID[rng.integers(0, 8, (8, 128))] * rng.choice([-1, 1], (8, 128))
        g[:, ::block] = 6.0                              # every block reaches 6 * S with S = 1
        x = g.astype(np.float32)
        codes, scales, G = oracle.quantize(x, fmt, block)
        v = oracle.dequantize(codes, scales, G, 8, 128, fmt, block)
        assert np.array_equal(v, x)


def test_dequantized_value_is_a_nearest_grid_point():
    x = workloads.gaussian_f32(8, 256, 0.02, seed=4).numpy()
    for fmt, block in [(oracle.E8M0, 32), (oracle.UE4M3, 16)]:
        codes, scales, G = oracle.quantize(x, fmt, block)
        v = oracle.dequantize(codes, scales, G, 8, 256, fmt, block).astype(np.float64)
        S = np.repeat(np.array([[oracle.e8m0_decode(int(s)) if fmt == 0 else UE4M3[s] * G
                                 for s in row] for row in scales]), block, axis=1)
        err = np.abs(x - v)
        cand = np.abs(x[..., None] - np.sign(x)[..., None] * GRID * S[..., None]).min(-1)
        cand2 = np.abs(x[..., None] + np.sign(x)[..., None] * GRID * S[..., None]).min(-1)
        assert (err <= np.minimum(cand, cand2) * (1 + 1e-6) + 1e-30).all()


def test_ragged_and_empty_shapes():
    for rows, cols, block in [(1, 8, 8), (3, 24, 8), (1, 32, 32), (3, 64, 32), (0, 64, 16), (5, 0, 16)]:
        x = workloads.gaussian_bf16(rows, cols, 0.02, seed=rows + cols)
        xb = _bf16_bits(x)
        codes, scales, _ = oracle.quantize(xb, oracle.UE4M3, block, 0, oracle.G_COMPUTE)
        assert codes.shape == (rows, cols // 2) and scales.shape == (rows, cols // block)
        if rows * cols:
            _check_tensor(oracle.bf16_bits_to_f32(xb), codes, scales,
                          oracle.global_scale_from_amax(float(np.abs(oracle.bf16_bits_to_f32(xb)).max())),
                          oracle.UE4M3, block)


def test_rejects_bad_layouts():
    x = np.zeros((2, 48), np.float32)
    with pytest.raises(ValueError):
        oracle.quantize(x, oracle.E8M0, 32)              # 48 % 32
    with pytest.raises(ValueError):
        oracle.quantize(x, oracle.E8M0, 16, 32)           # rotation does not divide cols
    with pytest.raises(ValueError):
        oracle.quantize(x, oracle.E8M0, 16, 0, oracle.G_COMPUTE)   # MX has no tensor scale
    with pytest.raises(ValueError):
        oracle.quantize(x, oracle.UE4M3, 12)
