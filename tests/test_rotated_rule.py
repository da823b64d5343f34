"""The rotated-path comparison rule itself (tests/_helpers.check_rotated), on the
CPU: a stand-in for the GPU's result is made by rotating in fp32 butterflies
(the GPU's kind of arithmetic) and quantizing that with the oracle; the rule
must accept it and must reject mistakes planted in it.

The rule ("Bridging the Gap", s3.1: block-wise Hadamard rotation fused with
quantization; the rotated values differ between an fp32 butterfly and the
oracle's fp64 rotation by rounding only): a scale byte may differ only where the
exact block maximum sits within the butterfly's error bound of a scale
boundary, and only in a small fraction of the blocks; every code is compared,
against the oracle's code for the GPU's own scale byte where the bytes differ;
a code may differ by one grid step only next to an E2M1 threshold.
"""
import numpy as np
import pytest

import oracle
import workloads
from _helpers import bf16_bits, check_rotated

E8, U4 = 0, 1
NONE, COMP, GIVEN = 0, 1, 2


def _fwht_f32(xf: np.ndarray, k: int) -> np.ndarray:
    """Sylvester-order fast Walsh-Hadamard transform of each run of k, every
    add and the final scaling rounded to fp32."""
    y = xf.astype(np.float32).reshape(-1, k).copy()
    h = 1
    while h < k:
        y = y.reshape(-1, k // (2 * h), 2, h)
        a = y[:, :, 0, :].copy()
        b = y[:, :, 1, :].copy()
        y[:, :, 0, :] = a + b
        y[:, :, 1, :] = a - b
        y = y.reshape(-1, k)
        h *= 2
    return (y * np.float32(1.0 / np.sqrt(k))).reshape(xf.shape)


def _stand_in(xf, fmt, block, rot, gmode):
    """The oracle's quantizer applied to fp32-butterfly-rotated values."""
    y32 = _fwht_f32(xf, rot)
    codes, scales, G = oracle.quantize(y32, fmt, block, 0, gmode)
    return {"codes": codes, "scales": scales, "G": G}


@pytest.mark.parametrize("rot", [16, 32, 128])
@pytest.mark.parametrize("fmt,block,gmode", [(E8, 32, NONE), (U4, 16, COMP), (U4, 16, NONE)])
def test_fp32_butterfly_passes(rot, fmt, block, gmode):
    x, _ = workloads.student_t_outliers_bf16(64, 2048, seed=rot + block)
    xf = oracle.bf16_bits_to_f32(bf16_bits(x))
    g = _stand_in(xf, fmt, block, rot, gmode)
    o = dict(zip(("codes", "scales", "G"), oracle.quantize(xf, fmt, block, rot, gmode)))
    check_rotated(g, o, xf, fmt, block, rot)


def _fixture(rot=32):
    x, _ = workloads.student_t_outliers_bf16(32, 1024, seed=9)
    xf = oracle.bf16_bits_to_f32(bf16_bits(x))
    o = dict(zip(("codes", "scales", "G"), oracle.quantize(xf, U4, 16, rot, COMP)))
    return xf, o


def test_rejects_code_two_steps_off():
    xf, o = _fixture()
    g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in o.items()}
    nib = oracle.unpack_nibbles(g["codes"]).reshape(-1)
    i = int(np.nonzero((nib & 7) == 2)[0][0])            # a code of magnitude 1.0
    byte = g["codes"].reshape(-1)
    byte[i // 2] = (byte[i // 2] & (0x0F if i & 1 else 0xF0)) | ((nib[i] + 2) << (4 if i & 1 else 0))
    with pytest.raises(AssertionError):
        check_rotated(g, o, xf, U4, 16, 32)


def test_rejects_code_one_step_off_away_from_a_threshold():
    xf, o = _fixture()
    g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in o.items()}
    y, _ = __import__("_helpers").exact_rotation(xf, 32)
    S = np.array([oracle.ue4m3_decode(int(c)) for c in o["scales"].reshape(-1)]) * o["G"]
    q = np.abs(y.reshape(-1, 16)) / S[:, None]
    nib = oracle.unpack_nibbles(g["codes"]).reshape(-1)
    # an element with q = 1.0 +- 0.1: code 2, far from the thresholds 0.75 and 1.25
    i = int(np.nonzero((np.abs(q.reshape(-1) - 1.0) < 0.1) & ((nib & 7) == 2))[0][0])
    byte = g["codes"].reshape(-1)
    byte[i // 2] = (byte[i // 2] & (0x0F if i & 1 else 0xF0)) | ((nib[i] + 1) << (4 if i & 1 else 0))
    with pytest.raises(AssertionError):
        check_rotated(g, o, xf, U4, 16, 32)


def test_rejects_scale_byte_away_from_a_boundary():
    xf, o = _fixture()
    g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in o.items()}
    g["scales"].reshape(-1)[5] += 1
    with pytest.raises(AssertionError):
        check_rotated(g, o, xf, U4, 16, 32)


def _tie_tensor(rows):
    """Rows whose single spike 25.5 rotates (k = 16) to |y| = 6.375 everywhere:
    m / 6 = 1.0625, the midpoint of the UE4M3 values 1.0 (0x38) and 1.125
    (0x39); the oracle takes the even code 0x38."""
    x = np.zeros((rows, 16), np.float32)
    x[:, 0] = 25.5
    return x


def test_scale_tie_is_accepted_and_its_codes_are_compared():
    xf = _tie_tensor(1)
    o = dict(zip(("codes", "scales", "G"), oracle.quantize(xf, U4, 16, 16, NONE)))
    assert int(o["scales"][0, 0]) == 0x38
    # the other side of the tie: scale 0x39 with the oracle's codes for it
    s = np.array([[0x39]], np.uint8)
    g = {"codes": oracle.quantize_with_scales(xf, s, 1.0, U4, 16, 16), "scales": s, "G": 1.0}
    assert check_rotated(g, o, xf, U4, 16, 16) == (0, 1)
    # the same scale byte with one code of the block changed: rejected
    bad = dict(g, codes=g["codes"].copy())
    bad["codes"][0, 3] ^= 0x02
    with pytest.raises(AssertionError):
        check_rotated(bad, o, xf, U4, 16, 16)


def test_rejects_too_many_scale_ties():
    xf = _tie_tensor(64)
    o = dict(zip(("codes", "scales", "G"), oracle.quantize(xf, U4, 16, 16, NONE)))
    s = np.full((64, 1), 0x39, np.uint8)
    g = {"codes": oracle.quantize_with_scales(xf, s, 1.0, U4, 16, 16), "scales": s, "G": 1.0}
    with pytest.raises(AssertionError):
        check_rotated(g, o, xf, U4, 16, 16)
    # within the allowance when the bound is lifted
    check_rotated(g, o, xf, U4, 16, 16, max_scale_frac=1.0)


def test_rejects_a_global_scale_off_by_more_than_the_bound():
    xf, o = _fixture()
    g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in o.items()}
    g["G"] = float(np.float32(o["G"]) * np.float32(1.001))
    with pytest.raises(AssertionError):
        check_rotated(g, o, xf, U4, 16, 32)
