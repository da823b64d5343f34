"""Device codecs against the oracle, through the C ABI (fp4q_e2m1_encode_f32 and
fp4q_scale_encode_f32 run the same device functions as the quantize kernel).

Exhaustive over every fp32 bit pattern in the range where the code changes
(E2M1: [2^-4, 16); UE4M3: [2^-12, 2^10); UE5M3: [2^-20, 2^18); E8M0: every
binade edge), both signs for E2M1, plus a strided sweep of all other finite
patterns, zeros, subnormals and infinities.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import microscaling_fp4_quantization_block_b200 as m
    return m


def _bits(lo: float, hi: float):
    a = int(np.array([lo], np.float32).view(np.uint32)[0])
    b = int(np.array([hi], np.float32).view(np.uint32)[0])
    return a, b


def _gpu_e2m1_nibbles(fq, bits_u32: np.ndarray) -> np.ndarray:
    n = bits_u32.size
    n2 = n + (n & 1)
    src = np.zeros(n2, np.uint32)
    src[:n] = bits_u32
    r = torch.from_numpy(src.view(np.int32)).cuda().view(torch.float32)
    packed = fq.fp4q_e2m1_encode_f32(r).cpu().numpy()
    return oracle.unpack_nibbles(packed[None, :])[0][:n]


def _oracle_e2m1(bits_u32: np.ndarray) -> np.ndarray:
    return oracle.e2m1_encode(bits_u32.view(np.float32))


CHUNK = 1 << 26


def _sweep(lo, hi, step=1):
    for a in range(lo, hi, CHUNK * step):
        yield np.arange(a, min(hi, a + CHUNK * step), step, dtype=np.uint64).astype(np.uint32)


def test_e2m1_exhaustive_active_range(fq):
    lo, hi = _bits(2.0 ** -4, 16.0)
    for sign in (0, 0x80000000):
        for b in _sweep(lo, hi):
            b = b | np.uint32(sign)
            g = _gpu_e2m1_nibbles(fq, b)
            o = _oracle_e2m1(b)
            bad = np.nonzero(g != o)[0]
            assert bad.size == 0, (hex(int(b[bad[0]])), g[bad[0]], o[bad[0]])


def test_e2m1_strided_everything_else(fq):
    inf = 0x7F800000
    for sign in (0, 0x80000000):
        b = np.concatenate([np.arange(0, inf + 1, 4099, dtype=np.uint64).astype(np.uint32),
                            np.arange(0, 4096, dtype=np.uint32),                 # zeros, subnormals
                            np.array([inf, inf - 1], np.uint32)])
        b = b | np.uint32(sign)
        g = _gpu_e2m1_nibbles(fq, b)
        o = _oracle_e2m1(b)
        bad = np.nonzero(g != o)[0]
        assert bad.size == 0, (hex(int(b[bad[0]])), g[bad[0]], o[bad[0]])


def _gpu_scale(fq, bits_u32, fmt):
    s = torch.from_numpy(bits_u32.view(np.int32)).cuda().view(torch.float32)
    return fq.fp4q_scale_encode_f32(s, fmt).cpu().numpy()


def _oracle_scale(bits_u32, fmt):
    v = bits_u32.view(np.float32)
    if fmt == 1:
        return oracle.ue4m3_encode_array(v)
    if fmt == 2:
        return oracle.ue5m3_encode_array(v)
    return np.array([oracle.e8m0_from_amax(float(x)) for x in v], np.uint8)


@pytest.mark.parametrize("fmt,lo,hi", [(1, 2.0 ** -12, 2.0 ** 10), (2, 2.0 ** -20, 2.0 ** 18)])
def test_ue_scale_exhaustive_active_range(fq, fmt, lo, hi):
    a, b = _bits(lo, hi)
    for bits in _sweep(a, b):
        g = _gpu_scale(fq, bits, fmt)
        o = _oracle_scale(bits, fmt)
        bad = np.nonzero(g != o)[0]
        assert bad.size == 0, (fmt, hex(int(bits[bad[0]])), g[bad[0]], o[bad[0]])


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_scale_strided_everything_else(fq, fmt):
    inf = 0x7F800000
    bits = np.concatenate([np.arange(0, inf + 1, 65537, dtype=np.uint64).astype(np.uint32),
                           np.arange(0, 4096, dtype=np.uint32), np.array([inf], np.uint32)])
    if fmt == 0:
        # every binade edge of E8M0 and its neighbours
        edges = (np.arange(0, 255, dtype=np.uint64) << 23).astype(np.int64)
        near = (edges[:, None] + np.arange(-2, 3)[None, :]).ravel()
        bits = np.concatenate([bits, near[(near >= 0) & (near <= inf)].astype(np.uint32)])
    g = _gpu_scale(fq, bits, fmt)
    o = _oracle_scale(bits, fmt)
    bad = np.nonzero(g != o)[0]
    assert bad.size == 0, (fmt, hex(int(bits[bad[0]])), g[bad[0]], o[bad[0]])
