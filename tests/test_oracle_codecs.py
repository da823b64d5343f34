"""Pins for the oracle's number-format codecs (E2M1, E8M0, UE4M3, UE5M3, bf16).

Each check compares the oracle with something other than itself: the format
facts the pages state (tests/golden), torch's own float8 / bf16 conversions
(a library opinion), hand-listed expected codes at the rounding boundaries,
and brute-force searches over the whole code table.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _next_up(x):
    return np.nextafter(np.float32(x), np.float32(np.inf), dtype=np.float32)


def _next_down(x):
    return np.nextafter(np.float32(x), np.float32(-np.inf), dtype=np.float32)


# ----------------------------------------------------------------------------- E2M1
def test_e2m1_grid_points_are_fixed_points():
    grid = _load("e2m1_grid.json")["magnitudes"]
    for i, g in enumerate(grid):
        assert oracle.e2m1_encode([g])[0] == i
        assert oracle.e2m1_encode([-g])[0] == 8 | i
        assert oracle.e2m1_decode(i) == g
        assert oracle.e2m1_decode(8 | i) == -g


def test_e2m1_ties_go_to_even_code():
    for value, code in _load("e2m1_grid.json")["ties"]:
        assert oracle.e2m1_encode([value])[0] == code, value
        assert oracle.e2m1_encode([-value])[0] == 8 | code, value


def test_e2m1_one_ulp_off_each_tie_goes_to_nearer_neighbour():
    ties = _load("e2m1_grid.json")["ties"]
    grid = _load("e2m1_grid.json")["magnitudes"]
    for value, _ in ties:
        lo = max(i for i, g in enumerate(grid) if g < value)
        hi = min(i for i, g in enumerate(grid) if g > value)
        assert oracle.e2m1_encode([_next_down(value)])[0] == lo
        assert oracle.e2m1_encode([_next_up(value)])[0] == hi


def test_e2m1_saturates_at_six():
    vals = np.array([6.0, _next_up(6.0), 7.0, 8.0, 1e30, np.inf], np.float32)
    assert (oracle.e2m1_encode(vals) == 7).all()
    assert (oracle.e2m1_encode(-vals) == 15).all()


def test_e2m1_sign_of_zero_is_kept():
    assert oracle.e2m1_encode([0.0])[0] == 0x0
    assert oracle.e2m1_encode([-0.0])[0] == 0x8
    assert oracle.e2m1_encode([-0.1])[0] == 0x8
    assert oracle.e2m1_encode([np.float32(-1e-40)])[0] == 0x8


def test_e2m1_matches_brute_force_on_a_dense_sample():
    """Brute force: decode every one of the 8 magnitude codes and pick the one at
    the smallest fp64 distance; an exact tie picks the even code."""
    rng = np.random.default_rng(5)
    pts = [rng.uniform(0, 8, 200_000).astype(np.float32),
           (2.0 ** rng.uniform(-30, 10, 50_000)).astype(np.float32)]
    for value, _ in _load("e2m1_grid.json")["ties"]:
        b = np.float32(value).view(np.uint32)
        pts.append((b + np.arange(-64, 65, dtype=np.int64)).astype(np.uint32).view(np.float32))
    a = np.concatenate(pts)
    grid = np.array(_load("e2m1_grid.json")["magnitudes"])
    dist = np.abs(a.astype(np.float64)[:, None] - grid[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # even code among equals if present, else the single nearest one
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    assert (oracle.e2m1_encode(a) == pick).all()
    assert (oracle.e2m1_encode(-a) == (pick | 8)).all()


def test_e2m1_is_monotone_over_bit_patterns():
    # every fp32 in [0, 8): codes never decrease as the value grows
    lo = 0
    hi = int(np.float32(8.0).view(np.uint32))
    step = 997
    bits = np.arange(lo, hi, step, dtype=np.uint64).astype(np.uint32)
    codes = oracle.e2m1_encode(bits.view(np.float32)).astype(int)
    assert (np.diff(codes) >= 0).all()


# ----------------------------------------------------------------------------- E8M0
def test_e8m0_decode_matches_torch_table():
    codes = torch.arange(255, dtype=torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).float().numpy()
    got = np.array([oracle.e8m0_decode(int(c)) for c in codes], np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert math.isnan(oracle.e8m0_decode(255))


@pytest.mark.parametrize("k", [-120, -20, -7, -1, 0, 1, 3, 10, 100])
def test_e8m0_scale_steps_at_powers_of_two(k):
    m = np.float32(2.0 ** k)
    assert oracle.e8m0_from_amax(float(m)) == k - 2 + 127
    assert oracle.e8m0_from_amax(float(_next_down(m))) == k - 3 + 127
    assert oracle.e8m0_from_amax(float(np.float32(1.75) * m)) == k - 2 + 127


def test_e8m0_block_max_lands_in_top_binade():
    """With S = 2^(floor(log2 m) - 2) the scaled maximum lies in [4, 8): the
    E2M1 top binade (codes 4 and 6 of magnitude 4 and 6)."""
    rng = np.random.default_rng(0)
    m = (2.0 ** rng.uniform(-100, 100, 20000)).astype(np.float32)
    for v in m[:2000]:
        S = oracle.e8m0_decode(oracle.e8m0_from_amax(float(v)))
        assert 4.0 <= float(v) / S < 8.0


def test_e8m0_extremes():
    assert oracle.e8m0_from_amax(0.0) == 0
    assert oracle.e8m0_from_amax(float(np.float32(1e-45))) == 0        # clamps at 2^-127
    assert oracle.e8m0_from_amax(float(np.finfo(np.float32).max)) == 127 + 125
    assert oracle.e8m0_from_amax(float("inf")) == 255
    assert oracle.e8m0_decode(0) == 2.0 ** -127


# ----------------------------------------------------------------------------- UE4M3
def test_ue4m3_decode_matches_torch_e4m3fn():
    codes = torch.arange(127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.ue4m3_decode(int(c)) for c in codes], np.float32)
    assert np.array_equal(got, ref)
    assert math.isnan(oracle.ue4m3_decode(0x7F))


def test_ue4m3_range_matches_pages():
    c = _load("format_constants.json")
    assert oracle.ue4m3_decode(1) == 2.0 ** c["ue4m3_min_nonzero_log2"]["value"]
    assert oracle.ue4m3_decode(0x7E) == 448.0


def test_ue4m3_encode_matches_torch_cast_in_range():
    """torch's fp32 -> float8_e4m3fn cast rounds to nearest even; it is a valid
    third opinion for every non-negative value below 464 (448 + half an ulp)."""
    rng = np.random.default_rng(1)
    vals = [(2.0 ** rng.uniform(-14, 8.85, 300_000)).astype(np.float32)]
    table = np.array([oracle.ue4m3_decode(c) for c in range(127)], np.float64)
    mids = ((table[1:] + table[:-1]) / 2).astype(np.float32)
    for d in range(-3, 4):               # every midpoint and its 3 neighbours each side
        vals.append((mids.view(np.uint32).astype(np.int64) + d).astype(np.uint32).view(np.float32))
    v = np.concatenate(vals)
    v = v[(v >= 0) & (v < 464)]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.ue4m3_encode_array(v), ref)


def test_ue4m3_saturates_and_rounds_small_values_to_zero():
    for s in [448.0, 463.9, 464.0, 500.0, 1e30]:
        assert oracle.ue4m3_encode(s) == 0x7E
    half_min = 2.0 ** -10
    assert oracle.ue4m3_encode(half_min) == 0                        # tie to even code 0
    assert oracle.ue4m3_encode(float(_next_up(half_min))) == 1
    assert oracle.ue4m3_encode(float(_next_down(half_min))) == 0
    assert oracle.ue4m3_encode(0.0) == 0


# ----------------------------------------------------------------------------- UE5M3
def test_ue5m3_layout():
    c = _load("format_constants.json")
    assert oracle.ue5m3_decode(1) == 2.0 ** c["ue5m3_min_nonzero_log2"]["value"]
    assert oracle.ue5m3_decode(8) == 2.0 ** -14                       # smallest normal, bias 15
    assert oracle.ue5m3_decode(0xFE) == 1.75 * 2.0 ** 16
    assert math.isnan(oracle.ue5m3_decode(0xFF))
    vals = [oracle.ue5m3_decode(c) for c in range(255)]
    assert all(b > a for a, b in zip(vals, vals[1:]))
    for code in range(255):
        assert oracle.ue5m3_encode(vals[code]) == code


def test_ue5m3_encode_brute_force():
    table = np.array([oracle.ue5m3_decode(c) for c in range(255)], np.float64)
    rng = np.random.default_rng(3)
    v = (2.0 ** rng.uniform(-19, 17, 20000)).astype(np.float32)
    mids = ((table[1:] + table[:-1]) / 2).astype(np.float32)     # exact ties
    v = np.concatenate([v, mids])
    d = np.abs(table[None, :] - v.astype(np.float64)[:, None])
    cand = d == d.min(axis=1, keepdims=True)
    even = cand & (np.arange(255)[None, :] % 2 == 0)
    want = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    assert np.array_equal(oracle.ue5m3_encode_array(v), want.astype(np.uint8))
    for big in (114688.0, 2.0 ** 17, 1e30):          # saturation to the largest finite code
        assert oracle.ue5m3_encode(big) == 0xFE


# ----------------------------------------------------------------------------- bf16
def test_bf16_widening_matches_torch():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_bits_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(2)
    b = rng.integers(0, 1 << 32, 1_000_000, dtype=np.uint64).astype(np.uint32)
    b = np.concatenate([b, (b & 0xFFFF0000) | 0x8000])              # exact ties
    x = b.view(np.float32)
    x = x[np.isfinite(x)]
    got = oracle.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
