"""Gaussian model of the block-quantization MSE and its three-term split.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

"Finer is better? Limits of micro-scaling formats in LLMs", Theoretical
framework: for weights drawn from N(0, sigma^2) the per-tensor MSE of block
quantization splits into (1) the error of the non-max elements, (2) the error
of the block maximum, which is not zero because the scale itself is quantized,
and (3) the error of zero-rounded blocks, whose maximum falls below the
smallest representable scale so that every element becomes 0.  The page gives
no formula; this module derives it from first principles:

* Block of b i.i.d. X ~ N(0, s^2); M = max |X_i| has density
  f_M(m) = b * 2 phi(m) * F(m)^(b-1), with F(m) = P(|X| < m) = 2 Phi(m) - 1.
* Given M = m the scale S(m) is a deterministic function of m (the format's
  "max" rule), the maximum's error is (m - Q_S(m))^2, and the other b-1
  elements are i.i.d. |X| < m, whose expected error is
  (2 / F(m)) * int_0^m (x - Q_S(x))^2 phi(x) dx.
* If S(m) = 0 the whole block is zero: error m^2 + (b-1) E[X^2 | |X| < m].
* Per element, each term is (1/b) * E_M[block term].  The integrals over x are
  closed-form Gaussian moments on each quantization cell; the integral over m
  is Gauss-Legendre on pieces between the points where S(m) or the cell of
  the maximum changes, so every integrand is smooth on its piece.

Scale rules (the same readings as the oracle): E8M0 S = 2^(floor(log2 m) - 2);
UE4M3 / UE5M3 S = decode(nearest code to m / (6 G)) * G, 0 below the smallest
code's half-way point.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import ndtr

E8M0, UE4M3, UE5M3 = 0, 1, 2

# E2M1 magnitudes and the boundaries between their rounding cells, in units of S.
_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_EDGES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _fp8_unsigned_values(exp_bits: int, bias: int, last_code: int) -> np.ndarray:
    """Finite non-negative values of an unsigned 3-mantissa-bit float, by code."""
    vals = []
    for c in range(last_code + 1):
        e, m = c >> 3, c & 7
        vals.append(m * 2.0 ** (1 - bias - 3) if e == 0 else (1 + m / 8) * 2.0 ** (e - bias))
    return np.array(vals)


UE4M3_VALUES = _fp8_unsigned_values(4, 7, 0x7E)    # 0 .. 448, smallest non-zero 2^-9
UE5M3_VALUES = _fp8_unsigned_values(5, 15, 0xFE)   # 0 .. 114688, smallest non-zero 2^-17


class _Normal:
    def __init__(self, sigma: float):
        self.s = float(sigma)

    def pdf(self, x):
        x = np.asarray(x, float)
        return np.exp(-0.5 * (x / self.s) ** 2) / (self.s * math.sqrt(2 * math.pi))

    def cdf(self, x):
        return ndtr(np.asarray(x, float) / self.s)

    def moment(self, a, b, q):
        """int_a^b (x - q)^2 phi(x) dx, elementwise, for finite 0 <= a <= b."""
        a = np.asarray(a, float)
        b = np.asarray(b, float)
        s2 = self.s * self.s
        pa, pb = self.pdf(a), self.pdf(b)
        i0 = self.cdf(b) - self.cdf(a)                 # int phi
        i1 = s2 * (pa - pb)                            # int x phi
        i2 = s2 * i0 + s2 * (a * pa - b * pb)          # int x^2 phi
        return i2 - 2.0 * q * i1 + q * q * i0


def _quantized_magnitude(m, S):
    """Q_S(m) for m >= 0 and S > 0 (ties have zero probability here)."""
    r = np.asarray(m, float) / S
    idx = np.searchsorted(_EDGES, r, side="left")
    return _GRID[idx] * S


def _partial_error(norm: _Normal, m, S):
    """int_0^m (x - Q_S(x))^2 phi(x) dx for an array of m (S > 0)."""
    m = np.asarray(m, float)
    lo_edges = np.concatenate([[0.0], _EDGES]) * S
    hi_edges = np.concatenate([_EDGES, [np.inf]]) * S
    total = np.zeros_like(m)
    for lo, hi, g in zip(lo_edges, hi_edges, _GRID):
        upper = np.minimum(hi, m)
        inside = upper > lo
        if np.any(inside):
            total += np.where(inside, norm.moment(np.full_like(m, lo), np.maximum(upper, lo), g * S), 0.0)
    return total


def _scale_pieces(fmt: int, G: float, m_lo: float, m_hi: float):
    """[(a, b, S)] covering [m_lo, m_hi] with the block scale S constant on each."""
    pieces = []
    if fmt == E8M0:
        n = math.floor(math.log2(m_lo))
        while 2.0 ** n < m_hi:
            a, b = max(2.0 ** n, m_lo), min(2.0 ** (n + 1), m_hi)
            if b > a:
                pieces.append((a, b, 2.0 ** (n - 2)))
            n += 1
        return pieces
    vals = UE4M3_VALUES if fmt == UE4M3 else UE5M3_VALUES
    mids = 0.5 * (vals[1:] + vals[:-1]) * 6.0 * G        # m where the code steps up
    bounds = np.concatenate([[0.0], mids, [np.inf]])
    for c in range(len(vals)):
        a, b = max(bounds[c], m_lo), min(bounds[c + 1], m_hi)
        if b > a:
            pieces.append((a, b, vals[c] * G))
    return pieces


def three_terms(fmt: int, block: int, sigma: float, G: float = 1.0, nodes: int = 48):
    """Expected per-element squared error split as (non-max, max, zero-rounded)."""
    norm = _Normal(sigma)
    b = int(block)
    m_lo, m_hi = sigma * 1e-7, sigma * 14.0
    xg, wg = np.polynomial.legendre.leggauss(nodes)
    t_nonmax = t_max = t_zero = 0.0
    for a, c, S in _scale_pieces(fmt, G, m_lo, m_hi):
        cuts = [a, c]
        if S > 0:
            cuts += [e * S for e in _EDGES if a < e * S < c]
        # keep pieces short relative to sigma so the polynomial rule stays exact
        cuts = sorted(set(cuts))
        fine = []
        for lo, hi in zip(cuts[:-1], cuts[1:]):
            k = max(1, int(math.ceil((hi - lo) / (0.25 * sigma))))
            fine += [lo + (hi - lo) * i / k for i in range(k)]
        fine.append(cuts[-1])
        for lo, hi in zip(fine[:-1], fine[1:]):
            m = 0.5 * (hi - lo) * xg + 0.5 * (hi + lo)
            w = 0.5 * (hi - lo) * wg
            F = 2.0 * norm.cdf(m) - 1.0
            dens = 2.0 * norm.pdf(m)
            if S == 0.0:
                second = norm.moment(np.zeros_like(m), m, 0.0)       # int_0^m x^2 phi
                t_zero += np.sum(w * dens * (F ** (b - 1) * m * m + (b - 1) * F ** (b - 2) * 2.0 * second))
            else:
                emax = (m - _quantized_magnitude(m, S)) ** 2
                t_max += np.sum(w * dens * F ** (b - 1) * emax)
                t_nonmax += np.sum(w * dens * (b - 1) * F ** (b - 2) * 2.0 * _partial_error(norm, m, S))
    return float(t_nonmax), float(t_max), float(t_zero)


def total_mse(fmt: int, block: int, sigma: float, G: float = 1.0) -> float:
    return float(sum(three_terms(fmt, block, sigma, G)))
