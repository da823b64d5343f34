"""Shared test helpers: CUDA-path runs through the C ABI, oracle runs on the same
bytes, and the comparison rules.

Comparison rules (the parity bar):
* unrotated path: codes, scales, G and dequantized values bit-exact; per-block
  MSE and the four tensor terms within 2e-6 relative (fp32 block sums on the GPU
  against fp64 in the oracle);
* rotated path: the GPU rotates in fp32 butterflies, the oracle densely in fp64,
  so y may differ by the butterfly's rounding.  A scale byte may differ only in
  a block whose exact maximum lies within that rounding bound of a scale
  boundary; a code may differ only by one grid step, only where the exact y / S
  lies within the bound of an E2M1 rounding threshold; at most 1e-6 of the
  codes may differ.  MSE (GPU codes, both sides) within 1e-5 relative.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg
import torch

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
EDGES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
UE4M3_VALUES = np.array([oracle.ue4m3_decode(c) for c in range(127)], np.float64)
UE5M3_VALUES = np.array([oracle.ue5m3_decode(c) for c in range(255)], np.float64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def gpu_run(fq, x: torch.Tensor, fmt: int, block: int, rot: int, gmode: int, gval: float | None = None,
            want_mse: bool = True, want_deq: bool = True):
    """Run the CUDA path on a CPU bf16 tensor; returns numpy results."""
    xd = x.cuda()
    rows, cols = x.shape
    gs = None
    if gmode == 2:
        gs = torch.tensor([gval], dtype=torch.float32, device="cuda")
    codes, scales, gs = fq.fp4q_quantize(xd, fmt, block, rot, gmode, gscale=gs)
    out = {}
    gptr = gs if fmt != 0 else None
    if want_deq:
        out["deq32"] = fq.fp4q_dequantize(codes, scales, gptr, rows, cols, fmt, block, 0, torch.float32)
        out["deqbf"] = fq.fp4q_dequantize(codes, scales, gptr, rows, cols, fmt, block, 0, torch.bfloat16)
    if want_mse:
        out["bm"], out["terms"] = fq.fp4q_block_mse(xd, codes, scales, gptr, fmt, block, rot)
    torch.cuda.synchronize()
    res = {}
    for k, v in out.items():
        v = v.cpu()
        res[k] = v.view(torch.int16).numpy().view(np.uint16) if v.dtype == torch.bfloat16 else v.numpy()
    res["codes"] = codes.cpu().numpy()
    res["scales"] = scales.cpu().numpy()
    res["G"] = float(gs.item()) if gs is not None else 1.0
    return res


def oracle_run(xb: np.ndarray, fmt: int, block: int, rot: int, gmode: int, gval: float | None = None,
               want_mse: bool = True, want_deq: bool = True):
    rows, cols = xb.shape
    codes, scales, G = oracle.quantize(xb, fmt, block, rot, gmode, 1.0 if gval is None else gval)
    res = {"codes": codes, "scales": scales, "G": G}
    if want_deq:
        d = oracle.dequantize(codes, scales, G, rows, cols, fmt, block, 0)
        res["deq32"] = d
        res["deqbf"] = oracle.f32_to_bf16_bits(d)
    if want_mse:
        res["bm"], res["terms"] = oracle.block_mse(xb, codes, scales, G, fmt, block, rot)
    return res


def assert_exact(g, o, what=("codes", "scales", "deq32", "deqbf")):
    assert np.float32(g["G"]).view(np.uint32) == np.float32(o["G"]).view(np.uint32), (g["G"], o["G"])
    for k in what:
        if k not in g:
            continue
        a, b = g[k], o[k]
        if a.dtype == np.float32:
            a, b = a.view(np.uint32), b.view(np.uint32)
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{k}: {len(bad)} mismatches, first at {bad[:5].tolist()}: "
                                 f"gpu {a[tuple(bad[0])]} oracle {b[tuple(bad[0])]}")


def assert_mse_close(g_bm, g_terms, o_bm, o_terms, rtol):
    assert np.allclose(g_bm.astype(np.float64), o_bm, rtol=rtol, atol=1e-30), \
        np.max(np.abs(g_bm - o_bm) / np.maximum(np.abs(o_bm), 1e-30))
    for i in range(4):
        assert abs(g_terms[i] - o_terms[i]) <= rtol * abs(o_terms[0]) + 1e-300, (i, g_terms, o_terms)


# ----------------------------------------------------------------------------- rotated path
def exact_rotation(xf: np.ndarray, k: int):
    """fp64 y = H x / sqrt(k) per run of k, and a bound on the fp32 butterfly's
    error for each output: (log2 k + 2) * 2^-24 * sum|x| / sqrt(k) per run."""
    H = scipy.linalg.hadamard(k).astype(np.float64)
    xs = xf.astype(np.float64).reshape(-1, k)
    y = (xs @ H.T) / np.sqrt(k)
    l1 = np.abs(xs).sum(1, keepdims=True) / np.sqrt(k)
    bound = (np.log2(k) + 2) * 2.0 ** -24 * l1 * np.ones_like(y)
    return y.reshape(xf.shape), bound.reshape(xf.shape)


def _scale_values(fmt, codes, G):
    if fmt == 0:
        return np.array([oracle.e8m0_decode(int(c)) for c in range(256)], np.float64)[codes]
    table = UE4M3_VALUES if fmt == 1 else UE5M3_VALUES
    return (table[np.minimum(codes, len(table) - 1)] * np.float64(G)).astype(np.float32).astype(np.float64)


def check_rotated(g, o, xf: np.ndarray, fmt, block, rot, max_frac=1e-6, max_scale_frac=2e-5):
    """Apply the rotated-path rule; returns (n_code_mismatch, n_scale_mismatch).

    * G: may differ from the oracle's only through the tensor maximum, by the
      butterfly's error bound carried through amax / 2688.
    * A scale byte may differ only in a block whose exact maximum lies within
      the butterfly's error bound of a scale boundary.  At most
      max_scale_frac of the blocks (plus one) may differ: a differing byte
      needs m / 6G within a relative distance d of one of the 8 UE4M3 rounding
      midpoints per octave (1 power of two per octave for E8M0), which for
      log-uniform maxima is a fraction 8 * 2d / ln 2 = 23 d of the blocks;
      with y off by up to ~4 fp32 ulps and G by up to 2, d <= 6 * 2^-24 and
      the fraction is <= 8e-6.  The default 2e-5 leaves a factor of 2.5.
    * Every code is compared.  In a block whose scale byte agrees, against the
      oracle's code; in a block whose byte differs, against the code the oracle
      gives for the GPU's own scale byte and G.  A code may differ only by one
      grid step, in sign-agreeing pairs, where the exact y / S lies within the
      error bound of an E2M1 threshold, and at most max_frac of the codes
      (plus one) may differ.
    """
    rows, cols = xf.shape
    y, bound = exact_rotation(xf, rot)
    G = o["G"]
    # per-tensor scale: both sides may differ only through the maximum itself
    if not np.float32(g["G"]) == np.float32(G):
        assert abs(g["G"] - G) <= (bound.max() / 2688.0) * 2 + 2 ** -22 * G, (g["G"], G)
    gs, os_ = g["scales"].astype(np.int64), o["scales"].astype(np.int64)
    yb = y.reshape(rows, cols // block, block)
    bb = bound.reshape(rows, cols // block, block).max(-1)
    m = np.abs(yb).max(-1)
    scale_bad = gs != os_
    n_scale_bad = int(scale_bad.sum())
    if n_scale_bad:
        r, c = np.nonzero(scale_bad)
        for rr, cc in zip(r, c):
            mm, tol = m[rr, cc], bb[rr, cc] + 2 ** -22 * m[rr, cc]
            if fmt == 0:
                p = 2.0 ** np.round(np.log2(mm))
                assert abs(mm - p) <= tol, ("E8M0 scale differs away from a power of two", rr, cc, mm)
            else:
                table = UE4M3_VALUES if fmt == 1 else UE5M3_VALUES
                mids = 0.5 * (table[1:] + table[:-1]) * 6.0 * g["G"]
                assert np.min(np.abs(mids - mm)) <= tol + 2 ** -21 * mm, ("UE scale differs", rr, cc, mm)
    assert n_scale_bad <= max_scale_frac * scale_bad.size + 1, (n_scale_bad, scale_bad.size)
    gn = oracle.unpack_nibbles(g["codes"]).reshape(rows, cols // block, block).astype(np.int64)
    on = oracle.unpack_nibbles(o["codes"]).reshape(rows, cols // block, block).astype(np.int64)
    S_blk = _scale_values(fmt, os_, G)
    if n_scale_bad:
        # the oracle's codes for the GPU's own scale bytes (and G), used where the bytes differ
        rc = oracle.quantize_with_scales(np.ascontiguousarray(xf, np.float32), g["scales"], g["G"], fmt,
                                         block, rot)
        rn = oracle.unpack_nibbles(rc).reshape(rows, cols // block, block).astype(np.int64)
        on = np.where(scale_bad[..., None], rn, on)
        S_blk = np.where(scale_bad, _scale_values(fmt, gs, g["G"]), S_blk)
    diff = gn != on
    n_diff = int(diff.sum())
    if n_diff:
        S = S_blk[..., None] * np.ones_like(yb)
        idx = np.nonzero(diff)
        q = np.abs(yb[idx]) / S[idx]
        qb = bound.reshape(rows, cols // block, block)[idx] / S[idx] + 2 ** -21 * q
        near = np.min(np.abs(q[:, None] - EDGES[None, :]), axis=1) <= qb
        assert near.all(), ("code differs away from a rounding threshold", q[~near][:5])
        step = np.abs((gn[idx] & 7) - (on[idx] & 7))
        assert (step <= 1).all() and ((gn[idx] & 8) == (on[idx] & 8)).all()
    assert n_diff <= max_frac * rows * cols + 1, (n_diff, rows * cols)
    return n_diff, n_scale_bad
