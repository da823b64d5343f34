"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no quantization arithmetic: it only draws random tensors
and names their shapes.  It is the one module that both the CUDA path's tests
and benchmark and the CPU oracle's tests draw inputs from.

Distributions (the pages measure on real Qwen2.5 / Llama weights and WikiText
activations, which are not available here; these synthetic tensors stand in):

* weights: i.i.d. N(0, sigma^2) ("Finer is better?", Theoretical framework:
  pre-trained weights closely follow a zero-mean Normal law);
* activations: Student-t with nu = 3, scaled to unit standard deviation, with a
  few outlier channels multiplied by a large factor ("Bridging the Gap",
  technical summary s2: heavy-tailed, Laplace-like activations; "Diagnosing
  FP4 inference", outlier analysis of the Max/P99.9 ratio);
* whole-model weight passes: one sigma per layer, jittered uniformly.

Every tensor is drawn in fp32 by torch's seeded generator on the requested
device and rounded to bf16 (round to nearest even) with ``Tensor.to``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_bf16(rows: int, cols: int, sigma: float, seed: int, device="cpu") -> torch.Tensor:
    """rows x cols bf16 tensor with i.i.d. N(0, sigma^2) entries."""
    g = _gen(seed, device)
    x = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    return (x * sigma).to(torch.bfloat16)


def gaussian_f32(rows: int, cols: int, sigma: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32) * sigma


def student_t_outliers_bf16(rows: int, cols: int, seed: int, nu: int = 3, n_outlier: int = 8,
                            factor: float = 50.0, device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """Activations [tokens, channels]: t_nu / sqrt(nu / (nu - 2)) (unit std), with
    ``n_outlier`` seeded channels multiplied by ``factor``.  Returns (x, channels)."""
    g = _gen(seed, device)
    z = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros((rows, cols), device=device, dtype=torch.float32)
    for _ in range(nu):
        w = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
        chi2 += w * w
    t = z / torch.sqrt(chi2 / nu)
    t = t / (nu / (nu - 2)) ** 0.5
    cg = _gen(seed + 7919, "cpu")
    channels = torch.randperm(cols, generator=cg)[:n_outlier].sort().values
    t[:, channels.to(device)] *= factor
    return t.to(torch.bfloat16), channels


def layer_sigmas(n_layers: int, base: float, jitter: float, seed: int) -> List[float]:
    """sigma_l = base * U(1 - jitter, 1 + jitter), one per layer."""
    g = _gen(seed, "cpu")
    u = torch.rand((n_layers,), generator=g, dtype=torch.float64)
    return [float(base * (1.0 - jitter + 2.0 * jitter * v)) for v in u]


# --------------------------------------------------------------------------- named workloads
@dataclasses.dataclass(frozen=True)
class Tensor2D:
    name: str
    rows: int
    cols: int


# Qwen2.5-7B MLP projections (weights [out, in]).
QWEN25_7B_MLP = (Tensor2D("gate", 18944, 3584), Tensor2D("up", 18944, 3584),
                 Tensor2D("down", 3584, 18944))
QWEN25_7B_SIGMAS = (0.005, 0.02, 0.05)

# Qwen2.5-14B decoder layer: the seven projections, 48 layers.
QWEN25_14B_LAYER = (Tensor2D("q", 5120, 5120), Tensor2D("k", 1024, 5120), Tensor2D("v", 1024, 5120),
                    Tensor2D("o", 5120, 5120), Tensor2D("gate", 13824, 5120),
                    Tensor2D("up", 13824, 5120), Tensor2D("down", 5120, 13824))
QWEN25_14B_LAYERS = 48

SWEEP_SHAPE = (4096, 4096)
SWEEP_BLOCKS = (256, 128, 64, 32, 16, 8)
SWEEP_SIGMAS = (0.002, 0.005, 0.01, 0.02)

ACT_SHAPE = (8192, 5120)
ACT_ROTATIONS = (0, 16, 32, 128)

MX_SMALL_SHAPE = (1024, 1024)

# The five workloads by name (sizes as stated; the benchmark and tests pick from these).
WORKLOADS: Dict[str, dict] = {
    "mxfp4_gaussian_1024x1024": dict(shape=MX_SMALL_SHAPE, sigma=0.02, seed=0, fmt="mxfp4", block=32,
                                    rot=0),
    "nvfp4_qwen25_7b_mlp": dict(tensors=QWEN25_7B_MLP, sigmas=QWEN25_7B_SIGMAS, fmt="nvfp4", block=16,
                                rot=0, gmode="compute"),
    "ue4m3_block_sweep_4096x4096": dict(shape=SWEEP_SHAPE, blocks=SWEEP_BLOCKS, sigmas=SWEEP_SIGMAS),
    "rotated_activations_8192x5120": dict(shape=ACT_SHAPE, rotations=ACT_ROTATIONS),
    "qwen25_14b_weight_pass": dict(layer=QWEN25_14B_LAYER, layers=QWEN25_14B_LAYERS, base_sigma=0.02,
                                   jitter=0.5, rotations=(0, 32)),
}


def nvfp4_mlp_tensors(device="cpu", seed: int = 1000):
    """The nine (sigma x {gate, up, down}) Qwen2.5-7B MLP weights, as (name, tensor)."""
    out = []
    for si, sigma in enumerate(QWEN25_7B_SIGMAS):
        for ti, t in enumerate(QWEN25_7B_MLP):
            out.append((f"{t.name}_s{sigma}", gaussian_bf16(t.rows, t.cols, sigma, seed + 10 * si + ti,
                                                             device)))
    return out
