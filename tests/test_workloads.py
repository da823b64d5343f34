"""The seeded input generators: deterministic, right shapes, right laws."""
import numpy as np
import torch

import workloads


def test_gaussian_is_seeded_and_scaled():
    a = workloads.gaussian_bf16(256, 512, 0.02, seed=0)
    b = workloads.gaussian_bf16(256, 512, 0.02, seed=0)
    c = workloads.gaussian_bf16(256, 512, 0.02, seed=1)
    assert a.dtype == torch.bfloat16 and a.shape == (256, 512)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert abs(a.float().std().item() - 0.02) < 0.0005


def test_student_t_outlier_channels():
    x, ch = workloads.student_t_outliers_bf16(4096, 512, seed=3)
    assert x.shape == (4096, 512) and len(ch) == 8
    xf = x.float()
    mask = torch.ones(512, dtype=torch.bool)
    mask[ch] = False
    # unit std for t_3 / sqrt(3) is a slow, heavy-tailed estimate; check a robust scale instead
    mad = xf[:, mask].abs().median().item()
    mad_out = xf[:, ch].abs().median().item()
    assert 30 < mad_out / mad < 70
    x2, ch2 = workloads.student_t_outliers_bf16(4096, 512, seed=3)
    assert torch.equal(x, x2) and torch.equal(ch, ch2)


def test_layer_sigmas_jitter():
    s = workloads.layer_sigmas(48, 0.02, 0.5, seed=0)
    assert len(s) == 48 and min(s) >= 0.01 and max(s) <= 0.03
    assert s == workloads.layer_sigmas(48, 0.02, 0.5, seed=0)


def test_named_shapes():
    assert [(t.rows, t.cols) for t in workloads.QWEN25_7B_MLP] == [(18944, 3584), (18944, 3584),
                                                                   (3584, 18944)]
    n = sum(t.rows * t.cols for t in workloads.QWEN25_14B_LAYER)
    assert n == 275_251_200
    assert workloads.SWEEP_BLOCKS == (256, 128, 64, 32, 16, 8)
