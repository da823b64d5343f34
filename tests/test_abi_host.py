"""The C ABI without a GPU: the library loads, exports every entry point that
include/fp4q.h declares, and rejects bad arguments on the host before it
enqueues anything (these calls never reach the CUDA runtime)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4q.h")


@pytest.fixture(scope="module")
def fp4q():
    from microscaling_fp4_quantization_block_b200 import build
    build.build()
    import microscaling_fp4_quantization_block_b200 as m
    return m


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FP4Q_API\s+[\w\s\*]+?\b(fp4q_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ["fp4q_quantize", "fp4q_dequantize", "fp4q_block_mse", "fp4q_block_mse_workspace_size",
                 "fp4q_tensor_amax", "fp4q_status_string", "fp4q_version"]:
        assert must in names


def test_every_declared_symbol_is_exported(fp4q):
    out = subprocess.run(["nm", "-D", "--defined-only", fp4q.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (fp4q_\w+)", out))
    assert set(_declared()) <= exported
    lib = ctypes.CDLL(fp4q.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name)


def test_version_and_status_strings(fp4q):
    assert fp4q.fp4q_version() == 1
    for st in range(0, -7, -1):
        s = fp4q.fp4q_status_string(st)
        assert s and s != "unknown status"
    assert fp4q.fp4q_status_string(-99) == "unknown status"


# Fake device addresses: never dereferenced, because every call below is
# rejected by the host-side checks that run before any launch.
A32 = 0x7F0000000000          # 32-byte aligned
A4 = A32 + 4                  # 4-byte aligned only


def test_quantize_rejects_bad_arguments(fp4q):
    q = fp4q.lib().fp4q_quantize
    E8, U4, U5 = 0, 1, 2
    NONE, COMP, GIVEN = 0, 1, 2
    assert q(A32, -1, 64, E8, 32, 0, NONE, A32, A32, None, None) == -2          # negative rows
    assert q(A32, 4, 48, E8, 32, 0, NONE, A32, A32, None, None) == -2           # 48 % 32
    assert q(A32, 4, 64, E8, 16, 128, NONE, A32, A32, None, None) == -2         # 64 % 128
    assert q(A32, 4, 64, 3, 16, 0, NONE, A32, A32, None, None) == -4            # unknown format
    assert q(A32, 4, 64, U4, 12, 0, NONE, A32, A32, None, None) == -4           # block not pow2
    assert q(A32, 4, 512, U4, 512, 0, NONE, A32, A32, None, None) == -4         # block > 256
    assert q(A32, 4, 512, U4, 4, 0, NONE, A32, A32, None, None) == -4           # block < 8
    assert q(A32, 4, 64, U4, 16, 64, NONE, A32, A32, None, None) == -4          # rot 64 unsupported
    assert q(A32, 4, 64, U4, 16, 0, 7, A32, A32, None, None) == -4              # unknown gmode
    assert q(A32, 4, 64, E8, 32, 0, COMP, A32, A32, A32, None) == -4            # MX has no tensor scale
    assert q(A32, 4, 64, U4, 16, 0, GIVEN, A32, A32, None, None) == -1          # gscale needed
    assert q(None, 4, 64, U4, 16, 0, NONE, A32, A32, None, None) == -1
    assert q(A32, 4, 64, U4, 16, 0, NONE, None, A32, None, None) == -1
    assert q(A32, 4, 64, U4, 16, 0, NONE, A32, None, None, None) == -1
    assert q(A32 + 16, 4, 64, U4, 16, 0, NONE, A32, A32, None, None) == -3      # x not 32-aligned
    assert q(A32, 4, 64, U4, 16, 0, NONE, A32 + 8, A32, None, None) == -3
    assert q(A32, 4, 64, U4, 16, 0, NONE, A32, A32 + 8, None, None) == -3       # scales not 16-aligned
    assert q(A32, 4, 64, U4, 16, 0, GIVEN, A32, A32, A32 + 2, None) == -3
    assert q(A32, 1 << 62, 1 << 8, U4, 16, 0, NONE, A32, A32, None, None) == -2  # overflow
    # empty tensors are valid and enqueue nothing without a per-tensor scale
    assert q(None, 0, 64, U4, 16, 0, NONE, None, None, None, None) == 0
    assert q(None, 5, 0, E8, 32, 0, NONE, None, None, None, None) == 0
    assert q(None, 0, 64, U5, 16, 32, GIVEN, None, None, A4, None) == 0


def test_dequantize_and_mse_reject_bad_arguments(fp4q):
    L = fp4q.lib()
    assert L.fp4q_dequantize(A32, A32, None, 4, 64, 1, 16, 0, 2, A32, None) == -4       # bad out dtype
    assert L.fp4q_dequantize(None, A32, None, 4, 64, 1, 16, 0, 0, A32, None) == -1
    assert L.fp4q_dequantize(A32, A32, None, 4, 64, 1, 16, 0, 0, A32 + 16, None) == -3
    assert L.fp4q_dequantize(None, None, None, 0, 64, 1, 16, 0, 0, None, None) == 0
    ws = L.fp4q_block_mse_workspace_size(4, 64, 16)
    assert ws >= 32 and ws % 8 == 0
    assert L.fp4q_block_mse(A32, A32, A32, None, 4, 64, 1, 16, 0, None, A32, A32, ws - 8, None) == -6
    assert L.fp4q_block_mse(A32, A32, A32, None, 4, 64, 1, 16, 0, None, None, A32, ws, None) == -1
    assert L.fp4q_block_mse(A32, A32, A32, None, 4, 64, 1, 16, 0, A32 + 4, A32, A32, ws, None) == -3
    assert L.fp4q_block_mse(A32, A32, A32, None, 4, 60, 1, 16, 0, None, A32, A32, ws, None) == -2
    assert L.fp4q_tensor_amax(A32, 4, 64, 0, None, None) == -1
    assert L.fp4q_tensor_amax(A32, 4, 64, 12, A32, None) == -4
    assert L.fp4q_e2m1_encode_f32(A32, 7, A32, None) == -2                            # odd count
    assert L.fp4q_scale_encode_f32(A32, 8, 9, A32, None) == -4
    assert L.fp4q_e2m1_encode_f32(None, 0, None, None) == 0
    assert L.fp4q_quantize_mse(A32, 4, 64, 1, 16, 0, 0, A32, A32, None, None, None, A32, ws, None) == -1
    assert L.fp4q_quantize_mse(A32, 4, 64, 1, 16, 0, 0, A32, A32, None, None, A32, A32, ws - 8, None) == -6
    assert L.fp4q_quantize_mse(A32, 4, 64, 0, 32, 0, 1, A32, A32, A32, None, A32, A32, ws, None) == -4
    assert L.fp4q_quantize_mse(A32, 4, 64, 1, 16, 0, 0, A32, A32, None, A32 + 8, A32, A32, ws, None) == -3
    assert L.fp4q_global_scale(None, A32, None) == -1
    assert L.fp4q_global_scale(A32 + 2, A32, None) == -3


def test_search_and_outlier_stats_reject_bad_arguments(fp4q):
    L = fp4q.lib()
    qs = L.fp4q_quantize_search
    assert qs(A32, 4, 64, 1, 16, 0, 0, -1, 1, A32, A32, None, None) == -4         # window below 0
    assert qs(A32, 4, 64, 1, 16, 0, 0, 1, 17, A32, A32, None, None) == -4         # window above 16
    assert qs(A32, 4, 48, 0, 32, 0, 0, 1, 1, A32, A32, None, None) == -2          # 48 % 32
    assert qs(A32, 4, 64, 0, 32, 0, 1, 1, 1, A32, A32, A32, None) == -4           # MX has no tensor scale
    assert qs(None, 4, 64, 1, 16, 0, 0, 1, 1, A32, A32, None, None) == -1
    assert qs(A32 + 16, 4, 64, 1, 16, 0, 0, 1, 1, A32, A32, None, None) == -3
    assert qs(None, 0, 64, 1, 16, 0, 0, 3, 2, None, None, None, None) == 0        # empty: nothing enqueued
    ws = L.fp4q_outlier_stats_workspace_size()
    assert ws == 2 * 32768 * 8 + 2 * 256 * 8 + 16
    os_ = L.fp4q_outlier_stats
    assert os_(A32, 4, 60, 0.999, A32, None, A32, ws, None) == -2                 # cols % 8
    assert os_(A32, -1, 64, 0.999, A32, None, A32, ws, None) == -2
    for p in (0.0, -0.1, 1.01, float("nan")):
        assert os_(A32, 4, 64, p, A32, None, A32, ws, None) == -4
    assert os_(A32, 4, 64, 0.999, None, None, A32, ws, None) == -1                # stats
    assert os_(A32, 4, 64, 0.999, A32, None, None, ws, None) == -1                # workspace
    assert os_(None, 4, 64, 0.999, A32, None, A32, ws, None) == -1                # x
    assert os_(A32, 4, 64, 0.999, A32, None, A32, ws - 8, None) == -6
    assert os_(A32 + 8, 4, 64, 0.999, A32, None, A32, ws, None) == -3             # x 16-aligned
    assert os_(A32, 4, 64, 0.999, A32 + 2, None, A32, ws, None) == -3
    assert os_(A32, 4, 64, 0.999, A32, A32 + 2, A32, ws, None) == -3
    assert os_(A32, 4, 64, 0.999, A32, None, A32 + 4, ws, None) == -3


def test_workspace_size_is_bounded(fp4q):
    L = fp4q.lib()
    small = L.fp4q_block_mse_workspace_size(1, 16, 16)
    big = L.fp4q_block_mse_workspace_size(1 << 20, 1 << 14, 16)
    assert small == 32 + 16             # one CTA's partials + the completion counter
    assert big == 4096 * 32 + 16
    assert L.fp4q_block_mse_workspace_size(-1, 16, 16) == 0


def test_binding_refuses_cpu_tensors(fp4q):
    import torch
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fp4q.fp4q_quantize(x, "nvfp4", 16)


def test_gemm_and_mma_layout_reject_bad_arguments(fp4q):
    """fp4q_gemm and fp4q_quantize_mma reject bad arguments before any launch;
    fp4q_mma_scales_size is 512 bytes per (128-row, 4-block) atom."""
    L = fp4q.lib()
    E8, U4, U5 = 0, 1, 2
    assert L.fp4q_mma_scales_size(128, 256, 16) == 512 * 4
    assert L.fp4q_mma_scales_size(129, 256, 16) == 512 * 4 * 2
    assert L.fp4q_mma_scales_size(1, 64, 32) == 512          # 2 block columns pad to one atom
    assert L.fp4q_mma_scales_size(0, 64, 32) == 0
    g = L.fp4q_gemm
    assert g(A32, A32, None, 128, A32, A32, None, 128, 96, E8, A32, None) == -2      # k % 64
    assert g(A32, A32, None, -1, A32, A32, None, 128, 64, E8, A32, None) == -2
    assert g(A32, A32, None, 128, A32, A32, None, 128, 64, U5, A32, None) == -4      # not an MMA scale type
    assert g(A32, A32, A32, 128, A32, A32, None, 128, 64, E8, A32, None) == -4       # E8M0: no tensor scale
    assert g(A32, A32, None, 128, A32, A32, None, 128, 64, E8, None, None) == -1
    assert g(A32, A32, None, 128, A32, A32, None, 128, 64, E8, A32 + 4, None) == -3  # y 16-aligned
    assert g(None, A32, None, 128, A32, A32, None, 128, 64, E8, A32, None) == -1
    assert g(A32 + 8, A32, None, 128, A32, A32, None, 128, 64, E8, A32, None) == -3
    assert g(A32, A32, A32 + 2, 128, A32, A32, None, 128, 64, U4, A32, None) == -3
    assert g(None, None, None, 0, None, None, None, 128, 64, E8, None, None) == 0    # empty: nothing to do
    qm = L.fp4q_quantize_mma
    assert qm(A32, 4, 64, U4, 32, 0, 0, A32, A32, None, None) == -4                 # NVFP4 is block 16
    assert qm(A32, 4, 64, E8, 16, 0, 0, A32, A32, None, None) == -4                 # MXFP4 is block 32
    assert qm(A32, 4, 64, U5, 16, 0, 0, A32, A32, None, None) == -4
    assert qm(A32, 4, 48, E8, 32, 0, 0, A32, A32, None, None) == -2
    assert qm(A32, 4, 64, U4, 16, 0, 0, A32, A32 + 8, None, None) == -3
    assert qm(None, 0, 64, U4, 16, 0, 0, None, None, None, None) == 0
    assert L.fp4q_device_fault(None, 0) == -1


def test_global_scale_search_rejects_bad_arguments(fp4q):
    L = fp4q.lib()
    ws = L.fp4q_global_scale_search_workspace_size()
    assert ws >= 32 + 4096 * 24 * 8
    g = L.fp4q_global_scale_search
    assert g(A32, 4, 64, 0, 32, 0, 1, 1, A32, None, A32, ws, None) == -4       # E8M0: no per-tensor scale
    assert g(A32, 4, 64, 1, 16, 0, 9, 1, A32, None, A32, ws, None) == -4       # below > 8
    assert g(A32, 4, 64, 1, 16, 0, 1, 16, A32, None, A32, ws, None) == -4      # above > 15
    assert g(A32, 4, 60, 1, 16, 0, 1, 1, A32, None, A32, ws, None) == -2
    assert g(A32, 4, 64, 1, 16, 0, 1, 1, None, None, A32, ws, None) == -1
    assert g(A32, 4, 64, 1, 16, 0, 1, 1, A32, None, None, ws, None) == -1
    assert g(A32, 4, 64, 1, 16, 0, 1, 1, A32, None, A32, ws - 8, None) == -6
    assert g(A32, 4, 64, 1, 16, 0, 1, 1, A32 + 2, None, A32, ws, None) == -3
    assert g(A32, 4, 64, 1, 16, 0, 1, 1, A32, A32 + 4, A32, ws, None) == -3
    assert g(A32 + 16, 4, 64, 1, 16, 0, 1, 1, A32, None, A32, ws, None) == -3


def test_batched_amax_rejects_bad_arguments(fp4q):
    L = fp4q.lib()
    f = L.fp4q_tensor_amax_batched

    def arrs(xs, rows, cols, slots):
        n = len(xs)
        return ((ctypes.c_void_p * n)(*xs), (ctypes.c_int64 * n)(*rows), (ctypes.c_int64 * n)(*cols),
                (ctypes.c_void_p * n)(*slots))

    x, r, c, s = arrs([A32, A32], [4, 8], [64, 128], [A32, A32 + 4])
    assert f(-1, x, r, c, 0, s, 0, None) == -2
    assert f(0, None, None, None, 0, None, 0, None) == 0                          # nothing to do
    assert f(2, None, r, c, 0, s, 0, None) == -1
    assert f(2, x, r, c, 0, None, 0, None) == -1
    assert f(2, x, r, c, 12, s, 0, None) == -4                                     # rot 12
    assert f(2, *arrs([A32, A32], [4, 8], [64, 60], [A32, A32 + 4])[:3], 0, s, 0, None) == -2
    assert f(2, *arrs([A32, A32], [4, -8], [64, 64], [A32, A32 + 4])[:3], 0, s, 0, None) == -2
    assert f(2, *arrs([A32, A32], [4, 8], [64, 64], [A32, A32 + 4])[:3], 128, s, 0, None) == -2  # 64 % 128
    xs, rs, cs, ss = arrs([A32, A32 + 16], [4, 8], [64, 128], [A32, A32 + 4])
    assert f(2, xs, rs, cs, 0, ss, 0, None) == -3                                  # x not 32-byte aligned
    xs, rs, cs, ss = arrs([A32, A32], [4, 8], [64, 128], [A32, A32 + 2])
    assert f(2, xs, rs, cs, 0, ss, 0, None) == -3                                  # slot not 4-byte aligned
    xs, rs, cs, ss = arrs([A32, None], [4, 8], [64, 128], [A32, A32 + 4])
    assert f(2, xs, rs, cs, 0, ss, 0, None) == -1                                  # non-empty tensor, no data
    xs, rs, cs, ss = arrs([A32, A32], [4, 8], [64, 128], [A32, None])
    assert f(2, xs, rs, cs, 0, ss, 1, None) == -1


def test_batched_quantizer_rejects_bad_arguments(fp4q):
    L = fp4q.lib()
    f = L.fp4q_quantize_mse_dequantize_batched
    T = fp4q.Fp4qTensor
    ws = L.fp4q_quantize_batch_workspace_size(2)
    assert ws >= 2 * (16 + 4096 * 32) and L.fp4q_quantize_batch_workspace_size(0) == 0

    def batch(*ts):
        return (T * len(ts))(*ts)

    ok = T(A32, 4, 64, A32, A32, A32, A32, None, A32)
    assert f(-1, batch(ok), 1, 16, 0, 3, A32, ws, None) == -2
    assert f(0, None, 1, 16, 0, 3, None, 0, None) == 0                                  # nothing to do
    assert f(2, None, 1, 16, 0, 3, A32, ws, None) == -1
    assert f(2, batch(ok, ok), 1, 16, 0, 3, None, ws, None) == -1
    assert f(2, batch(ok, ok), 1, 32, 0, 3, A32, ws, None) == -4                        # NVFP4 is block 16
    assert f(2, batch(ok, ok), 0, 16, 0, 0, A32, ws, None) == -4                        # MXFP4 is block 32
    assert f(2, batch(ok, ok), 2, 16, 0, 3, A32, ws, None) == -4                        # UE5M3: single calls
    assert f(2, batch(ok, ok), 0, 32, 0, 3, A32, ws, None) == -4                        # E8M0 takes no G
    assert f(2, batch(ok, ok), 1, 16, 12, 3, A32, ws, None) == -4                       # rot 12
    assert f(2, batch(ok, ok), 1, 16, 0, 3, A32, ws - 8, None) == -6
    assert f(2, batch(ok, ok), 1, 16, 0, 3, A32 + 4, ws, None) == -3
    assert f(2, batch(ok, T(A32, 4, 60, A32, A32, A32, A32, None, A32)), 1, 16, 0, 3, A32, ws, None) == -2
    assert f(2, batch(ok, T(A32, 4, 64, A32, A32, None, A32, None, A32)), 1, 16, 0, 3, A32, ws, None) == -1
    assert f(2, batch(ok, T(A32, 4, 64, A32, A32, A32, None, None, A32)), 1, 16, 0, 3, A32, ws, None) == -1
    assert f(2, batch(ok, T(A32, 4, 64, A32, A32, A32, A32, None, None)), 1, 16, 0, 3, A32, ws, None) == -1
    assert f(2, batch(ok, T(A32 + 16, 4, 64, A32, A32, A32, A32, None, A32)), 1, 16, 0, 3, A32, ws, None) == -3
    assert f(2, batch(ok, T(A32, 4, 64, A32 + 16, A32, A32, A32, None, A32)), 1, 16, 0, 3, A32, ws, None) == -3
    assert f(2, batch(ok, T(A32, 4, 64, A32, A32, A32, A32, A32 + 8, A32)), 1, 16, 0, 3, A32, ws, None) == -3
