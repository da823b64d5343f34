"""Python binding of libfp4q.so (B200 block-wise microscaling FP4 quantization).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch supplies device memory and streams; each function below has
the name of the C entry point it calls (see include/fp4q.h), takes CUDA
tensors, allocates any output that is not given, checks the returned status
and raises ``Fp4qError`` on failure.  There is no CPU fallback: if the
library is missing, the first call raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp4q.so")

# enums of include/fp4q.h
FP4Q_OK = 0
FP4Q_SCALE_E8M0, FP4Q_SCALE_UE4M3, FP4Q_SCALE_UE5M3 = 0, 1, 2
FP4Q_GLOBAL_NONE, FP4Q_GLOBAL_COMPUTE, FP4Q_GLOBAL_GIVEN, FP4Q_GLOBAL_FROM_AMAX = 0, 1, 2, 3
FP4Q_OUT_BF16, FP4Q_OUT_F32 = 0, 1

_FMT_NAMES = {"e8m0": FP4Q_SCALE_E8M0, "mxfp4": FP4Q_SCALE_E8M0, "ue4m3": FP4Q_SCALE_UE4M3,
              "nvfp4": FP4Q_SCALE_UE4M3, "ue5m3": FP4Q_SCALE_UE5M3}
_GMODE_NAMES = {"none": FP4Q_GLOBAL_NONE, "compute": FP4Q_GLOBAL_COMPUTE, "given": FP4Q_GLOBAL_GIVEN,
                "from_amax": FP4Q_GLOBAL_FROM_AMAX}


class Fp4qError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fp4q_status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m microscaling_fp4_quantization_block_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "fp4q_quantize": (I, [P, I64, I64, I, I, I, I, P, P, P, P]),
        "fp4q_quantize_search": (I, [P, I64, I64, I, I, I, I, I, I, P, P, P, P]),
        "fp4q_outlier_stats": (I, [P, I64, I64, ctypes.c_double, P, P, P, SZ, P]),
        "fp4q_outlier_stats_workspace_size": (SZ, []),
        "fp4q_tensor_amax": (I, [P, I64, I64, I, P, P]),
        "fp4q_tensor_amax_accumulate": (I, [P, I64, I64, I, P, P]),
        "fp4q_tensor_amax_batched": (I, [I, P, P, P, I, P, I, P]),
        "fp4q_quantize_batch_workspace_size": (SZ, [I]),
        "fp4q_quantize_mse_dequantize_batched": (I, [I, P, I, I, I, I, P, SZ, P]),
        "fp4q_global_scale": (I, [P, P, P]),
        "fp4q_dequantize": (I, [P, P, P, I64, I64, I, I, I, I, P, P]),
        "fp4q_block_mse": (I, [P, P, P, P, I64, I64, I, I, I, P, P, P, SZ, P]),
        "fp4q_block_mse_workspace_size": (SZ, [I64, I64, I]),
        "fp4q_block_mse_noalloc": (I, [P, P, P, P, I64, I64, I, I, I, P, P, P]),
        "fp4q_quantize_mse": (I, [P, I64, I64, I, I, I, I, P, P, P, P, P, P, SZ, P]),
        "fp4q_quantize_mse_dequantize": (I, [P, I64, I64, I, I, I, I, P, P, P, P, P, P, P, SZ, P]),
        "fp4q_e2m1_encode_f32": (I, [P, I64, P, P]),
        "fp4q_scale_encode_f32": (I, [P, I64, I, P, P]),
        "fp4q_status_string": (ctypes.c_char_p, [I]),
        "fp4q_version": (I, []),
        "fp4q_device_fault": (I, [P, I]),
        "fp4q_quantize_mma": (I, [P, I64, I64, I, I, I, I, P, P, P, P]),
        "fp4q_mma_scales_size": (ctypes.c_size_t, [I64, I64, I]),
        "fp4q_gemm": (I, [P, P, P, I64, P, P, P, I64, I64, I, P, P]),
        "fp4q_global_scale_search": (I, [P, I64, I64, I, I, I, I, I, P, P, P, ctypes.c_size_t, P]),
        "fp4q_global_scale_search_workspace_size": (ctypes.c_size_t, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raw pointer-level access); loaded on first use and
    raising ImportError if libfp4q.so has not been built."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def _fmt(f) -> int:
    return _FMT_NAMES[f.lower()] if isinstance(f, str) else int(f)


def _gmode(g) -> int:
    return _GMODE_NAMES[g.lower()] if isinstance(g, str) else int(g)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str) -> None:
    if status != FP4Q_OK:
        raise Fp4qError(status, where)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("fp4q tensors must live on a CUDA device")


def fp4q_version() -> int:
    return lib().fp4q_version()


def fp4q_status_string(status: int) -> str:
    return lib().fp4q_status_string(status).decode()


def fp4q_device_fault(clear: bool = False) -> int:
    """The library's device fault word on the current device (0, or 1 after a
    tensor-core kernel gave up a bounded wait); synchronizes the device."""
    out = ctypes.c_uint(0)
    _check(lib().fp4q_device_fault(ctypes.addressof(out), int(bool(clear))), "fp4q_device_fault")
    return int(out.value)


def fp4q_quantize(x: torch.Tensor, fmt, block: int, rot: int = 0, gmode="none",
                  codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                  gscale: Optional[torch.Tensor] = None, stream=None
                  ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """Quantize a 2-D bf16 CUDA tensor; returns (codes, scales, gscale)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    fmt, gmode = _fmt(fmt), _gmode(gmode)
    dev = x.device
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // block if block else 0), dtype=torch.uint8, device=dev)
    if gscale is None and gmode == FP4Q_GLOBAL_FROM_AMAX:
        raise ValueError("from_amax mode reads the tensor maximum from gscale[0]: pass a 2-float gscale")
    if gscale is None and gmode != FP4Q_GLOBAL_NONE:
        gscale = torch.empty((1,), dtype=torch.float32, device=dev)
    if gmode == FP4Q_GLOBAL_FROM_AMAX and gscale.numel() < 2:
        raise ValueError("from_amax mode needs gscale with 2 floats: [amax in, G out]")
    _need_cuda(codes, scales, gscale)
    st = lib().fp4q_quantize(_ptr(x), rows, cols, fmt, block, rot, gmode, _ptr(codes), _ptr(scales),
                            _ptr(gscale), _stream(stream))
    _check(st, "fp4q_quantize")
    return codes, scales, gscale


def fp4q_global_scale_search(x: torch.Tensor, fmt, block: int, rot: int = 0, below: int = 8, above: int = 15,
                             gscale: Optional[torch.Tensor] = None, errors: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None
                             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """MSE-optimised per-tensor scale: returns (gscale [1], errors [below + above + 1])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    dev = x.device
    if gscale is None:
        gscale = torch.empty((1,), dtype=torch.float32, device=dev)
    if errors is None:
        errors = torch.empty((below + above + 1,), dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.empty((lib().fp4q_global_scale_search_workspace_size(),), dtype=torch.uint8, device=dev)
    _need_cuda(gscale, errors, workspace)
    st = lib().fp4q_global_scale_search(_ptr(x), rows, cols, _fmt(fmt), block, rot, below, above, _ptr(gscale),
                                        _ptr(errors), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "fp4q_global_scale_search")
    return gscale, errors


def fp4q_mma_scales_size(rows: int, cols: int, block: int) -> int:
    return int(lib().fp4q_mma_scales_size(rows, cols, block))


def fp4q_quantize_mma(x: torch.Tensor, fmt, block: int, rot: int = 0, gmode="none",
                      codes: Optional[torch.Tensor] = None, scales_mma: Optional[torch.Tensor] = None,
                      gscale: Optional[torch.Tensor] = None, stream=None
                      ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """fp4q_quantize with the scale bytes in the block-scaled MMA layout (the
    operand layout of fp4q_gemm); returns (codes, scales_mma, gscale)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    fmt, gmode = _fmt(fmt), _gmode(gmode)
    dev = x.device
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales_mma is None:
        scales_mma = torch.zeros((max(fp4q_mma_scales_size(rows, cols, block), 1),), dtype=torch.uint8, device=dev)
    if gscale is None and gmode == FP4Q_GLOBAL_FROM_AMAX:
        raise ValueError("from_amax mode reads the tensor maximum from gscale[0]: pass a 2-float gscale")
    if gscale is None and gmode != FP4Q_GLOBAL_NONE:
        gscale = torch.empty((1,), dtype=torch.float32, device=dev)
    _need_cuda(codes, scales_mma, gscale)
    st = lib().fp4q_quantize_mma(_ptr(x), rows, cols, fmt, block, rot, gmode, _ptr(codes), _ptr(scales_mma),
                                 _ptr(gscale), _stream(stream))
    _check(st, "fp4q_quantize_mma")
    return codes, scales_mma, gscale


def fp4q_gemm(codes_a: torch.Tensor, scales_a: torch.Tensor, gscale_a: Optional[torch.Tensor],
              codes_b: torch.Tensor, scales_b: torch.Tensor, gscale_b: Optional[torch.Tensor], fmt,
              y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = G_A G_B (A . S_A)(B . S_B)^T from two fp4q_quantize_mma outputs;
    returns y, fp32 [m][n]."""
    m, kb = codes_a.shape
    n, kb2 = codes_b.shape
    if kb != kb2:
        raise ValueError("A and B must have the same k")
    fmt = _fmt(fmt)
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=codes_a.device)
    _need_cuda(codes_a, scales_a, gscale_a, codes_b, scales_b, gscale_b, y)
    st = lib().fp4q_gemm(_ptr(codes_a), _ptr(scales_a), _ptr(gscale_a), m, _ptr(codes_b), _ptr(scales_b),
                         _ptr(gscale_b), n, 2 * kb, fmt, _ptr(y), _stream(stream))
    _check(st, "fp4q_gemm")
    return y


def fp4q_quantize_search(x: torch.Tensor, fmt, block: int, rot: int = 0, gmode="none", below: int = 1,
                         above: int = 1, codes: Optional[torch.Tensor] = None,
                         scales: Optional[torch.Tensor] = None, gscale: Optional[torch.Tensor] = None,
                         stream=None) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """fp4q_quantize with MSE-optimised block scales: per block the max-rule code,
    then up to `above` codes above and `below` below it are tried, and the code
    of least squared error is kept.  Returns (codes, scales, gscale)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    fmt, gmode = _fmt(fmt), _gmode(gmode)
    dev = x.device
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // block if block else 0), dtype=torch.uint8, device=dev)
    if gscale is None and gmode == FP4Q_GLOBAL_FROM_AMAX:
        raise ValueError("from_amax mode reads the tensor maximum from gscale[0]: pass a 2-float gscale")
    if gscale is None and gmode != FP4Q_GLOBAL_NONE:
        gscale = torch.empty((1,), dtype=torch.float32, device=dev)
    if gmode == FP4Q_GLOBAL_FROM_AMAX and gscale.numel() < 2:
        raise ValueError("from_amax mode needs gscale with 2 floats: [amax in, G out]")
    _need_cuda(codes, scales, gscale)
    st = lib().fp4q_quantize_search(_ptr(x), rows, cols, fmt, block, rot, gmode, below, above, _ptr(codes),
                                    _ptr(scales), _ptr(gscale), _stream(stream))
    _check(st, "fp4q_quantize_search")
    return codes, scales, gscale


def fp4q_outlier_stats(x: torch.Tensor, p: float = 0.999, channels: bool = True,
                       workspace: Optional[torch.Tensor] = None, stream=None):
    """Activation outlier statistics of a 2-D bf16 CUDA tensor [tokens, channels]:
    returns (stats, col_absmax) with stats = [max |x|, nearest-rank p-quantile of
    |x|] (a 2-float CUDA tensor) and the per-channel maxima (or None)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    dev = x.device
    stats = torch.empty((2,), dtype=torch.float32, device=dev)
    col = torch.empty((cols,), dtype=torch.float32, device=dev) if channels else None
    ws_bytes = lib().fp4q_outlier_stats_workspace_size()
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    _need_cuda(workspace)
    st = lib().fp4q_outlier_stats(_ptr(x), rows, cols, float(p), _ptr(stats), _ptr(col), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "fp4q_outlier_stats")
    return stats, col


def fp4q_tensor_amax(x: torch.Tensor, rot: int = 0, amax: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    if amax is None:
        amax = torch.empty((1,), dtype=torch.float32, device=x.device)
    st = lib().fp4q_tensor_amax(_ptr(x), x.shape[0], x.shape[1], rot, _ptr(amax), _stream(stream))
    _check(st, "fp4q_tensor_amax")
    return amax


def fp4q_tensor_amax_accumulate(x: torch.Tensor, amax: torch.Tensor, rot: int = 0, stream=None) -> torch.Tensor:
    """amax <- max(amax, max |y|) in place (amax: a 1-float CUDA tensor holding a
    non-negative value, e.g. 0 or the maximum of other shards)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x, amax)
    x = x.contiguous()
    st = lib().fp4q_tensor_amax_accumulate(_ptr(x), x.shape[0], x.shape[1], rot, _ptr(amax), _stream(stream))
    _check(st, "fp4q_tensor_amax_accumulate")
    return amax


def fp4q_tensor_amax_batched(xs, rot: int = 0, amax: Optional[torch.Tensor] = None, accumulate: bool = False,
                             stream=None) -> torch.Tensor:
    """max |y| of every tensor of xs (2-D bf16 CUDA tensors) in one pass:
    amax[i] (a float32 CUDA tensor of len(xs) entries, allocated if None) is
    set to, or with accumulate raised to, tensor i's maximum."""
    xs = list(xs)
    for x in xs:
        if x.dtype != torch.bfloat16 or x.dim() != 2:
            raise ValueError("every x must be a 2-D bf16 tensor")
    _need_cuda(*xs)
    xs = [x.contiguous() for x in xs]
    if amax is None:
        amax = torch.zeros((len(xs),), dtype=torch.float32, device=xs[0].device if xs else "cuda")
    if amax.dtype != torch.float32 or amax.numel() < len(xs):
        raise ValueError("amax must be a float32 tensor of len(xs) entries")
    _need_cuda(amax)
    n = len(xs)
    ptrs = (ctypes.c_void_p * max(n, 1))(*[_ptr(x) for x in xs])
    rows = (ctypes.c_int64 * max(n, 1))(*[x.shape[0] for x in xs])
    cols = (ctypes.c_int64 * max(n, 1))(*[x.shape[1] for x in xs])
    slots = (ctypes.c_void_p * max(n, 1))(*[amax.data_ptr() + 4 * i for i in range(n)])
    st = lib().fp4q_tensor_amax_batched(n, ptrs, rows, cols, rot, slots, 1 if accumulate else 0, _stream(stream))
    _check(st, "fp4q_tensor_amax_batched")
    return amax


def fp4q_global_scale(amax: torch.Tensor, gscale: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """G = amax / (6 * 448), or 1 if amax = 0 (device scalar in, device scalar out)."""
    _need_cuda(amax)
    if gscale is None:
        gscale = torch.empty((1,), dtype=torch.float32, device=amax.device)
    _check(lib().fp4q_global_scale(_ptr(amax), _ptr(gscale), _stream(stream)), "fp4q_global_scale")
    return gscale


def fp4q_dequantize(codes: torch.Tensor, scales: torch.Tensor, gscale: Optional[torch.Tensor],
                    rows: int, cols: int, fmt, block: int, rot: int = 0,
                    out_dtype: torch.dtype = torch.bfloat16, y: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Dequantize codes/scales into a [rows, cols] bf16 or fp32 tensor."""
    _need_cuda(codes, scales, gscale)
    od = FP4Q_OUT_F32 if out_dtype == torch.float32 else FP4Q_OUT_BF16
    if y is None:
        y = torch.empty((rows, cols), dtype=torch.float32 if od == FP4Q_OUT_F32 else torch.bfloat16,
                        device=codes.device)
    st = lib().fp4q_dequantize(_ptr(codes), _ptr(scales), _ptr(gscale), rows, cols, _fmt(fmt), block, rot,
                              od, _ptr(y), _stream(stream))
    _check(st, "fp4q_dequantize")
    return y


def fp4q_block_mse_workspace_size(rows: int, cols: int, block: int) -> int:
    return int(lib().fp4q_block_mse_workspace_size(rows, cols, block))


def fp4q_block_mse(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                   gscale: Optional[torch.Tensor], fmt, block: int, rot: int = 0,
                   block_mse: Optional[torch.Tensor] = None, want_block_mse: bool = True,
                   terms: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[Optional[torch.Tensor], torch.Tensor]:
    """Per-block MSE (fp32) and terms [total, non-max, max, zero-rounded] (fp64)."""
    _need_cuda(x, codes, scales, gscale)
    x = x.contiguous()
    rows, cols = x.shape
    dev = x.device
    if block_mse is None and want_block_mse:
        block_mse = torch.empty((rows, cols // block), dtype=torch.float32, device=dev)
    if terms is None:
        terms = torch.empty((4,), dtype=torch.float64, device=dev)
    ws = fp4q_block_mse_workspace_size(rows, cols, block)
    if workspace is None:
        workspace = torch.zeros((ws,), dtype=torch.uint8, device=dev)
    st = lib().fp4q_block_mse(_ptr(x), _ptr(codes), _ptr(scales), _ptr(gscale), rows, cols, _fmt(fmt),
                             block, rot, _ptr(block_mse), _ptr(terms), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "fp4q_block_mse")
    return block_mse, terms


def fp4q_block_mse_noalloc(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                           gscale: Optional[torch.Tensor], fmt, block: int, rot: int = 0,
                           block_mse: Optional[torch.Tensor] = None, terms: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[Optional[torch.Tensor], torch.Tensor]:
    """fp4q_block_mse with the library's fixed device scratch instead of a
    workspace, for callers that cannot allocate device memory: with
    ``block_mse`` and ``terms`` passed in, this function allocates nothing
    (block_mse may be None to skip the per-block output).  Calls in flight at
    the same time on one device race on the shared scratch; calls ordered on
    one stream do not."""
    _need_cuda(x, codes, scales, gscale)
    if not x.is_contiguous():
        raise ValueError("x must be contiguous (no copy is made here)")
    rows, cols = x.shape
    if terms is None:
        terms = torch.empty((4,), dtype=torch.float64, device=x.device)
    st = lib().fp4q_block_mse_noalloc(_ptr(x), _ptr(codes), _ptr(scales), _ptr(gscale), rows, cols, _fmt(fmt),
                                      block, rot, _ptr(block_mse), _ptr(terms), _stream(stream))
    _check(st, "fp4q_block_mse_noalloc")
    return block_mse, terms


def fp4q_quantize_mse(x: torch.Tensor, fmt, block: int, rot: int = 0, gmode="none",
                      codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                      gscale: Optional[torch.Tensor] = None, block_mse: Optional[torch.Tensor] = None,
                      want_block_mse: bool = True, terms: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """Quantize and measure the MSE in one pass: (codes, scales, gscale, block_mse, terms)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    fmt, gmode = _fmt(fmt), _gmode(gmode)
    dev = x.device
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // block if block else 0), dtype=torch.uint8, device=dev)
    if gscale is None and gmode == FP4Q_GLOBAL_FROM_AMAX:
        raise ValueError("from_amax mode reads the tensor maximum from gscale[0]: pass a 2-float gscale")
    if gscale is None and gmode != FP4Q_GLOBAL_NONE:
        gscale = torch.empty((1,), dtype=torch.float32, device=dev)
    if gmode == FP4Q_GLOBAL_FROM_AMAX and gscale.numel() < 2:
        raise ValueError("from_amax mode needs gscale with 2 floats: [amax in, G out]")
    if block_mse is None and want_block_mse:
        block_mse = torch.empty((rows, cols // block if block else 0), dtype=torch.float32, device=dev)
    if terms is None:
        terms = torch.empty((4,), dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.zeros((fp4q_block_mse_workspace_size(rows, cols, block),), dtype=torch.uint8,
                                device=dev)
    _need_cuda(codes, scales, gscale, block_mse, terms, workspace)
    st = lib().fp4q_quantize_mse(_ptr(x), rows, cols, fmt, block, rot, gmode, _ptr(codes), _ptr(scales),
                                 _ptr(gscale), _ptr(block_mse), _ptr(terms), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "fp4q_quantize_mse")
    return codes, scales, gscale, block_mse, terms


def fp4q_quantize_mse_dequantize(x: torch.Tensor, fmt, block: int, rot: int = 0, gmode="none",
                                 codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                                 gscale: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                                 block_mse: Optional[torch.Tensor] = None, want_block_mse: bool = True,
                                 terms: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                                 stream=None):
    """Quantize, measure the MSE and write the dequantized bf16 tensor in one pass:
    (codes, scales, gscale, y, block_mse, terms)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor")
    _need_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    fmt, gmode = _fmt(fmt), _gmode(gmode)
    dev = x.device
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // block if block else 0), dtype=torch.uint8, device=dev)
    if gscale is None and gmode == FP4Q_GLOBAL_FROM_AMAX:
        raise ValueError("from_amax mode reads the tensor maximum from gscale[0]: pass a 2-float gscale")
    if gscale is None and gmode != FP4Q_GLOBAL_NONE:
        gscale = torch.empty((1,), dtype=torch.float32, device=dev)
    if y is None:
        y = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    if block_mse is None and want_block_mse:
        block_mse = torch.empty((rows, cols // block if block else 0), dtype=torch.float32, device=dev)
    if terms is None:
        terms = torch.empty((4,), dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.zeros((fp4q_block_mse_workspace_size(rows, cols, block),), dtype=torch.uint8,
                                device=dev)
    _need_cuda(codes, scales, gscale, y, block_mse, terms, workspace)
    st = lib().fp4q_quantize_mse_dequantize(_ptr(x), rows, cols, fmt, block, rot, gmode, _ptr(codes), _ptr(scales),
                                            _ptr(gscale), _ptr(y), _ptr(block_mse), _ptr(terms), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "fp4q_quantize_mse_dequantize")
    return codes, scales, gscale, y, block_mse, terms


class Fp4qTensor(ctypes.Structure):
    """One tensor of a batched call (include/fp4q.h: fp4q_tensor)."""
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("gscale", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("block_mse", ctypes.c_void_p), ("terms", ctypes.c_void_p)]


def fp4q_quantize_batch_workspace_size(count: int) -> int:
    return lib().fp4q_quantize_batch_workspace_size(count)


def fp4q_quantize_mse_dequantize_batched(xs, fmt, block: int, rot: int = 0, gmode="none", gscales=None,
                                         want_block_mse: bool = True, workspace: Optional[torch.Tensor] = None,
                                         stream=None):
    """fp4q_quantize_mse_dequantize for every tensor of xs in one pass (MXFP4 b32
    or NVFP4 b16): a list of (codes, scales, gscale, y, block_mse, terms).
    gscales: per-tensor gscale buffers (FROM_AMAX: [amax, G] each), else allocated."""
    xs = [x.contiguous() for x in xs]
    for x in xs:
        if x.dtype != torch.bfloat16 or x.dim() != 2:
            raise ValueError("every x must be a 2-D bf16 tensor")
    _need_cuda(*xs)
    fmt, gmode = _fmt(fmt), _gmode(gmode)
    if gmode == FP4Q_GLOBAL_FROM_AMAX and gscales is None:
        raise ValueError("from_amax mode reads each tensor maximum from gscale[0]: pass 2-float gscales")
    n = len(xs)
    dev = xs[0].device if xs else torch.device("cuda")
    outs, descs = [], (Fp4qTensor * max(n, 1))()
    for i, x in enumerate(xs):
        rows, cols = x.shape
        g = gscales[i] if gscales is not None else (
            torch.empty((1,), dtype=torch.float32, device=dev) if gmode != FP4Q_GLOBAL_NONE else None)
        o = (torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
             torch.empty((rows, cols // block), dtype=torch.uint8, device=dev), g,
             torch.empty((rows, cols), dtype=torch.bfloat16, device=dev),
             torch.empty((rows, cols // block), dtype=torch.float32, device=dev) if want_block_mse else None,
             torch.empty((4,), dtype=torch.float64, device=dev))
        _need_cuda(*[t for t in o if t is not None])
        descs[i] = Fp4qTensor(_ptr(x), rows, cols, _ptr(o[0]), _ptr(o[1]), _ptr(o[2]), _ptr(o[3]), _ptr(o[4]),
                              _ptr(o[5]))
        outs.append(o)
    if workspace is None:
        workspace = torch.zeros((max(1, fp4q_quantize_batch_workspace_size(n)),), dtype=torch.uint8, device=dev)
    st = lib().fp4q_quantize_mse_dequantize_batched(n, descs, fmt, block, rot, gmode, _ptr(workspace),
                                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "fp4q_quantize_mse_dequantize_batched")
    return outs


def fp4q_e2m1_encode_f32(r: torch.Tensor, packed: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    _need_cuda(r)
    r = r.contiguous()
    if packed is None:
        packed = torch.empty((r.numel() // 2,), dtype=torch.uint8, device=r.device)
    _check(lib().fp4q_e2m1_encode_f32(_ptr(r), r.numel(), _ptr(packed), _stream(stream)),
           "fp4q_e2m1_encode_f32")
    return packed


def fp4q_scale_encode_f32(s: torch.Tensor, fmt, codes: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    _need_cuda(s)
    s = s.contiguous()
    if codes is None:
        codes = torch.empty((s.numel(),), dtype=torch.uint8, device=s.device)
    _check(lib().fp4q_scale_encode_f32(_ptr(s), s.numel(), _fmt(fmt), _ptr(codes), _stream(stream)),
           "fp4q_scale_encode_f32")
    return codes
