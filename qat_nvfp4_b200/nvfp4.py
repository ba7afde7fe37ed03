"""Python binding of libnvfp4.so (the C ABI in include/nvfp4.h).

Argument marshalling only: each function checks dtypes, devices and contiguity, allocates
outputs with torch when the caller does not pass them, and hands raw device pointers and
the current CUDA stream to the library.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing this module
raises if the library has not been built (``python -m qat_nvfp4_b200.build``).

Sources (web pages): fp4_optimization.py (VideoX-Fun) -- quantize_weight_to_float4,
dequantize_weight_from_float4; the verl ``linear.py`` tutorial -- section 2 (the
straight-through estimator), section 4 (sibling fusion), section 5 (observers).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python -m qat_nvfp4_b200.build, or __graft_entry__.build()).")

_lib = ctypes.CDLL(LIB_PATH)

MAX_SIBLINGS = 16
WORKSPACE_BYTES = 256
STATIC_MINMAX = 0
EMA = 1
OBSERVERS = {"static_minmax": STATIC_MINMAX, "minmax": EMA, "ema": EMA}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_status = ctypes.c_int


def _sig(name, args, res=_status):
    fn = getattr(_lib, name)
    fn.argtypes = args
    fn.restype = res
    return fn


_c_amax = _sig("nvfp4_amax", [_vp, _i64, _vp, _vp])
_c_amax_accumulate = _sig("nvfp4_amax_accumulate", [_vp, _i64, _vp, _vp])
_c_amax_multi = _sig("nvfp4_amax_multi", [ctypes.POINTER(_vp), ctypes.POINTER(_i64), ctypes.c_int, _vp, _vp])
_c_observer_update = _sig("nvfp4_observer_update", [_vp, _vp, ctypes.c_int, ctypes.c_double, _vp])
_c_observe_amax = _sig("nvfp4_observe_amax", [_vp, _i64, _vp, ctypes.c_int, ctypes.c_double, _vp, _vp])
_c_amax_ws = _sig("nvfp4_amax_ws", [_vp, _i64, _vp, _vp, _vp])
_c_observe_amax_ws = _sig("nvfp4_observe_amax_ws", [_vp, _i64, _vp, ctypes.c_int, ctypes.c_double, _vp, _vp, _vp])
_c_fake_quant_fused = _sig("nvfp4_fake_quant_fused", [_vp, _vp, _i64, _i64, _vp, _vp, _vp])
_c_observe_fake_quant = _sig("nvfp4_observe_fake_quant",
                             [_vp, _vp, _i64, _i64, _vp, ctypes.c_int, ctypes.c_double, _vp, _vp, _vp])
_c_workspace_check = _sig("nvfp4_workspace_check", [_vp, _vp])
_c_selftest_barrier_timeout = _sig("nvfp4_selftest_barrier_timeout",
                                   [_vp, _vp, _i64, _i64, _vp, _vp, ctypes.c_uint32, _vp])
_c_quantize = _sig("nvfp4_quantize", [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp])
_c_quantize_mma = _sig("nvfp4_quantize_mma", [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp])
_c_quantize_fused = _sig("nvfp4_quantize_fused", [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp])
_c_dequantize = _sig("nvfp4_dequantize", [_vp, _vp, _vp, _i64, _i64, _vp, _vp])
_c_fake_quant = _sig("nvfp4_fake_quant", [_vp, _vp, _i64, _i64, _vp, _vp])
_c_amax_strided = _sig("nvfp4_amax_strided", [_vp, _i64, _i64, _i64, _vp, _vp])
_c_quantize_strided = _sig("nvfp4_quantize_strided", [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp])
_c_fake_quant_strided = _sig("nvfp4_fake_quant_strided", [_vp, _i64, _vp, _i64, _i64, _i64, _vp, _vp])
_c_quantize_bs = _sig("nvfp4_quantize_bs", [_vp, _i64, _i64, ctypes.c_int, _vp, _vp, _vp, _vp, _vp])
_c_dequantize_bs = _sig("nvfp4_dequantize_bs", [_vp, _vp, _vp, _i64, _i64, ctypes.c_int, _vp, _vp])
_c_fake_quant_bs = _sig("nvfp4_fake_quant_bs", [_vp, _vp, _i64, _i64, ctypes.c_int, _vp, _vp])
_c_quantize_f32scale = _sig("nvfp4_quantize_f32scale", [_vp, _i64, _i64, _vp, _vp, _vp])
_c_dequantize_f32scale = _sig("nvfp4_dequantize_f32scale", [_vp, _vp, _i64, _i64, _vp, _vp])
_c_fake_quant_f32scale = _sig("nvfp4_fake_quant_f32scale", [_vp, _vp, _i64, _i64, _vp])
_c_fake_quant_siblings = _sig("nvfp4_fake_quant_siblings",
                              [ctypes.c_int, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_i64),
                               ctypes.POINTER(_i64), _vp, _vp])
_c_w4a16_tiled_bytes = _sig("nvfp4_w4a16_tiled_bytes", [_i64, _i64], _i64)
_c_w4a16_pack = _sig("nvfp4_w4a16_pack", [_vp, _vp, _i64, _i64, _vp, _vp])
_c_w4a16_linear = _sig("nvfp4_w4a16_linear", [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _vp])
_c_w4a16_workspace_bytes = _sig("nvfp4_w4a16_workspace_bytes", [_i64, _i64, _i64], _i64)
_c_w4a16_plan = _sig("nvfp4_w4a16_plan", [_i64, _i64, _i64, _i64, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)])
_c_w4a16_selftest_timeout = _sig("nvfp4_w4a16_selftest_timeout",
                                 [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _i64, ctypes.c_uint32, _vp])
_c_status_string = _sig("nvfp4_status_string", [ctypes.c_int], ctypes.c_char_p)
_c_launch_count = _sig("nvfp4_kernel_launch_count", [], ctypes.c_uint64)


class NVFP4Error(RuntimeError):
    """A libnvfp4 call returned a non-OK status."""


def nvfp4_status_string(status: int) -> str:
    return _c_status_string(int(status)).decode()


def nvfp4_kernel_launch_count() -> int:
    """Kernels launched by libnvfp4 in this process."""
    return int(_c_launch_count())


def _check(status: int, what: str):
    if status != 0:
        raise NVFP4Error(f"{what}: {nvfp4_status_string(status)}")


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _cuda(t: torch.Tensor, name: str, dtype=None, contiguous: bool = True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise RuntimeError(f"{name} must be a CUDA tensor (libnvfp4 has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise RuntimeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise RuntimeError(f"{name} must be contiguous")
    return t


def _as_rows(t: torch.Tensor, name: str):
    """(t, None) for a contiguous bf16 tensor; (rows, ld) for a view the strided calls take:
    its leading dimensions flatten into rows without a copy (a 2-D view, or e.g. [B, T, N]
    cut from a [B, T, 3N] fused output), its columns are contiguous, N % 16 == 0 and the row
    stride ld is a multiple of 16 and at least N."""
    _cuda(t, name, torch.bfloat16, contiguous=False)
    if t.is_contiguous():
        return t, None
    rows = None
    if t.dim() >= 2:
        try:
            rows = t.view(-1, t.shape[-1])
        except RuntimeError:
            rows = None
    if (rows is None or rows.stride(1) != 1 or rows.shape[1] % 16 or rows.stride(0) % 16
            or rows.stride(0) < rows.shape[1]):
        raise RuntimeError(f"{name} must be contiguous, or a view with contiguous rows (leading dimensions that "
                           f"flatten without a copy), a row stride that is a multiple of 16 elements and a "
                           f"multiple-of-16 row length")
    return rows, rows.stride(0)


def _scalar(t: torch.Tensor, name: str):
    _cuda(t, name, torch.float32)
    if t.numel() != 1:
        raise RuntimeError(f"{name} must hold exactly one fp32 value")
    return t


def _matrix(x: torch.Tensor, name: str = "x"):
    """(M, N) of a bf16 tensor seen as [M, N] rows along its last dimension."""
    _cuda(x, name, torch.bfloat16)
    if x.dim() < 1:
        raise RuntimeError(f"{name} must have at least one dimension")
    N = x.shape[-1]
    return math.prod(x.shape[:-1]), N


BLOCK_SIZES = (16, 32)


def padded_blocks(N: int, block: int = 16) -> int:
    """Blocks per row: rows are zero-padded to block * ceil(N / block) columns."""
    return (N + block - 1) // block


def _block(block) -> int:
    if block not in BLOCK_SIZES:
        raise ValueError(f"block must be one of {BLOCK_SIZES}, got {block!r}")
    return int(block)


def new_workspace(device) -> torch.Tensor:
    """A zero-filled workspace for the single-launch calls (one per stream in flight)."""
    return torch.zeros(WORKSPACE_BYTES, dtype=torch.uint8, device=device)


def _workspace(ws: torch.Tensor, device):
    _cuda(ws, "workspace", torch.uint8)
    if ws.numel() < WORKSPACE_BYTES or ws.device != device:
        raise RuntimeError(f"workspace must hold {WORKSPACE_BYTES} bytes on {device}")
    return ws


def nvfp4_amax(x: torch.Tensor, out: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Exact max |x| of a bf16 tensor, as a 1-element fp32 CUDA tensor.  With a workspace
    (see new_workspace) it is one kernel launch instead of a memset and a kernel.  x may also
    be a row-strided 2-D view (one of q/k/v inside a fused projection output), read in place
    by nvfp4_amax_strided."""
    rows, ld = _as_rows(x, "x")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _scalar(out, "out")
    with torch.cuda.device(x.device):
        if ld is not None:
            _check(_c_amax_strided(rows.data_ptr(), rows.shape[0], rows.shape[1], ld, out.data_ptr(),
                                   _stream(x.device)), "nvfp4_amax_strided")
        elif workspace is None:
            _check(_c_amax(x.data_ptr(), x.numel(), out.data_ptr(), _stream(x.device)), "nvfp4_amax")
        else:
            _workspace(workspace, x.device)
            _check(_c_amax_ws(x.data_ptr(), x.numel(), out.data_ptr(), workspace.data_ptr(), _stream(x.device)),
                   "nvfp4_amax_ws")
    return out


def nvfp4_amax_accumulate(x: torch.Tensor, running: torch.Tensor) -> torch.Tensor:
    """running <- max(running, max |x|) on the device; running is a 1-element fp32 CUDA
    tensor holding a non-negative value (0 to start)."""
    _cuda(x, "x", torch.bfloat16)
    if not x.is_contiguous():
        raise RuntimeError("x must be contiguous")
    _scalar(running, "running")
    with torch.cuda.device(x.device):
        _check(_c_amax_accumulate(x.data_ptr(), x.numel(), running.data_ptr(), _stream(x.device)),
               "nvfp4_amax_accumulate")
    return running


def nvfp4_amax_multi(xs: Sequence[torch.Tensor], out: torch.Tensor | None = None) -> torch.Tensor:
    """Shared amax of fused sibling tensors (max over all of them)."""
    xs = list(xs)
    if not 1 <= len(xs) <= MAX_SIBLINGS:
        raise RuntimeError(f"between 1 and {MAX_SIBLINGS} tensors")
    for i, t in enumerate(xs):
        _cuda(t, f"xs[{i}]", torch.bfloat16)
        if t.device != xs[0].device:
            raise RuntimeError("all siblings must be on one device")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=xs[0].device)
    _scalar(out, "out")
    k = len(xs)
    ptrs = (_vp * k)(*[t.data_ptr() for t in xs])
    ns = (_i64 * k)(*[t.numel() for t in xs])
    with torch.cuda.device(xs[0].device):
        _check(_c_amax_multi(ptrs, ns, k, out.data_ptr(), _stream(xs[0].device)), "nvfp4_amax_multi")
    return out


def _kind(kind) -> int:
    if isinstance(kind, str):
        if kind not in OBSERVERS:
            raise RuntimeError(f"unknown observer {kind!r}; one of {sorted(OBSERVERS)}")
        return OBSERVERS[kind]
    return int(kind)


def nvfp4_observer_update(state: torch.Tensor, cur_amax: torch.Tensor, kind="static_minmax",
                          decay: float = 0.01) -> torch.Tensor:
    """One observer step on an already computed (and already all-reduced) amax; in place."""
    _scalar(state, "state")
    _scalar(cur_amax, "cur_amax")
    with torch.cuda.device(state.device):
        _check(_c_observer_update(state.data_ptr(), cur_amax.data_ptr(), _kind(kind), float(decay),
                                  _stream(state.device)), "nvfp4_observer_update")
    return state


def nvfp4_observe_amax(x: torch.Tensor, state: torch.Tensor, kind="static_minmax", decay: float = 0.01,
                       cur_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """amax of x, then the observer step on ``state`` (in place); returns this step's amax.
    With a workspace it is one kernel launch.  A row-strided view x takes the strided amax
    and a separate observer step."""
    rows, ld = _as_rows(x, "x")
    _scalar(state, "state")
    if cur_out is None:
        cur_out = torch.empty(1, dtype=torch.float32, device=x.device)
    _scalar(cur_out, "cur_out")
    if ld is not None:
        nvfp4_amax(x, out=cur_out)
        nvfp4_observer_update(state, cur_out, kind, decay)
        return cur_out
    with torch.cuda.device(x.device):
        if workspace is None:
            _check(_c_observe_amax(x.data_ptr(), x.numel(), state.data_ptr(), _kind(kind), float(decay),
                                   cur_out.data_ptr(), _stream(x.device)), "nvfp4_observe_amax")
        else:
            _workspace(workspace, x.device)
            _check(_c_observe_amax_ws(x.data_ptr(), x.numel(), state.data_ptr(), _kind(kind), float(decay),
                                      cur_out.data_ptr(), workspace.data_ptr(), _stream(x.device)),
                   "nvfp4_observe_amax_ws")
    return cur_out


def nvfp4_quantize(x: torch.Tensor, amax: torch.Tensor, packed: torch.Tensor | None = None,
                   scales: torch.Tensor | None = None, global_scale: torch.Tensor | None = None,
                   block: int = 16):
    """bf16 [..., N] -> (packed uint8 [..., P/2], E4M3 scale bytes uint8 [..., P/block],
    global scale fp32 [1]), P = block * ceil(N / block).  ``amax`` is the tensor's (or
    siblings', or observer's) amax; ``block`` is 16 (NVFP4) or 32."""
    block = _block(block)
    rows, ld = _as_rows(x, "x")
    if ld is not None and block != 16:
        raise RuntimeError("row-strided views are quantized in blocks of 16")
    M, N = (rows.shape[0], rows.shape[1]) if ld is not None else _matrix(x)
    _scalar(amax, "amax")
    B = padded_blocks(N, block)
    lead = tuple(x.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (block // 2 * B,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (B,), dtype=torch.uint8, device=x.device)
    if global_scale is None:
        global_scale = torch.empty(1, dtype=torch.float32, device=x.device)
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.uint8)
    _scalar(global_scale, "global_scale")
    if packed.numel() != M * block // 2 * B or scales.numel() != M * B:
        raise RuntimeError("packed / scales have the wrong number of elements")
    with torch.cuda.device(x.device):
        if ld is not None:
            st = _c_quantize_strided(rows.data_ptr(), M, N, ld, amax.data_ptr(), packed.data_ptr(),
                                     scales.data_ptr(), global_scale.data_ptr(), _stream(x.device))
        elif block == 16:
            st = _c_quantize(x.data_ptr(), M, N, amax.data_ptr(), packed.data_ptr(), scales.data_ptr(),
                             global_scale.data_ptr(), _stream(x.device))
        else:
            st = _c_quantize_bs(x.data_ptr(), M, N, block, amax.data_ptr(), packed.data_ptr(), scales.data_ptr(),
                                global_scale.data_ptr(), _stream(x.device))
        _check(st, "nvfp4_quantize")
    return packed, scales, global_scale


def nvfp4_quantize_fused(x: torch.Tensor, packed: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                         global_scale: torch.Tensor | None = None, amax_out: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None):
    """quantize_weight_to_float4 in one call: the tensor's own amax, then quantize with it
    (one kernel launch up to twice the L2 size).  Returns (packed, scales, global scale,
    amax)."""
    M, N = _matrix(x)
    B = padded_blocks(N)
    lead = tuple(x.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (8 * B,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (B,), dtype=torch.uint8, device=x.device)
    if global_scale is None:
        global_scale = torch.empty(1, dtype=torch.float32, device=x.device)
    if amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=x.device)
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.uint8)
    _scalar(global_scale, "global_scale")
    _scalar(amax_out, "amax_out")
    if packed.numel() != M * 8 * B or scales.numel() != M * B:
        raise RuntimeError("packed / scales have the wrong number of elements")
    ws = new_workspace(x.device) if workspace is None else _workspace(workspace, x.device)
    with torch.cuda.device(x.device):
        _check(_c_quantize_fused(x.data_ptr(), M, N, amax_out.data_ptr(), packed.data_ptr(), scales.data_ptr(),
                                 global_scale.data_ptr(), ws.data_ptr(), _stream(x.device)), "nvfp4_quantize_fused")
    return packed, scales, global_scale, amax_out


def mma_scale_bytes(M: int, N: int) -> int:
    """Bytes of the tensor-core scale layout for an [M, N] tensor: 128 * ceil(M / 128)
    rows by 4 * ceil(B / 4) columns, B = ceil(N / 16)."""
    return (M + 127) // 128 * 128 * ((padded_blocks(N) + 3) // 4 * 4)


def nvfp4_quantize_mma(x: torch.Tensor, amax: torch.Tensor, packed: torch.Tensor | None = None,
                       scales_mma: torch.Tensor | None = None, global_scale: torch.Tensor | None = None):
    """nvfp4_quantize with the block scales written in the block-scaled tensor-core GEMM
    layout (128 x 4 tiles).  Returns (packed [..., 8*B], scales_mma uint8 [mma_scale_bytes],
    global scale fp32 [1]); the GEMM's per-tensor decode factor is 1 / global scale."""
    M, N = _matrix(x)
    _scalar(amax, "amax")
    B = padded_blocks(N)
    if packed is None:
        packed = torch.empty(tuple(x.shape[:-1]) + (8 * B,), dtype=torch.uint8, device=x.device)
    if scales_mma is None:
        scales_mma = torch.empty(mma_scale_bytes(M, N), dtype=torch.uint8, device=x.device)
    if global_scale is None:
        global_scale = torch.empty(1, dtype=torch.float32, device=x.device)
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales_mma, "scales_mma", torch.uint8)
    _scalar(global_scale, "global_scale")
    if packed.numel() != M * 8 * B or scales_mma.numel() != mma_scale_bytes(M, N):
        raise RuntimeError("packed / scales_mma have the wrong number of elements")
    with torch.cuda.device(x.device):
        _check(_c_quantize_mma(x.data_ptr(), M, N, amax.data_ptr(), packed.data_ptr(), scales_mma.data_ptr(),
                               global_scale.data_ptr(), _stream(x.device)), "nvfp4_quantize_mma")
    return packed, scales_mma, global_scale


def nvfp4_dequantize(packed: torch.Tensor, scales: torch.Tensor, global_scale: torch.Tensor,
                     out: torch.Tensor | None = None, n_cols: int | None = None, block: int = 16) -> torch.Tensor:
    """(packed [..., P/2], scales [..., P/block], global scale) -> bf16 [..., N].  ``n_cols``
    is the unpadded row length N (default P, the padded length), as the page keeps the
    original shape next to the packed weight."""
    block = _block(block)
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.uint8)
    _scalar(global_scale, "global_scale")
    P = packed.shape[-1] * 2
    N = P if n_cols is None else int(n_cols)
    if padded_blocks(N, block) * block != P:
        raise RuntimeError(f"n_cols={N} does not match packed rows of {P // 2} bytes")
    M = math.prod(packed.shape[:-1])
    if scales.numel() != M * (P // block):
        raise RuntimeError("scales has the wrong number of elements")
    if out is None:
        out = torch.empty(tuple(packed.shape[:-1]) + (N,), dtype=torch.bfloat16, device=packed.device)
    _cuda(out, "out", torch.bfloat16)
    if out.numel() != M * N:
        raise RuntimeError("out has the wrong number of elements")
    with torch.cuda.device(packed.device):
        if block == 16:
            st = _c_dequantize(packed.data_ptr(), scales.data_ptr(), global_scale.data_ptr(), M, N,
                               out.data_ptr(), _stream(packed.device))
        else:
            st = _c_dequantize_bs(packed.data_ptr(), scales.data_ptr(), global_scale.data_ptr(), M, N, block,
                                  out.data_ptr(), _stream(packed.device))
        _check(st, "nvfp4_dequantize")
    return out


def nvfp4_fake_quant(x: torch.Tensor, amax: torch.Tensor, out: torch.Tensor | None = None,
                     block: int = 16) -> torch.Tensor:
    """bf16 -> bf16 fake-quantization (dequantize(quantize(x)) in one pass).  ``out`` may be x;
    ``block`` is 16 (NVFP4) or 32.  With blocks of 16, x and out may also be row-strided
    views (q/k/v inside a fused projection output, 2-D or with leading dimensions that
    flatten into rows), read and written in place."""
    block = _block(block)
    xr, ld = _as_rows(x, "x")
    if out is None:
        out = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    outr, ld_out = _as_rows(out, "out")
    _scalar(amax, "amax")
    if out.numel() != x.numel():
        raise RuntimeError("out has the wrong number of elements")
    if ld is not None or ld_out is not None:
        _fake_quant_rows(xr, ld, outr, ld_out, amax, block)
        return out
    M, N = _matrix(x)
    with torch.cuda.device(x.device):
        if block == 16:
            st = _c_fake_quant(x.data_ptr(), out.data_ptr(), M, N, amax.data_ptr(), _stream(x.device))
        else:
            st = _c_fake_quant_bs(x.data_ptr(), out.data_ptr(), M, N, block, amax.data_ptr(), _stream(x.device))
        _check(st, "nvfp4_fake_quant")
    return out


# ---- the fp32-scale flavour (blocks of 32, one fp32 scale each, no global scale) ----

def nvfp4_quantize_f32scale(x: torch.Tensor, packed: torch.Tensor | None = None,
                            scales: torch.Tensor | None = None):
    """bf16 [..., N] -> (packed uint8 [..., P/2], fp32 block scales [..., P/32]),
    P = 32 * ceil(N / 32): blocks of 32 with scale = block amax / 6 kept in fp32 (the
    fp32-scale flavour of quantize_weight_to_float4; no per-tensor scale)."""
    M, N = _matrix(x)
    B = padded_blocks(N, 32)
    lead = tuple(x.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (16 * B,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (B,), dtype=torch.float32, device=x.device)
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    if packed.numel() != M * 16 * B or scales.numel() != M * B:
        raise RuntimeError("packed / scales have the wrong number of elements")
    with torch.cuda.device(x.device):
        _check(_c_quantize_f32scale(x.data_ptr(), M, N, packed.data_ptr(), scales.data_ptr(), _stream(x.device)),
               "nvfp4_quantize_f32scale")
    return packed, scales


def nvfp4_dequantize_f32scale(packed: torch.Tensor, scales: torch.Tensor, n_cols: int | None = None,
                              out: torch.Tensor | None = None) -> torch.Tensor:
    """(packed [..., P/2], fp32 scales [..., P/32]) -> bf16 [..., n_cols]: bf16(LUT * scale),
    cropped to n_cols (default P)."""
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    P = packed.shape[-1] * 2
    N = P if n_cols is None else int(n_cols)
    if padded_blocks(N, 32) * 32 != P:
        raise RuntimeError(f"n_cols={N} does not match packed rows of {P // 2} bytes")
    M = math.prod(packed.shape[:-1])
    if scales.numel() != M * (P // 32):
        raise RuntimeError("scales has the wrong number of elements")
    if out is None:
        out = torch.empty(tuple(packed.shape[:-1]) + (N,), dtype=torch.bfloat16, device=packed.device)
    _cuda(out, "out", torch.bfloat16)
    if out.numel() != M * N:
        raise RuntimeError("out has the wrong number of elements")
    with torch.cuda.device(packed.device):
        _check(_c_dequantize_f32scale(packed.data_ptr(), scales.data_ptr(), M, N, out.data_ptr(),
                                      _stream(packed.device)), "nvfp4_dequantize_f32scale")
    return out


def nvfp4_fake_quant_f32scale(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 -> bf16: dequantize_f32scale(quantize_f32scale(x)) in one pass; ``out`` may be x."""
    M, N = _matrix(x)
    if out is None:
        out = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    _cuda(out, "out", torch.bfloat16)
    if out.numel() != x.numel():
        raise RuntimeError("out has the wrong number of elements")
    with torch.cuda.device(x.device):
        _check(_c_fake_quant_f32scale(x.data_ptr(), out.data_ptr(), M, N, _stream(x.device)),
               "nvfp4_fake_quant_f32scale")
    return out


def _fake_quant_rows(xr, ld, outr, ld_out, amax, block):
    """Fake-quant between row views (either may be strided) through nvfp4_fake_quant_strided."""
    if ld is None:
        xr = xr.reshape(-1, xr.shape[-1])  # contiguous: a view
    if ld_out is None:
        outr = outr.reshape(-1, outr.shape[-1])
    if block != 16 or tuple(outr.shape) != tuple(xr.shape):
        raise RuntimeError("row-strided fake-quant takes views of one shape and blocks of 16")
    M, N = xr.shape
    with torch.cuda.device(xr.device):
        _check(_c_fake_quant_strided(xr.data_ptr(), N if ld is None else ld, outr.data_ptr(),
                                     N if ld_out is None else ld_out, M, N, amax.data_ptr(), _stream(xr.device)),
               "nvfp4_fake_quant_strided")


def nvfp4_fake_quant_siblings(xs: Sequence[torch.Tensor], outs: Sequence[torch.Tensor] | None = None,
                              amax_out: torch.Tensor | None = None):
    """Shared amax of the siblings, then each fake-quantized with it.  Returns (outs, amax)."""
    xs = list(xs)
    k = len(xs)
    if not 1 <= k <= MAX_SIBLINGS:
        raise RuntimeError(f"between 1 and {MAX_SIBLINGS} tensors")
    shapes = [_matrix(t, f"xs[{i}]") for i, t in enumerate(xs)]
    dev = xs[0].device
    if any(t.device != dev for t in xs):
        raise RuntimeError("all siblings must be on one device")
    outs = [torch.empty_like(t) for t in xs] if outs is None else list(outs)
    if len(outs) != k:
        raise RuntimeError("outs must match xs")
    for i, (o, t) in enumerate(zip(outs, xs)):
        _cuda(o, f"outs[{i}]", torch.bfloat16)
        if o.numel() != t.numel() or o.device != dev:
            raise RuntimeError(f"outs[{i}] does not match xs[{i}]")
    if amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=dev)
    _scalar(amax_out, "amax_out")
    xp = (_vp * k)(*[t.data_ptr() for t in xs])
    yp = (_vp * k)(*[t.data_ptr() for t in outs])
    Ms = (_i64 * k)(*[m for m, _ in shapes])
    Ns = (_i64 * k)(*[n for _, n in shapes])
    with torch.cuda.device(dev):
        _check(_c_fake_quant_siblings(k, xp, yp, Ms, Ns, amax_out.data_ptr(), _stream(dev)),
               "nvfp4_fake_quant_siblings")
    return outs, amax_out


def nvfp4_fake_quant_fused(x: torch.Tensor, out: torch.Tensor | None = None, amax_out: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None):
    """Fake-quantize x with its own amax in one pass (one cooperative kernel when x fits in
    L2).  Returns (y, amax).  ``out`` may be x."""
    M, N = _matrix(x)
    out = torch.empty_like(x) if out is None else out
    _cuda(out, "out", torch.bfloat16)
    if out.numel() != x.numel():
        raise RuntimeError("out has the wrong number of elements")
    amax_out = torch.empty(1, dtype=torch.float32, device=x.device) if amax_out is None else amax_out
    _scalar(amax_out, "amax_out")
    workspace = new_workspace(x.device) if workspace is None else _workspace(workspace, x.device)
    with torch.cuda.device(x.device):
        _check(_c_fake_quant_fused(x.data_ptr(), out.data_ptr(), M, N, amax_out.data_ptr(), workspace.data_ptr(),
                                   _stream(x.device)), "nvfp4_fake_quant_fused")
    return out, amax_out


def nvfp4_observe_fake_quant(x: torch.Tensor, state: torch.Tensor, kind="static_minmax", decay: float = 0.01,
                             out: torch.Tensor | None = None, cur_out: torch.Tensor | None = None,
                             workspace: torch.Tensor | None = None):
    """One W4A4 activation step in one pass: amax of x, observer step on ``state`` (in
    place), fake-quant with the updated state.  Returns (y, this step's amax).  Row-strided
    views (x or out) take three launches instead: strided amax, observer step, strided
    fake-quant."""
    xr, ld = _as_rows(x, "x")
    _scalar(state, "state")
    out = torch.empty(x.shape, dtype=x.dtype, device=x.device) if out is None else out
    outr, ld_out = _as_rows(out, "out")
    if out.numel() != x.numel():
        raise RuntimeError("out has the wrong number of elements")
    cur_out = torch.empty(1, dtype=torch.float32, device=x.device) if cur_out is None else cur_out
    _scalar(cur_out, "cur_out")
    if ld is not None or ld_out is not None:
        nvfp4_amax(x, out=cur_out)
        nvfp4_observer_update(state, cur_out, kind, decay)
        _fake_quant_rows(xr, ld, outr, ld_out, state, 16)
        return out, cur_out
    M, N = _matrix(x)
    workspace = new_workspace(x.device) if workspace is None else _workspace(workspace, x.device)
    with torch.cuda.device(x.device):
        _check(_c_observe_fake_quant(x.data_ptr(), out.data_ptr(), M, N, state.data_ptr(), _kind(kind), float(decay),
                                     cur_out.data_ptr(), workspace.data_ptr(), _stream(x.device)),
               "nvfp4_observe_fake_quant")
    return out, cur_out


def nvfp4_workspace_check(workspace: torch.Tensor) -> int:
    """Wait for the current stream; return 0 if no bounded device wait gave up since the
    last check, else the status code (NVFP4_ERR_TIMEOUT = 6), re-zeroing the workspace."""
    _workspace(workspace, workspace.device)
    with torch.cuda.device(workspace.device):
        return int(_c_workspace_check(workspace.data_ptr(), _stream(workspace.device)))


def nvfp4_selftest_barrier_timeout(x: torch.Tensor, workspace: torch.Tensor, timeout_us: int = 2000) -> int:
    """Run the fused kernel with a barrier that cannot complete and a short wait limit (a
    test of the bounded wait); returns the launch status."""
    M, N = _matrix(x)
    _workspace(workspace, x.device)
    y = torch.empty_like(x)
    amax = torch.empty(1, dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        return int(_c_selftest_barrier_timeout(x.data_ptr(), y.data_ptr(), M, N, amax.data_ptr(),
                                               workspace.data_ptr(), int(timeout_us), _stream(x.device)))


def nvfp4_w4a16_tiled_bytes(N: int, K: int) -> int:
    """Bytes of the operand form of an [N, K] packed weight (-1 if the shape is refused)."""
    return int(_c_w4a16_tiled_bytes(N, K))


def nvfp4_w4a16_pack(packed: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """Packed weight (packed [N, K/2], scales [N, K/16]) -> its operand form for
    nvfp4_w4a16_linear: one 4608-byte record per 128 x 64 tile (uint8, 1-D)."""
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.uint8)
    if packed.dim() != 2:
        raise RuntimeError("packed must be [N, K/2]")
    N, K = packed.shape[0], packed.shape[1] * 2
    if scales.numel() != N * (K // 16):
        raise RuntimeError("scales has the wrong number of elements")
    nbytes = nvfp4_w4a16_tiled_bytes(N, K)
    if nbytes < 0:
        raise RuntimeError(f"weight shape ({N}, {K}) not accepted (K must be a positive multiple of 16)")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=packed.device)
    _cuda(out, "out", torch.uint8)
    if out.numel() != nbytes:
        raise RuntimeError(f"out must hold {nbytes} bytes")
    with torch.cuda.device(packed.device):
        _check(_c_w4a16_pack(packed.data_ptr(), scales.data_ptr(), N, K, out.data_ptr(), _stream(packed.device)),
               "nvfp4_w4a16_pack")
    return out


def nvfp4_w4a16_linear(x: torch.Tensor, tiled: torch.Tensor, global_scale: torch.Tensor, n_out: int,
                       bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Forward of a Linear layer on an NVFP4 weight [n_out, K] in operand form (tiled, from
    nvfp4_w4a16_pack) with its encode global scale: x [..., K] bf16 -> bf16 [..., n_out] =
    x W^T + bias.  The weight is decoded inside the tensor-core kernel and is never
    materialised in device memory."""
    M, K = _matrix(x)
    _cuda(tiled, "tiled", torch.uint8)
    _scalar(global_scale, "global_scale")
    N = int(n_out)
    if tiled.numel() != nvfp4_w4a16_tiled_bytes(N, K):
        raise RuntimeError(f"tiled does not hold a [{N}, {K}] weight")
    if bias is not None:
        _cuda(bias, "bias", torch.bfloat16)
        if bias.numel() != N:
            raise RuntimeError("bias must have n_out elements")
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=torch.bfloat16, device=x.device)
    _cuda(out, "out", torch.bfloat16)
    if out.numel() != M * N:
        raise RuntimeError("out has the wrong number of elements")
    with torch.cuda.device(x.device):
        if workspace is None:
            workspace = nvfp4_w4a16_workspace(M, N, K, x.device)
        ws = _workspace(workspace, x.device)
        _check(_c_w4a16_linear(x.data_ptr(), M, K, tiled.data_ptr(), global_scale.data_ptr(), N,
                               bias.data_ptr() if bias is not None else None, out.data_ptr(), ws.data_ptr(),
                               ws.numel(), _stream(x.device)), "nvfp4_w4a16_linear")
    return out


def nvfp4_w4a16_selftest_timeout(x: torch.Tensor, tiled: torch.Tensor, global_scale: torch.Tensor, n_out: int,
                                 workspace: torch.Tensor, timeout_us: int = 2000) -> int:
    """Run the W4A16 kernel with a wait that nothing completes (limited to timeout_us) and
    return the status nvfp4_workspace_check then reports (NVFP4_ERR_TIMEOUT = 6 expected)."""
    M, K = _matrix(x)
    _cuda(tiled, "tiled", torch.uint8)
    _scalar(global_scale, "global_scale")
    ws = _workspace(workspace, x.device)
    y = torch.empty(tuple(x.shape[:-1]) + (int(n_out),), dtype=torch.bfloat16, device=x.device)
    with torch.cuda.device(x.device):
        _check(_c_w4a16_selftest_timeout(x.data_ptr(), M, K, tiled.data_ptr(), global_scale.data_ptr(), int(n_out),
                                         y.data_ptr(), ws.data_ptr(), ws.numel(), int(timeout_us),
                                         _stream(x.device)), "nvfp4_w4a16_selftest_timeout")
        return int(_c_workspace_check(ws.data_ptr(), _stream(x.device)))


def nvfp4_w4a16_workspace_bytes(M: int, N: int, K: int) -> int:
    """Workspace bytes with which nvfp4_w4a16_linear takes its fastest plan on this shape
    (current device: room for the partial sums of a split K or of the small kernel), at least
    WORKSPACE_BYTES; -1 if the shape is refused."""
    return int(_c_w4a16_workspace_bytes(M, N, K))


def nvfp4_w4a16_plan(M: int, N: int, K: int, workspace_bytes: int, sms: int) -> tuple[str, int, int]:
    """How nvfp4_w4a16_linear runs this shape with a workspace of workspace_bytes on a device
    with `sms` SMs: which kernel ("small": up to 8 rows of x on a weight with at most one
    output tile per two SMs, the weight shared evenly by two CTAs per SM; "shared" or
    "tensor": where the larger kernels keep the decoded weight; "cores": the CUDA-core kernel
    for one row), the rows of x per output tile, and the CTAs per tile over K (for "small":
    the CTAs that share the weight).  Host only, no GPU needed."""
    kernel, rows, splits = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(_c_w4a16_plan(M, N, K, workspace_bytes, sms, ctypes.byref(kernel), ctypes.byref(rows),
                         ctypes.byref(splits)), "nvfp4_w4a16_plan")
    return ("shared", "tensor", "cores", "small")[kernel.value], rows.value, splits.value


def nvfp4_w4a16_workspace(M: int, N: int, K: int, device) -> torch.Tensor:
    """A zeroed workspace large enough for nvfp4_w4a16_linear to split K on this shape
    (reusable across calls of the same or smaller shape, one call at a time)."""
    with torch.cuda.device(device):
        nbytes = int(_c_w4a16_workspace_bytes(M, N, K))
    if nbytes < 0:
        raise RuntimeError(f"linear shape M={M}, N={N}, K={K} not accepted")
    return torch.zeros(max(nbytes, WORKSPACE_BYTES), dtype=torch.uint8, device=device)


class FakeQuantSTE(torch.autograd.Function):
    """NVFP4 fake-quant forward with the straight-through backward (the gradient passes
    unchanged): the verl linear.py tutorial, section 2 (STEFP4QuantTriton)."""

    @staticmethod
    def forward(ctx, x, amax, block=16):
        # row-strided views go to the strided kernel as they are; other layouts are made
        # contiguous first
        if not x.is_contiguous():
            try:
                _as_rows(x, "x")
                if block != 16:
                    x = x.contiguous()
            except RuntimeError:
                x = x.contiguous()
        return nvfp4_fake_quant(x, amax, block=block)

    @staticmethod
    def backward(ctx, grad_output):
        return grad_output, None, None


def fake_quant_ste(x: torch.Tensor, amax: torch.Tensor, block: int = 16) -> torch.Tensor:
    return FakeQuantSTE.apply(x, amax, block)
