"""Host-side checks of the C ABI that need no GPU: every symbol the header declares is
exported, and every argument error is reported before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

from qat_nvfp4_b200.build import INCLUDE, LIB

NVFP4_OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_ARG, ERR_CUDA = 0, 1, 2, 3, 4, 5


def declared_symbols():
    names = set()
    for fn in os.listdir(INCLUDE):
        if fn.endswith(".h"):
            with open(os.path.join(INCLUDE, fn)) as f:
                text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
            names |= set(re.findall(r"\b(nvfp4_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(LIB)


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ["nvfp4_amax", "nvfp4_amax_multi", "nvfp4_observer_update", "nvfp4_observe_amax",
                     "nvfp4_quantize", "nvfp4_dequantize", "nvfp4_fake_quant", "nvfp4_fake_quant_siblings",
                     "nvfp4_quantize_bs", "nvfp4_dequantize_bs", "nvfp4_fake_quant_bs", "nvfp4_w4a16_linear",
                     "nvfp4_w4a16_pack", "nvfp4_w4a16_tiled_bytes", "nvfp4_quantize_fused",
                     "nvfp4_amax_accumulate", "nvfp4_w4a16_workspace_bytes", "nvfp4_amax_strided",
                     "nvfp4_quantize_strided", "nvfp4_fake_quant_strided", "nvfp4_w4a16_plan",
                     "nvfp4_status_string", "nvfp4_kernel_launch_count", "nvfp4_quantize_f32scale",
                     "nvfp4_dequantize_f32scale", "nvfp4_fake_quant_f32scale"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (nvfp4_\w+)", out))
    for name in declared_symbols():
        assert name in exported, f"{name} declared but not exported"
        assert getattr(lib, name) is not None
    # nothing else with the prefix leaks out
    assert exported <= set(declared_symbols())


def test_status_strings(lib):
    lib.nvfp4_status_string.restype = ctypes.c_char_p
    for code in range(7):
        assert lib.nvfp4_status_string(code).startswith(b"NVFP4_")
    assert b"unknown" in lib.nvfp4_status_string(99)


# Fake device addresses: validation must reject them before any CUDA call, so they are
# never dereferenced.
A32 = 0x7F0000000000  # 32-byte aligned
A8 = A32 + 8          # 8-byte aligned only
ODD = A32 + 2         # bf16 aligned only


def _call(lib, name, *args):
    fn = getattr(lib, name)
    fn.restype = ctypes.c_int
    return fn(*args)


def _i(v):
    return ctypes.c_int64(v)


def _p(v):
    return ctypes.c_void_p(v)


def _c(v):
    return ctypes.c_int(v)


def _gpu_visible():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


# These cases pass made-up device addresses; on a host with a GPU a case that wrongly got
# past validation would launch on them, so the test only runs where no GPU is visible
# (there such a case fails harmlessly with NVFP4_ERR_CUDA and the assertion catches it).
@pytest.mark.skipif(_gpu_visible(), reason="fake device addresses: host-only test")
def test_validation_errors_launch_nothing(lib):
    lib.nvfp4_kernel_launch_count.restype = ctypes.c_uint64
    before = lib.nvfp4_kernel_launch_count()
    S = _p(0)  # default stream
    amax, gs = _p(A32 + 64), _p(A32 + 128)
    cases = [
        # fake_quant
        (ERR_SHAPE, "nvfp4_fake_quant", _p(A32), _p(A32 + 4096), _i(4), _i(-24), amax, S),
        (ERR_SHAPE, "nvfp4_fake_quant", _p(A32), _p(A32 + 4096), _i(-1), _i(16), amax, S),
        (ERR_SHAPE, "nvfp4_fake_quant", _p(A32), _p(A32 + 4096), _i(1 << 40), _i(1 << 40), amax, S),
        (ERR_NULL, "nvfp4_fake_quant", _p(0), _p(A32 + 4096), _i(4), _i(16), amax, S),
        (ERR_NULL, "nvfp4_fake_quant", _p(A32), _p(A32 + 4096), _i(4), _i(16), _p(0), S),
        (ERR_ALIGN, "nvfp4_fake_quant", _p(ODD), _p(A32 + 4096), _i(4), _i(16), amax, S),
        (ERR_ALIGN, "nvfp4_fake_quant", _p(A32), _p(A32 + 4096), _i(4), _i(16), _p(A32 + 2), S),
        (ERR_ARG, "nvfp4_fake_quant", _p(A32), _p(A32 + 32), _i(4), _i(16), amax, S),  # partial overlap
        # quantize
        (ERR_SHAPE, "nvfp4_quantize", _p(A32), _i(2), _i(-8), amax, _p(A32), _p(A32), gs, S),
        (ERR_SHAPE, "nvfp4_quantize", _p(A32), _i(1 << 58), _i(17), amax, _p(A32), _p(A32), gs, S),
        (ERR_NULL, "nvfp4_quantize", _p(A32), _i(2), _i(16), amax, _p(0), _p(A32), gs, S),
        (ERR_NULL, "nvfp4_quantize", _p(A32), _i(2), _i(16), amax, _p(A32), _p(0), gs, S),
        (ERR_ALIGN, "nvfp4_quantize", _p(A32), _i(2), _i(16), amax, _p(A32 + 4), _p(A32), gs, S),
        (ERR_ALIGN, "nvfp4_quantize", _p(A8), _i(2), _i(16), amax, _p(A32), _p(A32), gs, S),
        # row-strided views: amax(x, M, N, ldx, amax), quantize(x, M, N, ldx, amax, packed, scales, gs),
        # fake_quant(x, ldx, y, ldy, M, N, amax)
        (ERR_ARG, "nvfp4_amax_strided", _p(A32), _i(4), _i(32), _i(16), amax, S),          # ldx < N
        (ERR_ARG, "nvfp4_amax_strided", _p(A32), _i(4), _i(32), _i(40), amax, S),          # ldx % 16
        (ERR_SHAPE, "nvfp4_amax_strided", _p(A32), _i(4), _i(24), _i(48), amax, S),        # N % 16
        (ERR_SHAPE, "nvfp4_amax_strided", _p(A32), _i(1 << 50), _i(16), _i(1 << 20), amax, S),  # span too large
        (ERR_NULL, "nvfp4_amax_strided", _p(0), _i(4), _i(32), _i(64), amax, S),
        (ERR_ALIGN, "nvfp4_amax_strided", _p(A8), _i(4), _i(32), _i(64), amax, S),
        (ERR_ARG, "nvfp4_quantize_strided", _p(A32), _i(2), _i(32), _i(16), amax, _p(A32), _p(A32), gs, S),
        (ERR_NULL, "nvfp4_quantize_strided", _p(A32), _i(2), _i(32), _i(64), _p(0), _p(A32), _p(A32), gs, S),
        (ERR_ALIGN, "nvfp4_quantize_strided", _p(A32), _i(2), _i(32), _i(64), amax, _p(A32 + 4), _p(A32), gs, S),
        (ERR_ARG, "nvfp4_fake_quant_strided", _p(A32), _i(64), _p(A32 + 64), _i(64), _i(2), _i(32), amax, S),  # k inside q's span
        (ERR_ARG, "nvfp4_fake_quant_strided", _p(A32), _i(64), _p(A32), _i(96), _i(2), _i(32), amax, S),  # same start, other stride
        (ERR_ARG, "nvfp4_fake_quant_strided", _p(A32), _i(64), _p(A32 + 8192), _i(24), _i(2), _i(32), amax, S),  # ldy < N
        (ERR_ALIGN, "nvfp4_fake_quant_strided", _p(A32), _i(64), _p(A32 + 8200), _i(64), _i(2), _i(32), amax, S),
        (ERR_NULL, "nvfp4_fake_quant_strided", _p(A32), _i(64), _p(A32 + 8192), _i(64), _i(2), _i(32), _p(0), S),
        # dequantize
        (ERR_NULL, "nvfp4_dequantize", _p(A32), _p(A32), _p(0), _i(2), _i(16), _p(A32), S),
        (ERR_ALIGN, "nvfp4_dequantize", _p(A32), _p(A32), gs, _i(2), _i(16), _p(A8), S),
        (ERR_SHAPE, "nvfp4_dequantize", _p(A32), _p(A32), gs, _i(-2), _i(17), _p(A32), S),
        # block-size variants: only 16 and 32; block 32 wants 16-byte aligned codes
        (ERR_ARG, "nvfp4_quantize_bs", _p(A32), _i(2), _i(64), _c(64), amax, _p(A32), _p(A32), gs, S),
        (ERR_ARG, "nvfp4_quantize_bs", _p(A32), _i(2), _i(64), _c(0), amax, _p(A32), _p(A32), gs, S),
        (ERR_ARG, "nvfp4_fake_quant_bs", _p(A32), _p(A32 + 4096), _i(2), _i(64), _c(8), amax, S),
        (ERR_ARG, "nvfp4_dequantize_bs", _p(A32), _p(A32), gs, _i(2), _i(64), _c(-32), _p(A32), S),
        (ERR_ALIGN, "nvfp4_quantize_bs", _p(A32), _i(2), _i(64), _c(32), amax, _p(A8), _p(A32), gs, S),
        (ERR_ALIGN, "nvfp4_dequantize_bs", _p(A8), _p(A32), gs, _i(2), _i(64), _c(32), _p(A32), S),
        (ERR_SHAPE, "nvfp4_quantize_bs", _p(A32), _i(1 << 56), _i(33), _c(32), amax, _p(A32), _p(A32), gs, S),
        (ERR_SHAPE, "nvfp4_fake_quant_bs", _p(A32), _p(A32 + 4096), _i(2), _i(-32), _c(32), amax, S),
        (ERR_NULL, "nvfp4_fake_quant_bs", _p(A32), _p(A32 + 4096), _i(2), _i(64), _c(32), _p(0), S),
        # fp32-scale flavour: quantize(x, M, N, packed, scales), dequantize(packed, scales, M, N, y),
        # fake_quant(x, y, M, N); codes 16-byte aligned, scales 4, bf16 tensors 32
        (ERR_NULL, "nvfp4_quantize_f32scale", _p(A32), _i(2), _i(64), _p(A32), _p(0), S),
        (ERR_ALIGN, "nvfp4_quantize_f32scale", _p(A32), _i(2), _i(64), _p(A8), _p(A32), S),
        (ERR_ALIGN, "nvfp4_quantize_f32scale", _p(A32), _i(2), _i(64), _p(A32), _p(A32 + 2), S),
        (ERR_ALIGN, "nvfp4_quantize_f32scale", _p(A32 + 16), _i(2), _i(64), _p(A32), _p(A32), S),
        (ERR_SHAPE, "nvfp4_quantize_f32scale", _p(A32), _i(-1), _i(64), _p(A32), _p(A32), S),
        (ERR_SHAPE, "nvfp4_quantize_f32scale", _p(A32), _i(1 << 56), _i(33), _p(A32), _p(A32), S),
        (NVFP4_OK, "nvfp4_quantize_f32scale", _p(0), _i(0), _i(64), _p(0), _p(0), S),
        (ERR_NULL, "nvfp4_dequantize_f32scale", _p(A32), _p(A32), _i(2), _i(64), _p(0), S),
        (ERR_ALIGN, "nvfp4_dequantize_f32scale", _p(A32), _p(A32), _i(2), _i(64), _p(A8), S),
        (ERR_ALIGN, "nvfp4_dequantize_f32scale", _p(A32), _p(A32 + 1), _i(2), _i(64), _p(A32), S),
        (ERR_SHAPE, "nvfp4_dequantize_f32scale", _p(A32), _p(A32), _i(2), _i(-64), _p(A32), S),
        (NVFP4_OK, "nvfp4_dequantize_f32scale", _p(0), _p(0), _i(3), _i(0), _p(0), S),
        (ERR_ARG, "nvfp4_fake_quant_f32scale", _p(A32), _p(A32 + 64), _i(2), _i(64), S),   # y inside x's span
        (ERR_NULL, "nvfp4_fake_quant_f32scale", _p(0), _p(A32), _i(2), _i(64), S),
        (ERR_ALIGN, "nvfp4_fake_quant_f32scale", _p(A32), _p(A8), _i(2), _i(64), S),
        (ERR_SHAPE, "nvfp4_fake_quant_f32scale", _p(A32), _p(A32), _i(-2), _i(64), S),
        # W4A16: linear(x, M, K, tiled, gs, N, bias, y, workspace), pack(packed, scales, N, K, tiled)
        (ERR_SHAPE, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(24), _p(A32), gs, _i(8), _p(0), _p(A32), _p(A32), _i(256), S),
        (ERR_SHAPE, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(0), _p(A32), gs, _i(8), _p(0), _p(A32), _p(A32), _i(256), S),
        (ERR_SHAPE, "nvfp4_w4a16_linear", _p(A32), _i(-1), _i(64), _p(A32), gs, _i(8), _p(0), _p(A32), _p(A32), _i(256), S),
        (ERR_NULL, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(64), _p(A32), gs, _i(8), _p(0), _p(A32), _p(0), _i(256), S),
        (ERR_NULL, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(64), _p(0), gs, _i(8), _p(0), _p(A32), _p(A32), _i(256), S),
        (ERR_ALIGN, "nvfp4_w4a16_linear", _p(A8), _i(4), _i(64), _p(A32), gs, _i(8), _p(0), _p(A32), _p(A32), _i(256), S),
        (ERR_ALIGN, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(64), _p(A8), gs, _i(8), _p(0), _p(A32), _p(A32), _i(256), S),
        (NVFP4_OK, "nvfp4_w4a16_linear", _p(0), _i(0), _i(64), _p(0), gs, _i(8), _p(0), _p(0), _p(A32), _i(256), S),
        (ERR_ARG, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(64), _p(A32), gs, _i(8), _p(0), _p(A32), _p(A32), _i(64), S),
        (ERR_ALIGN, "nvfp4_w4a16_linear", _p(A32), _i(4), _i(64), _p(A32), gs, _i(8), _p(0), _p(A32), _p(A32 + 128),
         _i(256), S),
        (ERR_SHAPE, "nvfp4_w4a16_pack", _p(A32), _p(A32), _i(8), _i(40), _p(A32), S),
        (ERR_NULL, "nvfp4_w4a16_pack", _p(A32), _p(0), _i(8), _i(64), _p(A32), S),
        (ERR_ALIGN, "nvfp4_w4a16_pack", _p(A32), _p(A32), _i(8), _i(64), _p(A8), S),
        (NVFP4_OK, "nvfp4_w4a16_pack", _p(0), _p(0), _i(0), _i(64), _p(0), S),
        # W4A16 self-test: x, M, K, tiled, gs, N, y, workspace, bytes, timeout_us
        (ERR_ARG, "nvfp4_w4a16_selftest_timeout", _p(A32), _i(4), _i(64), _p(A32), gs, _i(8), _p(A32), _p(A32),
         _i(256), ctypes.c_uint32(0), S),
        (ERR_ARG, "nvfp4_w4a16_selftest_timeout", _p(A32), _i(0), _i(64), _p(A32), gs, _i(8), _p(A32), _p(A32),
         _i(256), ctypes.c_uint32(1000), S),
        # fused quantize: x, M, N, amax, packed, scales, gs, workspace
        (ERR_NULL, "nvfp4_quantize_fused", _p(A32), _i(2), _i(16), amax, _p(A32), _p(A32), gs, _p(0), S),
        (ERR_ALIGN, "nvfp4_quantize_fused", _p(A32), _i(2), _i(16), amax, _p(A32), _p(A32), gs, _p(A32 + 8), S),
        (ERR_SHAPE, "nvfp4_quantize_fused", _p(A32), _i(-2), _i(16), amax, _p(A32), _p(A32), gs, _p(A32), S),
        # running amax
        (ERR_NULL, "nvfp4_amax_accumulate", _p(A32), _i(16), _p(0), S),
        (ERR_ALIGN, "nvfp4_amax_accumulate", _p(A32), _i(16), _p(A32 + 2), S),
        (ERR_SHAPE, "nvfp4_amax_accumulate", _p(A32), _i(-3), amax, S),
        (NVFP4_OK, "nvfp4_amax_accumulate", _p(0), _i(0), amax, S),
        # amax
        (ERR_NULL, "nvfp4_amax", _p(A32), _i(16), _p(0), S),
        (ERR_NULL, "nvfp4_amax", _p(0), _i(16), amax, S),
        (ERR_SHAPE, "nvfp4_amax", _p(A32), _i(-5), amax, S),
        (ERR_ALIGN, "nvfp4_amax", _p(A8), _i(16), amax, S),
        (ERR_ALIGN, "nvfp4_amax", _p(A32), _i(16), _p(A32 + 1), S),
    ]
    for expect, name, *args in cases:
        assert _call(lib, name, *args) == expect, (name, expect)

    # observers: unknown kind, bad decay
    lib.nvfp4_observer_update.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_void_p]
    assert _call(lib, "nvfp4_observer_update", A32, A32 + 4, 7, 0.01, None) == ERR_ARG
    assert _call(lib, "nvfp4_observer_update", A32, A32 + 4, 1, float("nan"), None) == ERR_ARG
    assert _call(lib, "nvfp4_observer_update", A32, A32 + 4, 1, 1.5, None) == ERR_ARG
    assert _call(lib, "nvfp4_observer_update", None, A32 + 4, 0, 0.01, None) == ERR_NULL
    assert _call(lib, "nvfp4_observer_update", A32 + 1, A32 + 4, 0, 0.01, None) == ERR_ALIGN
    lib.nvfp4_observe_amax.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p]
    assert _call(lib, "nvfp4_observe_amax", A32, 16, A32 + 64, 3, 0.01, A32 + 68, None) == ERR_ARG
    assert _call(lib, "nvfp4_observe_amax", A32, 16, A32 + 64, 0, 0.01, None, None) == ERR_NULL

    # lists: k out of range, null arrays, bad member
    VP = ctypes.c_void_p
    xs = (VP * 2)(A32, A32 + 1024)
    ns = (ctypes.c_int64 * 2)(32, 48)
    assert _call(lib, "nvfp4_amax_multi", xs, ns, 0, amax, S) == ERR_ARG
    assert _call(lib, "nvfp4_amax_multi", xs, ns, 17, amax, S) == ERR_ARG
    assert _call(lib, "nvfp4_amax_multi", None, ns, 2, amax, S) == ERR_NULL
    bad = (VP * 2)(A32, A8)
    assert _call(lib, "nvfp4_amax_multi", bad, ns, 2, amax, S) == ERR_ALIGN
    Ms = (ctypes.c_int64 * 2)(2, -3)
    Ns = (ctypes.c_int64 * 2)(16, 24)
    assert _call(lib, "nvfp4_fake_quant_siblings", ctypes.c_int(2), xs, xs, Ms, Ns, amax, S) == ERR_SHAPE
    Ns2 = (ctypes.c_int64 * 2)(16, 32)
    assert _call(lib, "nvfp4_fake_quant_siblings", ctypes.c_int(2), xs, xs, Ms, Ns2, _p(0), S) == ERR_NULL
    assert _call(lib, "nvfp4_fake_quant_siblings", ctypes.c_int(0), xs, xs, Ms, Ns2, amax, S) == ERR_ARG

    # workspace variants: null or misaligned workspace
    assert _call(lib, "nvfp4_amax_ws", _p(A32), _i(16), amax, _p(0), S) == ERR_NULL
    assert _call(lib, "nvfp4_amax_ws", _p(A32), _i(16), amax, _p(A32 + 8), S) == ERR_ALIGN
    assert _call(lib, "nvfp4_amax_ws", _p(A8), _i(16), amax, _p(A32), S) == ERR_ALIGN
    lib.nvfp4_observe_amax_ws.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert _call(lib, "nvfp4_observe_amax_ws", A32, 16, A32 + 64, 1, 0.01, A32 + 68, None, None) == ERR_NULL
    assert _call(lib, "nvfp4_observe_amax_ws", A32, 16, A32 + 64, 1, -0.5, A32 + 68, A32, None) == ERR_ARG

    # fused calls
    assert _call(lib, "nvfp4_fake_quant_fused", _p(A32), _p(A32 + 4096), _i(4), _i(-24), amax, _p(A32 + 512), S) == ERR_SHAPE
    assert _call(lib, "nvfp4_fake_quant_fused", _p(A32), _p(A32 + 4096), _i(4), _i(16), amax, _p(0), S) == ERR_NULL
    assert _call(lib, "nvfp4_fake_quant_fused", _p(A32), _p(A32 + 32), _i(4), _i(16), amax, _p(A32 + 512), S) == ERR_ARG
    assert _call(lib, "nvfp4_fake_quant_fused", _p(A8), _p(A32 + 4096), _i(4), _i(16), amax, _p(A32 + 512), S) == ERR_ALIGN
    lib.nvfp4_observe_fake_quant.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p]
    assert _call(lib, "nvfp4_observe_fake_quant", A32, A32 + 4096, 4, 16, None, 1, 0.01, A32 + 64, A32 + 512, None) == ERR_NULL
    assert _call(lib, "nvfp4_observe_fake_quant", A32, A32 + 4096, 4, 16, A32 + 68, 9, 0.01, A32 + 64, A32 + 512, None) == ERR_ARG
    lib.nvfp4_selftest_barrier_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    assert _call(lib, "nvfp4_selftest_barrier_timeout", A32, A32 + 4096, 4, 16, A32 + 64, A32 + 512, 0, None) == ERR_ARG
    assert _call(lib, "nvfp4_selftest_barrier_timeout", A32, A32 + 4096, 4, 16, A32 + 64, A32 + 512, 10**6, None) == ERR_ARG
    assert _call(lib, "nvfp4_workspace_check", _p(0), S) == ERR_NULL

    assert lib.nvfp4_kernel_launch_count() == before


def test_binding_refuses_cpu_tensors():
    import torch
    from qat_nvfp4_b200 import nvfp4
    x = torch.zeros(4, 16, dtype=torch.bfloat16)
    amax = torch.ones(1)
    for call in (lambda: nvfp4.nvfp4_fake_quant(x, amax), lambda: nvfp4.nvfp4_amax(x),
                 lambda: nvfp4.nvfp4_quantize(x, amax)):
        with pytest.raises(RuntimeError, match="CUDA tensor"):
            call()



BIG_WS = 1 << 40


@pytest.mark.parametrize("M,N,K,ws,sms,want", [
    # a weight with at most one 128-row output tile per two SMs: up to 8 rows of x with room
    # for the partial sums take the small kernel, 16-row tiles of x, shared by
    # min(2 x SMs, items) CTAs (items: 128 weight rows x 128 of K) ...
    (1, 4096, 4096, BIG_WS, 148, ("small", 16, 296)),        # 32 x 32 items
    (8, 4096, 4096, BIG_WS, 148, ("small", 16, 296)),
    (8, 4096, 4096, BIG_WS, 132, ("small", 16, 264)),
    (8, 4096, 512, BIG_WS, 148, ("small", 16, 128)),         # 32 x 4 items: one CTA each
    (5, 13, 16, BIG_WS, 148, ("small", 16, 1)),              # one item
    (4, 9472, 4096, BIG_WS, 148, ("small", 16, 296)),        # 74 tiles: still one per two SMs
    # ... one row without that room the CUDA cores ...
    (1, 4096, 4096, 256, 148, ("cores", 1, 1)),
    (1, 4096, 14336, 256, 148, ("cores", 1, 1)),
    # ... and more rows the shared-memory weight, K split when the workspace has room
    # (148 SMs / 32 tiles = 4 CTAs per tile, at least 8 atoms each), up to 32 rows unsplit
    (9, 13, 16, BIG_WS, 148, ("shared", 128, 1)),
    (16, 4096, 4096, BIG_WS, 148, ("shared", 128, 4)),
    (16, 4096, 4096, BIG_WS, 132, ("shared", 128, 4)),
    (2, 4096, 4096, 256, 148, ("shared", 128, 1)),
    (3, 4096, 4096, 256, 148, ("shared", 128, 1)),
    (16, 4096, 4096, 256, 148, ("shared", 128, 1)),
    (33, 4096, 4096, 256, 148, ("tensor", 64, 1)),
    (100, 4096, 4096, 256, 148, ("tensor", 128, 1)),
    # a weight with more tiles (14336 x 4096: 112, 9600 x 4096: 75): up to 64 rows of x the
    # tensor-memory weight with 64-row tiles, whatever the workspace
    (1, 14336, 4096, BIG_WS, 148, ("tensor", 64, 1)),
    (1, 14336, 4096, 256, 148, ("tensor", 64, 1)),
    (2, 14336, 4096, BIG_WS, 148, ("tensor", 64, 1)),
    (8, 9600, 4096, BIG_WS, 148, ("tensor", 64, 1)),
    (17, 14336, 4096, BIG_WS, 148, ("tensor", 64, 1)),
    (32, 14336, 4096, BIG_WS, 148, ("tensor", 64, 1)),
    (64, 14336, 4096, 256, 148, ("tensor", 64, 1)),
    (8, 14336, 4096, BIG_WS, 264, ("small", 16, 528)),       # 112 tiles on 264 SMs: few
    # 65 to 128 rows of x on a weight with few tiles: split K in shared memory when the
    # workspace has room (148 SMs / 32 tiles = 4 CTAs per tile, at least 8 atoms each) ...
    (100, 4096, 4096, BIG_WS, 148, ("shared", 128, 4)),
    (100, 4096, 4096, BIG_WS, 132, ("shared", 128, 4)),
    # ... not with too little K to split (8 atoms), nor on a weight with 112 tiles (148 / 112 = 1)
    (100, 4096, 512, BIG_WS, 148, ("tensor", 128, 1)),
    (65, 14336, 4096, BIG_WS, 148, ("tensor", 128, 1)),
    (128, 14336, 4096, BIG_WS, 148, ("tensor", 128, 1)),
    # more rows: 256-row tiles unless 128-row tiles need no more waves of one CTA per SM
    (129, 4096, 4096, BIG_WS, 148, ("tensor", 128, 1)),      # 32 vs 64 tiles: one wave either way
    (512, 4096, 4096, BIG_WS, 148, ("tensor", 128, 1)),      # 64 vs 128 tiles: one wave either way
    (1024, 4096, 4096, BIG_WS, 148, ("tensor", 256, 1)),     # 128 tiles: 1 wave vs 2
    (4096, 4096, 4096, BIG_WS, 148, ("tensor", 256, 1)),     # 512 vs 1024 tiles: 4 waves vs 7
    (1024, 14336, 4096, BIG_WS, 148, ("tensor", 256, 1)),    # 448 vs 896 tiles: 4 waves vs 7
    (1024, 4096, 4096, BIG_WS, 64, ("tensor", 256, 1)),      # 2 waves vs 4
    (1024, 4096, 4096, BIG_WS, 512, ("tensor", 128, 1)),     # 1 wave either way
    (200, 18944, 64, BIG_WS, 148, ("tensor", 256, 1)),       # 148 tiles: 1 wave vs 2
])
def test_w4a16_plan(M, N, K, ws, sms, want):
    """Host-only: which kernel, tile height and K split nvfp4_w4a16_linear takes, from the
    rules stated in the header (worked out by hand here)."""
    from qat_nvfp4_b200 import nvfp4 as nv
    assert nv.nvfp4_w4a16_plan(M, N, K, ws, sms) == want


def test_w4a16_plan_refusals(lib):
    f = lib.nvfp4_w4a16_plan
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int] + [ctypes.POINTER(ctypes.c_int)] * 3
    k, r, s = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    out = (ctypes.byref(k), ctypes.byref(r), ctypes.byref(s))
    assert f(16, 4096, 4096, 256, 148, *out) == NVFP4_OK
    assert f(16, 4096, 4096, 256, 0, *out) == ERR_ARG
    assert f(16, 4096, 24, 256, 148, *out) == ERR_SHAPE
    assert f(-1, 4096, 4096, 256, 148, *out) == ERR_SHAPE
    assert f(16, 4096, 4096, 256, 148, None, ctypes.byref(r), ctypes.byref(s)) == ERR_NULL


def test_w4a16_workspace_sizes(lib):
    """Host-only (148 SMs assumed without a GPU): for the small kernel (up to 8 rows of x on a
    weight with at most 74 output tiles) the status block, one counter per 128-row tile
    (rounded up to 256 bytes) and 2 x G x 128 x 16 fp32 partial sums (two slots per CTA),
    G = min(296, items); for a split K (65 to 128
    rows) the block, the counters and splits x tiles x 128 x 128 fp32 partial sums; otherwise
    the block alone."""
    f = lib.nvfp4_w4a16_workspace_bytes
    f.restype = ctypes.c_int64
    f.argtypes = [ctypes.c_int64] * 3

    def head(tiles):
        return -(-(256 + 4 * tiles) // 256) * 256

    assert f(1, 4096, 4096) == head(32) + 2 * 296 * 128 * 16 * 4
    assert f(8, 4096, 4096) == head(32) + 2 * 296 * 128 * 16 * 4
    assert f(2, 14336, 4096) == 256        # 112 tiles: the tensor-memory weight, nothing to split
    assert f(4, 4096, 14336) == head(32) + 2 * 296 * 128 * 16 * 4  # the down-projection: 32 tiles
    assert f(8, 4096, 512) == head(32) + 2 * 128 * 128 * 16 * 4   # 128 items: 128 CTAs
    assert f(17, 14336, 4096) == 256       # 112 tiles: not split
    assert f(16, 4096, 4096) == head(32) + 4 * 32 * 128 * 128 * 4     # split K, 4 CTAs per tile
    assert f(200, 4096, 4096) == 256        # tensor memory: never split
    assert f(100, 14336, 4096) == 256       # 112 tiles: 148 // 112 = 1 CTA per tile
    assert f(100, 4096, 4096) == head(32) + 4 * 32 * 128 * 128 * 4    # 4 splits, K has 64 atoms
    assert f(100, 4096, 1088) == head(32) + 2 * 32 * 128 * 128 * 4    # 17 atoms: 2
    assert f(16, 4096, 24) == -1 and f(-1, 4096, 64) == -1


def test_w4a16_record_sizes(lib):
    """Host-only: ceil(N / 128) * ceil(K / 64) records of 4608 bytes; refused shapes -> -1."""
    f = lib.nvfp4_w4a16_tiled_bytes
    f.restype = ctypes.c_int64
    f.argtypes = [ctypes.c_int64, ctypes.c_int64]
    for N, K in [(1, 16), (128, 64), (129, 64), (128, 65 - 1 + 16), (14336, 4096), (0, 16)]:
        assert f(N, K) == -(-N // 128) * -(-K // 64) * 4608
    for N, K in [(8, 0), (8, 24), (-1, 64), (8, -16)]:
        assert f(N, K) == -1
