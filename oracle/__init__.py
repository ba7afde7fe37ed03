"""CPU oracle for the NVFP4 quantize / fake-quantize path -- TEST INFRASTRUCTURE ONLY.

Thin numpy/ctypes wrapper around ``nvfp4_oracle.c`` (plain scalar C, fp32 IEEE with one
rounding per operation).  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the GPU library never uses it and
shares no code with it.

Tensors are passed as numpy arrays of raw bits: bf16 as ``uint16``, packed nibbles,
and E4M3 scale bytes as ``uint8``.  Sources cited in the C file: fp4_optimization.py
(VideoX-Fun) for the quantize / dequantize math, and the verl ``linear.py`` tutorial
for the fake-quant, STE, sibling fusion and activation observers.
"""
import ctypes
import os

import numpy as np

from .build import build_oracle

_LIB = None

STATIC_MINMAX = 0
EMA = 1


def _lib():
    global _LIB
    if _LIB is None:
        # NVFP4_ORACLE_LIB points at another build of the same source; the mutation test
        # uses it to check that the pins reject deliberately broken copies of the oracle.
        path = os.environ.get("NVFP4_ORACLE_LIB") or build_oracle()
        lib = ctypes.CDLL(path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i64 = ctypes.c_int64
        f32 = ctypes.c_float
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = f32
        lib.oracle_f32_to_bf16.argtypes = [f32]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = f32
        lib.oracle_e4m3_encode.argtypes = [f32]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e2m1_round_index.argtypes = [f32]
        lib.oracle_e2m1_round_index.restype = ctypes.c_int
        lib.oracle_e2m1_lut.argtypes = [ctypes.c_int]
        lib.oracle_e2m1_lut.restype = f32
        lib.oracle_amax.argtypes = [u16p, i64]
        lib.oracle_amax.restype = f32
        lib.oracle_amax_multi.argtypes = [ctypes.POINTER(u16p), ctypes.POINTER(i64), ctypes.c_int]
        lib.oracle_amax_multi.restype = f32
        lib.oracle_global_scale.argtypes = [f32]
        lib.oracle_global_scale.restype = f32
        lib.oracle_quantize.argtypes = [u16p, i64, i64, f32, u8p, u8p]
        lib.oracle_quantize.restype = None
        lib.oracle_dequantize.argtypes = [u8p, u8p, f32, i64, i64, u16p]
        lib.oracle_dequantize.restype = None
        lib.oracle_fake_quant.argtypes = [u16p, i64, i64, f32, u16p]
        lib.oracle_fake_quant.restype = ctypes.c_int
        lib.oracle_quantize_bs.argtypes = [u16p, i64, i64, i64, f32, u8p, u8p]
        lib.oracle_quantize_bs.restype = ctypes.c_int
        lib.oracle_dequantize_bs.argtypes = [u8p, u8p, f32, i64, i64, i64, u16p]
        lib.oracle_dequantize_bs.restype = ctypes.c_int
        lib.oracle_fake_quant_bs.argtypes = [u16p, i64, i64, i64, f32, u16p]
        lib.oracle_fake_quant_bs.restype = ctypes.c_int
        f32p = ctypes.POINTER(ctypes.c_float)
        lib.oracle_quantize_f32scale.argtypes = [u16p, i64, i64, u8p, f32p]
        lib.oracle_quantize_f32scale.restype = ctypes.c_int
        lib.oracle_dequantize_f32scale.argtypes = [u8p, f32p, i64, i64, u16p]
        lib.oracle_dequantize_f32scale.restype = None
        lib.oracle_fake_quant_f32scale.argtypes = [u16p, i64, i64, u16p]
        lib.oracle_fake_quant_f32scale.restype = ctypes.c_int
        lib.oracle_observer_update.argtypes = [f32, f32, ctypes.c_int, ctypes.c_double]
        lib.oracle_observer_update.restype = f32
        _LIB = lib
    return _LIB


def _u16(a):
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))


def _u8(a):
    a = np.ascontiguousarray(a, dtype=np.uint8)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def f32(v) -> float:
    """Round a Python number to the nearest fp32 and return it as a Python float."""
    return float(np.float32(v))


# ---- scalar codecs ------------------------------------------------------------------

def bf16_to_f32(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(values):
    """Round fp32 values to bf16 bits, one at a time through the oracle."""
    v = np.asarray(values, dtype=np.float32).ravel()
    lib = _lib()
    out = np.array([lib.oracle_f32_to_bf16(float(x)) for x in v], dtype=np.uint16)
    return out.reshape(np.shape(values))


def e4m3_decode(codes):
    lib = _lib()
    c = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.oracle_e4m3_decode(int(x)) for x in c], dtype=np.float32).reshape(np.shape(codes))


def e4m3_encode(values):
    lib = _lib()
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib.oracle_e4m3_encode(float(x)) for x in v], dtype=np.uint8).reshape(np.shape(values))


def e2m1_round_index(values):
    lib = _lib()
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib.oracle_e2m1_round_index(float(x)) for x in v], dtype=np.int32).reshape(np.shape(values))


def e2m1_lut(code: int) -> float:
    return _lib().oracle_e2m1_lut(int(code))


# ---- the method -----------------------------------------------------------------------

def amax(x_bits) -> float:
    a, p = _u16(x_bits)
    return _lib().oracle_amax(p, a.size)


def amax_multi(xs_bits) -> float:
    arrs = [_u16(x) for x in xs_bits]
    u16p = ctypes.POINTER(ctypes.c_uint16)
    ptrs = (u16p * len(arrs))(*[p for _, p in arrs])
    ns = (ctypes.c_int64 * len(arrs))(*[a.size for a, _ in arrs])
    return _lib().oracle_amax_multi(ptrs, ns, len(arrs))


def global_scale(amax_value: float) -> float:
    return _lib().oracle_global_scale(f32(amax_value))


def padded_blocks(N: int, block: int = 16) -> int:
    """Blocks per row: ceil(N / block) (rows are zero-padded to a multiple of block)."""
    return (N + block - 1) // block


def quantize(x_bits, global_scale_value: float, block: int = 16):
    """x_bits: uint16 [M, N].  Returns (packed [M, B*block/2], scales [M, B]),
    B = ceil(N / block)."""
    a, p = _u16(x_bits)
    M, N = a.shape
    B = padded_blocks(N, block)
    packed = np.empty((M, B * block // 2), dtype=np.uint8)
    scales = np.empty((M, B), dtype=np.uint8)
    rc = _lib().oracle_quantize_bs(p, M, N, block, f32(global_scale_value),
                                   packed.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                   scales.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    if rc != 0:
        raise ValueError(f"oracle_quantize_bs failed (block {block})")
    return packed, scales


def dequantize(packed, scales, global_scale_value: float, M: int, N: int, block: int = 16):
    pk, pp = _u8(packed)
    sc, sp = _u8(scales)
    y = np.empty((M, N), dtype=np.uint16)
    rc = _lib().oracle_dequantize_bs(pp, sp, f32(global_scale_value), M, N, block,
                                     y.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    if rc != 0:
        raise ValueError(f"oracle_dequantize_bs failed (block {block})")
    return y


def fake_quant(x_bits, amax_value: float, block: int = 16):
    a, p = _u16(x_bits)
    M, N = a.shape
    y = np.empty((M, N), dtype=np.uint16)
    rc = _lib().oracle_fake_quant_bs(p, M, N, block, f32(amax_value),
                                     y.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    if rc != 0:
        raise ValueError(f"oracle_fake_quant_bs failed (block {block})")
    return y


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 values (exact: bf16 is the top half of an fp32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def w4a16_linear(x_bits, packed, scales, global_scale_value: float, n_out: int, block: int = 16,
                 bias_bits=None):
    """The forward of a Linear layer whose weight is stored packed ([FP4OPT]
    _float4_autocast_forward): for the duration of one forward the packed weight is replaced
    by dequantize_weight_from_float4(...) in bf16, and the layer's own forward
    y = x W^T (+ bias) runs on it.

    x_bits: uint16 [M, K] (bf16 activations); packed / scales: the weight [n_out, K] as
    quantize() returns it; bias_bits: optional uint16 [n_out].  Returns float64 [M, n_out]:
    the exact products (a product of two bf16 values is exact in float64) summed by a
    library float64 matmul, before the forward's rounding of its output to bf16.  Rows are
    independent, so the caller may pass any subset of activation rows."""
    x = bf16_to_f64(x_bits)
    M, K = x.shape
    w = bf16_to_f64(dequantize(packed, scales, global_scale_value, n_out, K, block))
    y = x @ w.T
    if bias_bits is not None:
        y = y + bf16_to_f64(np.asarray(bias_bits).reshape(1, n_out))
    return y


def quantize_f32scale(x_bits):
    """The fp32-scale flavour with blocks of 32 (fp4_optimization.py, constants block):
    bf16 bits [M, N] -> (packed uint8 [M, P/2], fp32 block scales [M, P/32]),
    P = 32 ceil(N / 32)."""
    x, xp = _u16(x_bits)
    M, N = x.shape
    B = padded_blocks(N, 32)
    packed = np.empty((M, 16 * B), dtype=np.uint8)
    scales = np.empty((M, B), dtype=np.float32)
    rc = _lib().oracle_quantize_f32scale(xp, M, N, packed.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                         scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    if rc != 0:
        raise MemoryError("oracle_quantize_f32scale")
    return packed, scales


def dequantize_f32scale(packed, scales, M: int, N: int):
    """packed [M, P/2] + fp32 scales [M, P/32] -> bf16 bits [M, N]."""
    p, pp = _u8(packed)
    s = np.ascontiguousarray(scales, dtype=np.float32)
    y = np.empty((M, N), dtype=np.uint16)
    _lib().oracle_dequantize_f32scale(pp, s.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), M, N,
                                      y.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    return y


def fake_quant_f32scale(x_bits):
    """dequantize_f32scale(quantize_f32scale(x)), bf16 bits [M, N] -> bf16 bits [M, N]."""
    x, xp = _u16(x_bits)
    M, N = x.shape
    y = np.empty((M, N), dtype=np.uint16)
    if _lib().oracle_fake_quant_f32scale(xp, M, N, y.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))) != 0:
        raise MemoryError("oracle_fake_quant_f32scale")
    return y


def observer_update(state: float, cur: float, kind: int, decay: float = 0.01) -> float:
    return _lib().oracle_observer_update(f32(state), f32(cur), int(kind), float(decay))


def library_path() -> str:
    return os.path.abspath(build_oracle())
