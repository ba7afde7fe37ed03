"""Parity of the fp32-scale flavour (blocks of 32 with the block scale kept in fp32, which
VideoX-Fun's fp4_optimization.py constants block names as the OCP MXFP4 flavour) with the
CPU oracle, bit for bit: 0 ULP on every code byte, every fp32 scale (compared as bits) and
every bf16 output.  Shapes cover whole-block rows (the streaming kernels) and rows of any
other length (the staged kernels), several tiles with a ragged tail, the full bf16 range,
blocks that take the IEEE-division path, arbitrary stored scales, and the 14336 x 4096
weight and the 65536 x 8192 activation in full.
"""
import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import (assert_equal_bits, bits, oracle_dequantize_f32s_rows, oracle_quantize_f32s_rows, to_dev,
                            u8, u8_to_dev)

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("qat_nvfp4_b200.nvfp4")


def _f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def _check(x_bits, what=""):
    """quantize, dequantize, fake-quant (out of place and in place) against the oracle on the
    whole tensor."""
    M, N = x_bits.shape
    xd = to_dev(x_bits)
    packed_d, scales_d = nv.nvfp4_quantize_f32scale(xd)
    P = 32 * ((N + 31) // 32)
    assert tuple(packed_d.shape) == (M, P // 2) and tuple(scales_d.shape) == (M, P // 32)
    assert scales_d.dtype == torch.float32
    packed, scales = oracle_quantize_f32s_rows(x_bits)
    assert_equal_bits(_f32_bits(scales_d.cpu().numpy()), _f32_bits(scales), f"{what}: fp32 scales")
    assert_equal_bits(u8(packed_d), packed, f"{what}: packed codes")
    y = oracle_dequantize_f32s_rows(packed, scales, N)
    assert_equal_bits(bits(nv.nvfp4_dequantize_f32scale(packed_d, scales_d, n_cols=N)), y, f"{what}: dequantize")
    assert_equal_bits(bits(nv.nvfp4_fake_quant_f32scale(xd)), y, f"{what}: fake-quant")
    nv.nvfp4_fake_quant_f32scale(xd, out=xd)
    assert_equal_bits(bits(xd), y, f"{what}: fake-quant in place")
    return packed, scales, y


def test_oracle_wrapper_agrees_with_the_fake_quant_composition():
    x = synthetic.activation_normal((64, 96), 77)
    p, s = oracle.quantize_f32scale(x)
    assert np.array_equal(oracle.fake_quant_f32scale(x), oracle.dequantize_f32scale(p, s, 64, 96))


@pytest.mark.parametrize("M,N", [(1, 32), (256, 1024), (37, 96), (4099, 1056), (2, 32 * 1024 + 32)])
def test_whole_block_rows(M, N):
    _check(synthetic.activation_normal((M, N), 9100 + M + N), what=f"{M}x{N}")


@pytest.mark.parametrize("M,N", [(1, 1), (5, 15), (3, 16), (3, 48), (7, 20), (17, 1000), (255, 4097),
                                 (64, 8191), (2, 33), (4096, 1008), (1000, 80)])
def test_ragged_rows(M, N):
    rng = np.random.default_rng(M * 317 + N)
    _check(synthetic.to_bf16_bits(rng.standard_t(3, (M, N)).astype(np.float32)), what=f"{M}x{N} ragged")


def test_weight_with_outliers():
    _check(synthetic.weight_with_outliers(), what="weight with outliers")


def test_random_bit_patterns_full_range():
    """Every finite bf16 bit pattern class: subnormals, huge values (block amax above
    393216, where the element quotient takes the IEEE division), signed zeros."""
    rng = np.random.default_rng(331)
    raw = rng.integers(0, 1 << 16, size=(512, 1024), dtype=np.uint32).astype(np.uint16)
    finite = (raw & 0x7F80) != 0x7F80
    _check(np.where(finite, raw, raw & 0x807F), what="random bf16 bits")


def test_zero_tiny_and_huge_blocks():
    """Blocks of +-0 only (scale 0, divisor 1e-12, codes 0 or 8 by sign), blocks of
    subnormal bf16 values (scale below 1e-12: the divisor clamp decides), blocks around the
    fast-path guard (amax 393216 = 6 * 2^16) and at the top of the bf16 range."""
    M, N = 8, 32 * 6
    x = np.zeros((M, N), dtype=np.float32)
    rng = np.random.default_rng(332)
    x[:, 32:64] = rng.uniform(-1, 1, (M, 32)) * 2.0 ** -130                     # subnormal bf16
    x[:, 64:96] = rng.uniform(-1, 1, (M, 32)) * 2.0 ** -100                     # scale ~1e-31 < 1e-12
    x[:, 96:128] = rng.uniform(-1, 1, (M, 32)) * 393216.0
    x[:, 96] = 393216.0
    x[:, 128:160] = rng.uniform(-1, 1, (M, 32)) * 3.0e38
    x[:, 160:192] = rng.uniform(-1, 1, (M, 32)) * 393215.0
    bits_ = synthetic.to_bf16_bits(x.astype(np.float32))
    bits_[::2, :32] = 0x8000                                                     # -0.0 blocks
    _check(bits_, what="edge blocks")


def test_dequantize_arbitrary_bytes_and_scales():
    """Any code byte and any finite fp32 scale (negative, zero, subnormal, huge) decodes as
    bf16(LUT * scale)."""
    rng = np.random.default_rng(333)
    M, N = 256, 512
    packed = rng.integers(0, 256, size=(M, N // 2), dtype=np.uint8)
    mant = rng.uniform(-2, 2, size=(M, N // 32))
    expo = rng.integers(-149, 125, size=(M, N // 32))
    scales = (mant * np.exp2(expo.astype(np.float64))).astype(np.float32)
    scales[0, :4] = [0.0, -0.0, 1.4e-45, 3.0e38]
    got = nv.nvfp4_dequantize_f32scale(u8_to_dev(packed), torch.from_numpy(scales).cuda(), n_cols=N)
    want = oracle.dequantize_f32scale(packed, scales, M, N)
    assert_equal_bits(bits(got), want, "arbitrary bytes and fp32 scales")


def test_power_of_two_scaling_keeps_codes():
    """A property that holds at any size: x * 2^k (no overflow or subnormals on either side)
    gives the same codes and scales * 2^k."""
    rng = np.random.default_rng(334)
    x = rng.standard_normal((1024, 2048)).astype(np.float32)
    a, b = synthetic.to_bf16_bits(x), synthetic.to_bf16_bits(x * np.float32(2.0 ** 20))
    pa, sa = nv.nvfp4_quantize_f32scale(to_dev(a))
    pb, sb = nv.nvfp4_quantize_f32scale(to_dev(b))
    assert torch.equal(pa, pb)
    assert torch.equal(sa * 2.0 ** 20, sb)


@pytest.mark.parametrize("M,N", [(3, 20), (255, 4097), (1000, 48)])
def test_outputs_stay_inside_their_tensor(M, N):
    rng = np.random.default_rng(M + 13 * N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    xd = to_dev(x)
    pad = 64
    buf = torch.zeros((pad + M * N + pad,), dtype=torch.int16, device="cuda")
    buf.view(torch.uint8).fill_(0xA5)
    y = buf[pad:pad + M * N].view(torch.bfloat16).view(M, N)
    nv.nvfp4_fake_quant_f32scale(xd, out=y)
    p, s = nv.nvfp4_quantize_f32scale(xd)
    want = oracle.fake_quant_f32scale(x)
    for what in ("fake-quant", "dequantize"):
        head = buf[:pad].view(torch.uint8).cpu().numpy()
        tail = buf[pad + M * N:].view(torch.uint8).cpu().numpy()
        assert (head == 0xA5).all() and (tail == 0xA5).all(), f"{what} wrote outside y"
        assert_equal_bits(bits(y), want, what)
        buf.view(torch.uint8).fill_(0xA5)
        nv.nvfp4_dequantize_f32scale(p, s, n_cols=N, out=y)


def test_alignment_is_checked():
    x = to_dev(synthetic.activation_normal((4, 64), 5))
    raw = torch.empty(4 * 32 + 8, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        nv.nvfp4_quantize_f32scale(x, packed=raw[8:].view(4, 32))  # 8-byte but not 16-byte aligned


def test_full_weight_14336x4096():
    """The 14336 x 4096 MLP weight: every code byte, fp32 scale and output element."""
    xd = synthetic.activation_normal_device((14336, 4096), 103, "cuda") * 0.02
    _check(bits(xd), what="14336x4096 weight")


def test_full_activation_65536x8192():
    """The 65536 x 8192 bf16 activation (1 GiB): quantize and fake-quant in full."""
    M, N = 65536, 8192
    xd = synthetic.activation_normal_device((M, N), 424243, "cuda")
    x = bits(xd)
    packed_d, scales_d = nv.nvfp4_quantize_f32scale(xd)
    packed, scales = oracle_quantize_f32s_rows(x)
    assert_equal_bits(_f32_bits(scales_d.cpu().numpy()), _f32_bits(scales), "1 GiB: fp32 scales")
    assert_equal_bits(u8(packed_d), packed, "1 GiB: packed codes")
    del packed_d, scales_d
    y = oracle_dequantize_f32s_rows(packed, scales, N)
    assert_equal_bits(bits(nv.nvfp4_fake_quant_f32scale(xd)), y, "1 GiB: fake-quant")
