"""Parity of the block-32 variant (the ``block_size`` argument of VideoX-Fun's
fp4_optimization.py quantize_weight_to_float4 set to 32) with the CPU oracle, bit for bit.

Same tolerance as block 16: 0 ULP on codes, scale bytes, the global scale and every bf16
output.  Shapes cover aligned rows (N % 32 == 0), rows that are a multiple of 16 but not
of 32 (aligned for block 16, ragged for block 32), ragged rows, several tiles with a
ragged tail, and the full 65536 x 8192 activation on sampled rows.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import (assert_equal_bits, bits, f32_bits, oracle_dequantize_rows, oracle_fake_quant_rows,
                            oracle_quantize_rows, scalar, to_dev, u8, u8_to_dev)

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("qat_nvfp4_b200.nvfp4")

B32 = 32


def _full_check32(x_bits, amax_value=None, what=""):
    """amax (unless given), quantize, dequantize, fake-quant (out of place and in place)
    with blocks of 32, against the oracle on the whole tensor."""
    M, N = x_bits.shape
    xd = to_dev(x_bits)
    if amax_value is None:
        amax_d = nv.nvfp4_amax(xd)
        a = oracle.amax(x_bits)
        assert f32_bits(amax_d) == f32_bits(a), f"{what}: amax"
    else:
        amax_d = scalar(amax_value)
        a = amax_value
    gs = oracle.global_scale(a)
    packed_d, scales_d, gs_d = nv.nvfp4_quantize(xd, amax_d, block=B32)
    assert f32_bits(gs_d) == f32_bits(gs), f"{what}: global scale"
    P = B32 * ((N + B32 - 1) // B32)
    assert tuple(packed_d.shape) == (M, P // 2) and tuple(scales_d.shape) == (M, P // B32)
    packed, scales = oracle_quantize_rows(x_bits, gs, block=B32)
    assert_equal_bits(u8(scales_d), scales, f"{what}: scale bytes")
    assert_equal_bits(u8(packed_d), packed, f"{what}: packed codes")
    y_d = nv.nvfp4_dequantize(packed_d, scales_d, gs_d, n_cols=N, block=B32)
    y = oracle_dequantize_rows(packed, scales, gs, n_cols=N, block=B32)
    assert_equal_bits(bits(y_d), y, f"{what}: dequantize")
    assert_equal_bits(bits(nv.nvfp4_fake_quant(xd, amax_d, block=B32)), y, f"{what}: fake-quant")
    nv.nvfp4_fake_quant(xd, amax_d, out=xd, block=B32)
    assert_equal_bits(bits(xd), y, f"{what}: fake-quant in place")
    return packed, scales, y


def test_worked_block32_example_gpu(golden_dir):
    with open(os.path.join(golden_dir, "worked_examples.json")) as f:
        cases = [c for c in json.load(f)["cases"] if c.get("block", 16) == B32]
    assert cases, "the fixtures hold a block-32 case"
    for case in cases:
        M, N = case["rows"], case["cols"]
        x = synthetic.to_bf16_bits(np.array(case["x"], dtype=np.float32).reshape(M, N))
        xd = to_dev(x)
        amax_d = nv.nvfp4_amax(xd) if case["amax"] == "tensor" else scalar(case["amax"])
        packed_d, scales_d, gs_d = nv.nvfp4_quantize(xd, amax_d, block=B32)
        if "global_scale" in case:
            assert gs_d.item() == case["global_scale"]
        assert list(u8(scales_d).ravel()) == case["scales"], case["name"]
        assert list(u8(packed_d).ravel()) == case["packed"], case["name"]
        expect = synthetic.to_bf16_bits(np.array(case["dequant"], dtype=np.float32).reshape(M, N))
        assert_equal_bits(bits(nv.nvfp4_dequantize(packed_d, scales_d, gs_d, n_cols=N, block=B32)), expect,
                          case["name"])
        assert_equal_bits(bits(nv.nvfp4_fake_quant(xd, amax_d, block=B32)), expect, case["name"])


@pytest.mark.parametrize("M,N", [(1, 32), (256, 1024), (37, 96), (4099, 1056), (2, 32 * 1024 + 32)])
def test_aligned_rows(M, N):
    x = synthetic.activation_normal((M, N), 9000 + M + N)
    _full_check32(x, what=f"{M}x{N}")


@pytest.mark.parametrize("M,N", [(1, 1), (5, 15), (3, 16), (3, 48), (7, 20), (17, 1000), (255, 4097),
                                 (64, 8191), (2, 33), (4096, 1008), (1000, 80)])
def test_ragged_rows(M, N):
    rng = np.random.default_rng(M * 313 + N)
    x = synthetic.to_bf16_bits(rng.standard_t(3, (M, N)).astype(np.float32))
    _full_check32(x, what=f"{M}x{N} ragged")


def test_weight_with_outliers():
    x = synthetic.weight_with_outliers()
    _full_check32(x, what="weight with outliers")


def test_random_bit_patterns_full_range():
    rng = np.random.default_rng(321)
    raw = rng.integers(0, 1 << 16, size=(512, 1024), dtype=np.uint32).astype(np.uint16)
    finite = (raw & 0x7F80) != 0x7F80
    raw = np.where(finite, raw, raw & 0x807F)
    _full_check32(raw, what="random bf16 bits")
    for a in (1.0, 1e-30, 3.0e38, 7.5e-9):
        _full_check32(raw[:64], amax_value=a, what=f"random bits, amax {a}")


def test_wide_dynamic_range_blocks():
    rng = np.random.default_rng(322)
    M, N = 256, 512
    centre = rng.integers(-120, 120, size=(M, N // B32, 1))
    spread = rng.integers(0, 60, size=(M, N // B32, B32))
    mant = rng.uniform(1, 2, size=(M, N // B32, B32))
    sign = rng.choice([-1.0, 1.0], size=(M, N // B32, B32))
    vals = sign * mant * np.exp2(np.clip(centre - spread, -133, 127))
    x = synthetic.to_bf16_bits(vals.reshape(M, N).astype(np.float32))
    _full_check32(x, what="wide dynamic range")
    _full_check32(x, amax_value=1e-3, what="wide dynamic range, small amax")


def test_equal_halves_match_block16():
    """A block of 32 made of two identical halves has the block amax of each half, so its
    codes and outputs equal those of blocks of 16 (a property that holds at any size)."""
    rng = np.random.default_rng(323)
    half = synthetic.to_bf16_bits(rng.standard_normal((512, 2048)).astype(np.float32))
    x = np.repeat(half.reshape(512, -1, 1, 16), 2, axis=2).reshape(512, 4096)
    xd = to_dev(x)
    a = nv.nvfp4_amax(xd)
    y16 = nv.nvfp4_fake_quant(xd, a)
    y32 = nv.nvfp4_fake_quant(xd, a, block=B32)
    assert torch.equal(y16.view(torch.int16), y32.view(torch.int16))
    p16, s16, _ = nv.nvfp4_quantize(xd, a)
    p32, s32, _ = nv.nvfp4_quantize(xd, a, block=B32)
    assert torch.equal(p16, p32)
    assert torch.equal(s16[:, ::2], s32) and torch.equal(s16[:, 1::2], s32)


def test_dequantize_arbitrary_scale_bytes():
    rng = np.random.default_rng(329)
    M, N = 256, 512
    packed = rng.integers(0, 256, size=(M, N // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(M, N // B32), dtype=np.uint8)
    scales[(scales & 0x7F) == 0x7F] = 0x3C  # NaN bytes are outside the method
    gs = np.float32(7168.0)
    got = nv.nvfp4_dequantize(u8_to_dev(packed), u8_to_dev(scales), scalar(float(gs)), block=B32)
    want = oracle_dequantize_rows(packed, scales, float(gs), block=B32)
    assert_equal_bits(bits(got), want, "arbitrary bytes, block 32")


@pytest.mark.parametrize("M,N", [(3, 20), (255, 4097), (1000, 48)])
def test_ragged_outputs_stay_inside_their_tensor(M, N):
    rng = np.random.default_rng(M + 11 * N)
    x = synthetic.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    xd = to_dev(x)
    a = nv.nvfp4_amax(xd)
    pad = 64
    buf = torch.zeros((pad + M * N + pad,), dtype=torch.int16, device="cuda")
    buf.view(torch.uint8).fill_(0xA5)
    y = buf[pad:pad + M * N].view(torch.bfloat16).view(M, N)
    nv.nvfp4_fake_quant(xd, a, out=y, block=B32)
    p, s, gs = nv.nvfp4_quantize(xd, a, block=B32)
    want = oracle_fake_quant_rows(x, a.item(), block=B32)
    for what in ("fake-quant", "dequantize"):
        head = buf[:pad].view(torch.uint8).cpu().numpy()
        tail = buf[pad + M * N:].view(torch.uint8).cpu().numpy()
        assert (head == 0xA5).all() and (tail == 0xA5).all(), f"{what} wrote outside y"
        assert_equal_bits(bits(y), want, what)
        buf.view(torch.uint8).fill_(0xA5)
        nv.nvfp4_dequantize(p, s, gs, out=y, n_cols=N, block=B32)


def test_packed_alignment_is_checked():
    x = to_dev(synthetic.activation_normal((4, 64), 5))
    a = nv.nvfp4_amax(x)
    raw = torch.empty(4 * 32 + 8, dtype=torch.uint8, device="cuda")
    packed = raw[8:].view(4, 32)  # 8-byte but not 16-byte aligned
    scales = torch.empty((4, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        nv.nvfp4_quantize(x, a, packed=packed, scales=scales, block=B32)
    with pytest.raises(ValueError):
        nv.nvfp4_fake_quant(x, a, block=64)


def test_ste_block32():
    x = to_dev(synthetic.activation_normal((64, 256), 6)).requires_grad_(True)
    a = nv.nvfp4_amax(x.detach())
    y = nv.fake_quant_ste(x, a, block=B32)
    g = torch.randn_like(y)
    y.backward(g)
    assert torch.equal(x.grad.view(torch.int16), g.view(torch.int16))
    want = oracle_fake_quant_rows(bits(x.detach()), a.item(), block=B32)
    assert_equal_bits(bits(y.detach()), want, "STE forward, block 32")


def test_full_activation():
    """The 65536 x 8192 bf16 activation (1 GiB): amax over all of it, every code byte,
    scale byte, dequantized and fake-quantized element against the oracle."""
    M, N = 65536, 8192
    xd = synthetic.activation_normal_device((M, N), 424242, "cuda")
    amax_d = nv.nvfp4_amax(xd)
    x = bits(xd)
    assert f32_bits(amax_d) == f32_bits(oracle.amax(x))
    gs = oracle.global_scale(amax_d.item())
    packed_d, scales_d, gs_d = nv.nvfp4_quantize(xd, amax_d, block=B32)
    assert f32_bits(gs_d) == f32_bits(gs)
    packed, scales = oracle_quantize_rows(x, gs, block=B32)
    assert_equal_bits(u8(packed_d), packed, "1 GiB block 32: packed")
    assert_equal_bits(u8(scales_d), scales, "1 GiB block 32: scales")
    y = oracle_dequantize_rows(packed, scales, gs, block=B32)
    assert_equal_bits(bits(nv.nvfp4_dequantize(packed_d, scales_d, gs_d, block=B32)), y,
                      "1 GiB block 32: dequantize")
    del packed_d, scales_d
    assert_equal_bits(bits(nv.nvfp4_fake_quant(xd, amax_d, block=B32)), y, "1 GiB block 32: fake-quant")
