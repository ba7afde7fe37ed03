"""Quantizing straight into the block-scaled tensor-core GEMM layout.

1. The scale bytes of nvfp4_quantize_mma are the oracle's row-major scales moved to the
   128 x 4 tile layout (the permutation below is written from the layout's definition),
   with zeros in the padding; codes are those of nvfp4_quantize.
2. The hardware is the authority on the layout: the block-scaled FP4 GEMM of the
   library (torch.nn.functional.scaled_mm on the tensor cores, two-level NVFP4 recipe)
   run on our packed codes and scales must reproduce an fp64 product of the operands
   decoded by the oracle, within the error of fp32 accumulation and a bf16 result.  Row-
   major scales passed in their place must not.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from qat_nvfp4_b200 import synthetic
from nvfp4_testutil import assert_equal_bits, oracle_quantize_rows, to_dev, u8

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("qat_nvfp4_b200.nvfp4")


def tile_layout(scales_rowmajor: np.ndarray) -> np.ndarray:
    """[M, B] scale bytes -> the 128 x 4 tile layout, zero-padded."""
    M, B = scales_rowmajor.shape
    R, C = -(-M // 128) * 128, -(-B // 4) * 4
    out = np.zeros(R * C, dtype=np.uint8)
    for r in range(M):
        for c in range(B):
            tile = (r // 128) * (C // 4) + c // 4
            out[tile * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4] = scales_rowmajor[r, c]
    return out


@pytest.mark.parametrize("M,N", [(1, 16), (256, 1024), (130, 4112), (300, 40), (129, 65)])
def test_mma_scales_are_the_tile_permutation(M, N):
    rng = np.random.default_rng(M * 3 + N)
    x = synthetic.to_bf16_bits(rng.standard_t(3, (M, N)).astype(np.float32))
    xd = to_dev(x)
    a = nv.nvfp4_amax(xd)
    packed_mma, scales_mma, gs = nv.nvfp4_quantize_mma(xd, a)
    packed, scales = oracle_quantize_rows(x, oracle.global_scale(a.item()))
    assert_equal_bits(u8(packed_mma), packed, f"{M}x{N} packed")
    assert_equal_bits(u8(scales_mma), tile_layout(scales), f"{M}x{N} tile-layout scales")


def _decoded(x_bits, amax):
    """Operand values as the GEMM sees them, in float64: LUT[code] * E4M3(byte) / gs."""
    gs = oracle.global_scale(amax)
    packed, scales = oracle_quantize_rows(x_bits, gs)
    M, N = x_bits.shape
    codes = np.empty((M, packed.shape[1] * 2), dtype=np.uint8)
    codes[:, 0::2], codes[:, 1::2] = packed & 15, packed >> 4
    lut = np.array([oracle.e2m1_lut(c) for c in range(16)], dtype=np.float64)
    dec = oracle.e4m3_decode(scales).astype(np.float64)
    return lut[codes] * np.repeat(dec, 16, axis=1) / np.float64(np.float32(gs))


@pytest.mark.parametrize("M,N,K", [(256, 384, 1024), (128, 256, 4096), (200, 144, 544)])
def test_mma_scales_feed_the_block_scaled_gemm(M, N, K):
    rng = np.random.default_rng(M + N + K)
    a_bits = synthetic.to_bf16_bits(rng.standard_t(3, (M, K)).astype(np.float32))
    w_bits = synthetic.to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02))
    ad, wd = to_dev(a_bits), to_dev(w_bits)
    amax_a, amax_w = nv.nvfp4_amax(ad), nv.nvfp4_amax(wd)
    pa, sa, ga = nv.nvfp4_quantize_mma(ad, amax_a)
    pw, sw, gw = nv.nvfp4_quantize_mma(wd, amax_w)

    def gemm(sa_, sw_):
        return F.scaled_mm(pa.view(torch.float4_e2m1fn_x2), pw.view(torch.float4_e2m1fn_x2).t(),
                           [sa_.view(torch.float8_e4m3fn), (1.0 / ga).reshape(())],
                           [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                           [sw_.view(torch.float8_e4m3fn), (1.0 / gw).reshape(())],
                           [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                           swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE],
                           swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE],
                           output_dtype=torch.bfloat16).float().cpu().numpy().astype(np.float64)

    A = _decoded(a_bits, amax_a.item())
    W = _decoded(w_bits, amax_w.item())
    ref = A @ W.T
    bound = np.abs(ref) * 2.0 ** -8 + (np.abs(A) @ np.abs(W).T) * K * 2.0 ** -23 + 1e-30
    got = gemm(sa, sw)
    assert np.all(np.abs(got - ref) <= bound), f"max rel err {np.max(np.abs(got - ref) / bound):.3g} x bound"
    # negative control: the same scale bytes in row-major order are not what the GEMM reads
    rowmajor = [nv.nvfp4_quantize(t, am)[1] for t, am in ((ad, amax_a), (wd, amax_w))]
    pad = [torch.zeros_like(sa), torch.zeros_like(sw)]
    pad[0][:rowmajor[0].numel()] = rowmajor[0].view(-1)
    pad[1][:rowmajor[1].numel()] = rowmajor[1].view(-1)
    bad = gemm(pad[0], pad[1])
    assert not np.all(np.abs(bad - ref) <= bound)
